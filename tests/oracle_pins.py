"""Pins of the oracle: facts fixed by the pages and by mathematics.

Each ``pin_*`` function takes an :class:`oracle.Oracle` and raises on the first
violated fact. They are collected by ``test_oracle_pins.py`` (against the
committed oracle) and by ``test_oracle_mutants.py`` (against copies of the
oracle with a planted mistake, each of which must fail at least one pin).

No expected value here is produced by the oracle itself: each comes from the
pages (``tests/golden``), a closed form, a library routine (numpy, torch CPU in
fp64), exact rational arithmetic, or an invariant that holds exactly.
"""
from __future__ import annotations

import os
import sys
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

U32 = 2.0 ** -24  # unit roundoff of f32


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _fixed_offsets(F, B, L):
    return np.broadcast_to((np.arange(B) * L).astype(np.int32), (F, B)).copy()


def _rand_case(seed, B, F, N, D, L):
    rng = np.random.default_rng(seed)
    ws = [rng.normal(0.0, 0.1, size=(N, D)).astype(np.float32) for _ in range(F)]
    idx = rng.integers(0, N, size=(F, B * L)).astype(np.int32)
    dense = rng.normal(0.0, 1.0, size=(B, D)).astype(np.float32)
    return ws, idx, _fixed_offsets(F, B, L), dense


def _dyadic_table(rng, N, D):
    # k/256 with |k| < 128: every sum of up to 2^16 such values is exact in f32
    return (rng.integers(-127, 128, size=(N, D)) / 256.0).astype(np.float32)


def _expect_code(fn, code):
    from oracle import OracleError

    try:
        fn()
    except OracleError as e:  # noqa: PERF203
        assert e.code == code, f"expected oracle code {code}, got {e.code}"
        return
    raise AssertionError(f"oracle accepted an input it must reject (code {code})")


# --------------------------------------------------------------------------- pairs

def pin_pair_order_golden(orc):
    """The first pairs the pages print, (1,0), (2,0), (2,1)."""
    rows = _golden_rows("pair_order_head.txt")
    for nf in (3, 4, 9, 33):
        pi, pj = orc.pair_list(nf)
        for p, i, j in rows:
            assert (pi[int(p)], pj[int(p)]) == (int(i), int(j)), (nf, p)


def pin_pair_count_golden(orc):
    """528 dots at num_cat = 32 (F = 33 features), in both output layouts."""
    kv = {k: int(v) for k, v in _golden_rows("pairs_at_num_cat_32.txt")}
    F = kv["num_cat"]
    assert F + 1 == kv["features"]
    assert (kv["features"] - 1) // 2 == kv["reread_factor"]
    dense = np.ones((2, 3), np.float32)
    emb = np.ones((2, F, 3), np.float32)
    assert orc.interact_lower_tri(dense, emb).shape == (2, kv["pairs"])
    assert orc.interact_lower_tri(dense, emb, concat_dense=True).shape == (2, 3 + kv["pairs"])
    pi, _ = orc.pair_list(kv["features"])
    assert len(pi) == kv["pairs"]


def pin_pair_list_is_tril_indices(orc):
    """The pair table equals numpy's tril_indices(nf, -1) for every nf up to 129."""
    for nf in range(1, 130):
        pi, pj = orc.pair_list(nf)
        ri, rj = np.tril_indices(nf, -1)
        assert np.array_equal(pi, ri) and np.array_equal(pj, rj), nf


def pin_interaction_identifies_pairs(orc):
    """With D=1 and feature m equal to the m-th prime, dot p is prime_i * prime_j.

    The factorisation is unique, so this fixes which two features (dense first,
    then tables in order) every output column multiplies.
    """
    primes = [2, 3, 5, 7, 11, 13, 17, 19, 23, 29, 31, 37, 41, 43, 47, 53, 59, 61, 67, 71,
              73, 79, 83, 89, 97, 101, 103, 107, 109, 113, 127, 131, 137]
    for F in (1, 2, 5, 32):
        B = 3
        c = np.array(primes[: F + 1], dtype=np.float32)
        dense = np.tile(c[0], (B, 1)).astype(np.float32) * np.arange(1, B + 1)[:, None]
        emb = np.tile(c[1:], (B, 1))[:, :, None].astype(np.float32)
        z = orc.interact_lower_tri(dense, emb)
        ri, rj = np.tril_indices(F + 1, -1)
        for b in range(B):
            feat = np.concatenate([[c[0] * (b + 1)], c[1:]])
            want = (feat[ri] * feat[rj]).astype(np.float32)
            assert np.array_equal(z[b], want), (F, b)


def pin_interaction_vs_torch_bmm(orc):
    """Dots equal torch's cat -> bmm(T, T^T) -> tril gather, taken in fp64."""
    for seed, (B, F, D) in enumerate([(3, 5, 7), (2, 1, 16), (4, 12, 33)]):
        _, _, _, dense = _rand_case(seed, B, 1, 1, D, 1)
        emb = np.random.default_rng(100 + seed).normal(0, 0.3, (B, F, D)).astype(np.float32)
        T = torch.cat([torch.from_numpy(dense).double().unsqueeze(1),
                       torch.from_numpy(emb).double()], dim=1)
        Z = torch.bmm(T, T.transpose(1, 2))
        li, lj = torch.tril_indices(F + 1, F + 1, -1)
        ref = Z[:, li, lj].numpy()
        z32, z64, bound = orc.interact_lower_tri(dense, emb, with_f64=True)
        assert np.all(np.abs(z64 - ref) <= 1e-13 * bound + 1e-300), (B, F, D)
        assert np.array_equal(z32, ref.astype(np.float32)) or \
            np.all(np.abs(z32 - ref) <= U32 * np.abs(ref) + 1e-13 * bound)
        # S_ij is the sum of |v_i v_j|, which bounds |z| and equals it for v_i = v_j
        absT = T.abs()
        Sref = torch.bmm(absT, absT.transpose(1, 2))[:, li, lj].numpy()
        assert np.allclose(bound, Sref, rtol=1e-12, atol=0)


def pin_interaction_exact_rational(orc):
    """Brute force on tiny inputs with exact rationals: fp64 within gamma_D, f32 within 1 ulp."""
    rng = np.random.default_rng(7)
    B, F, D = 2, 3, 5
    dense = rng.normal(0, 1, (B, D)).astype(np.float32)
    emb = rng.normal(0, 1, (B, F, D)).astype(np.float32)
    z32, z64, _ = orc.interact_lower_tri(dense, emb, with_f64=True)
    for b in range(B):
        feats = [dense[b]] + [emb[b, k] for k in range(F)]
        p = 0
        for i in range(1, F + 1):
            for j in range(i):
                prods = [Fraction(float(x)) * Fraction(float(y))
                         for x, y in zip(feats[i], feats[j])]
                exact = sum(prods)
                # fp64 summation of D exact products: error <= D * 2^-53 * sum|prod|
                bound64 = Fraction(D, 2 ** 53) * sum(abs(t) for t in prods)
                assert abs(Fraction(float(z64[b, p])) - exact) <= bound64, (b, p)
                ulp = np.spacing(np.float32(abs(float(exact)) or 1e-38))
                assert abs(Fraction(float(z32[b, p])) - exact) <= Fraction(float(ulp)), (b, p)
                p += 1


def pin_concat_layout(orc):
    """With concat, row b is [dense[b] | dots of b], both parts bit-exact."""
    _, _, _, dense = _rand_case(3, 4, 1, 1, 6, 1)
    emb = np.random.default_rng(4).normal(0, 1, (4, 3, 6)).astype(np.float32)
    z = orc.interact_lower_tri(dense, emb)
    zc = orc.interact_lower_tri(dense, emb, concat_dense=True)
    assert zc.shape == (4, 6 + 6)
    assert np.array_equal(zc[:, :6].view(np.uint32), dense.view(np.uint32))
    assert np.array_equal(zc[:, 6:].view(np.uint32), z.view(np.uint32))


def pin_scale_dense(orc):
    """Doubling dense doubles exactly the dots that involve feature 0, nothing else."""
    _, _, _, dense = _rand_case(5, 3, 1, 1, 9, 1)
    emb = np.random.default_rng(6).normal(0, 1, (3, 4, 9)).astype(np.float32)
    z = orc.interact_lower_tri(dense, emb)
    z2 = orc.interact_lower_tri(dense * np.float32(2), emb)
    _, rj = np.tril_indices(5, -1)
    assert np.array_equal(z2[:, rj == 0], z[:, rj == 0] * np.float32(2))
    assert np.array_equal(z2[:, rj != 0], z[:, rj != 0])


# --------------------------------------------------------------------------- pooled sums

def pin_embbag_vs_torch(orc):
    """Pooled sums equal torch.nn.functional.embedding_bag(mode='sum') in fp64.

    Covers ragged bags (offsets not a fixed stride), empty bags and tables with
    different row counts.
    """
    rng = np.random.default_rng(11)
    B, F, D, L = 6, 3, 5, 4
    rows = [7, 13, 5]
    ws = [rng.normal(0, 0.1, (rows[k], D)).astype(np.float32) for k in range(F)]
    idx = np.stack([rng.integers(0, rows[k], B * L) for k in range(F)]).astype(np.int32)
    offs = np.array([[0, 4, 8, 12, 16, 20],
                     [0, 0, 3, 10, 10, 23],
                     [0, 1, 2, 3, 24, 24]], dtype=np.int32)
    out, o64, absum = orc.embbag_sum_multi(ws, idx, offs, B, L, with_f64=True)
    for k in range(F):
        ref = torch.nn.functional.embedding_bag(
            torch.from_numpy(idx[k]).long(), torch.from_numpy(ws[k]).double(),
            torch.from_numpy(offs[k]).long(), mode="sum").numpy()
        assert np.allclose(o64[:, k, :], ref, rtol=1e-14, atol=1e-300), k
        n_in_bag = np.diff(np.append(offs[k], B * L))
        tol = (n_in_bag[:, None] * U32) * absum[:, k, :]
        assert np.all(np.abs(out[:, k, :] - ref) <= tol), k


def pin_embbag_sequential_order(orc):
    """The f32 pooled sum accumulates from 0 in bag order, one rounding per add.

    With rows 1.0 and 2^-24: in bag order [1, t, t] each add of t ties back to
    1.0 (round half to even), so the sum is exactly 1.0; in order [t, t, 1] the
    two small terms first make 2^-23 and the sum is 1 + 2^-23.
    """
    W = np.array([[1.0], [2.0 ** -24]], dtype=np.float32)
    idx = np.array([[0, 1, 1, 1, 1, 0]], dtype=np.int32)
    offs = np.array([[0, 3]], dtype=np.int32)
    out = orc.embbag_sum_multi([W], idx, offs, 2, 3)
    assert out[0, 0, 0] == np.float32(1.0)
    assert out[1, 0, 0] == np.float32(1.0 + 2.0 ** -23)


def pin_l_copies(orc):
    """A bag of L copies of row r pools to exactly L * W[r] on dyadic tables."""
    rng = np.random.default_rng(12)
    for L in (1, 4, 20, 33):
        N, D, B, F = 9, 6, 5, 2
        ws = [_dyadic_table(rng, N, D) for _ in range(F)]
        r = rng.integers(0, N, size=(F, B))
        idx = np.repeat(r, L, axis=1).astype(np.int32)
        out = orc.embbag_sum_multi(ws, idx, _fixed_offsets(F, B, L), B, L)
        for k in range(F):
            assert np.array_equal(out[:, k, :], ws[k][r[k]] * np.float32(L)), (L, k)


def pin_one_hot_tables(orc):
    """Row r of a one-hot table is e_(r mod D): pooled values are index counts.

    The counts come from numpy's bincount and the dots from an integer einsum,
    so both parts of the stage are checked exactly.
    """
    rng = np.random.default_rng(13)
    B, F, N, D, L = 7, 4, 50, 8, 10
    eye = np.eye(D, dtype=np.float32)
    ws = [eye[np.arange(N) % D] for _ in range(F)]
    idx = rng.integers(0, N, size=(F, B * L)).astype(np.int32)
    pooled = orc.embbag_sum_multi(ws, idx, _fixed_offsets(F, B, L), B, L)
    counts = np.zeros((B, F, D), dtype=np.int64)
    for k in range(F):
        for b in range(B):
            counts[b, k] = np.bincount(idx[k, b * L:(b + 1) * L] % D, minlength=D)
    assert np.array_equal(pooled, counts.astype(np.float32))
    dense_i = rng.integers(-3, 4, size=(B, D))
    z = orc.interact_lower_tri(dense_i.astype(np.float32), pooled)
    feats = np.concatenate([dense_i[:, None, :], counts], axis=1)
    gram = np.einsum("bid,bjd->bij", feats, feats)
    ri, rj = np.tril_indices(F + 1, -1)
    assert np.array_equal(z, gram[:, ri, rj].astype(np.float32))


def pin_brute_force_tiny(orc):
    """Tiny random case against exact rational sums (pooled) in plain Python."""
    rng = np.random.default_rng(14)
    B, F, N, D, L = 3, 2, 6, 4, 3
    ws = [rng.normal(0, 0.1, (N, D)).astype(np.float32) for _ in range(F)]
    idx = rng.integers(0, N, size=(F, B * L)).astype(np.int32)
    out = orc.embbag_sum_multi(ws, idx, _fixed_offsets(F, B, L), B, L)
    for b in range(B):
        for k in range(F):
            for d in range(D):
                terms = [float(ws[k][idx[k, b * L + l], d]) for l in range(L)]
                exact = sum(Fraction(t) for t in terms)
                bound = Fraction(L) * Fraction(U32) * sum(abs(Fraction(t)) for t in terms)
                assert abs(Fraction(float(out[b, k, d])) - exact) <= bound, (b, k, d)


def pin_bag_permutation(orc):
    """Permuting entries inside bags leaves dyadic pooled sums bit-identical."""
    rng = np.random.default_rng(15)
    B, F, N, D, L = 4, 3, 11, 5, 7
    ws = [_dyadic_table(rng, N, D) for _ in range(F)]
    idx = rng.integers(0, N, size=(F, B * L)).astype(np.int32)
    perm = idx.reshape(F, B, L)[:, :, rng.permutation(L)].reshape(F, B * L)
    offs = _fixed_offsets(F, B, L)
    a = orc.embbag_sum_multi(ws, idx, offs, B, L)
    b = orc.embbag_sum_multi(ws, np.ascontiguousarray(perm), offs, B, L)
    assert np.array_equal(a, b)


def pin_swap_tables(orc):
    """Swapping two tables (with their indices) swaps their pooled slots and dots."""
    ws, idx, offs, dense = _rand_case(16, 3, 3, 10, 4, 5)
    pooled, inter = orc.sparse_interact(ws, idx, offs, dense, 3, 5)
    ws2 = [ws[1], ws[0], ws[2]]
    idx2 = np.ascontiguousarray(idx[[1, 0, 2]])
    pooled2, inter2 = orc.sparse_interact(ws2, idx2, offs, dense, 3, 5)
    assert np.array_equal(pooled2, pooled[:, [1, 0, 2], :])
    # feature m of the swapped run is feature sigma(m) of the original
    sigma = [0, 2, 1, 3]
    ri, rj = np.tril_indices(4, -1)
    col = {(int(i), int(j)): p for p, (i, j) in enumerate(zip(ri, rj))}
    for p, (i, j) in enumerate(zip(ri, rj)):
        a, b = sigma[i], sigma[j]
        q = col[(max(a, b), min(a, b))]
        assert np.array_equal(inter2[:, p], inter[:, q]), (i, j)


def pin_empty_bags_are_positive_zero(orc):
    """An empty bag (L = 0, or equal consecutive offsets) pools to +0.0."""
    rng = np.random.default_rng(17)
    ws = [rng.normal(0, 1, (4, 3)).astype(np.float32)]
    out = orc.embbag_sum_multi(ws, np.zeros((1, 0), np.int32), np.zeros((1, 5), np.int32), 5, 0)
    assert np.array_equal(out.view(np.uint32), np.zeros((5, 1, 3), np.uint32))
    idx = np.array([[1, 2, 3, 0]], dtype=np.int32)
    out = orc.embbag_sum_multi(ws, idx, np.array([[0, 2, 2, 4]], np.int32), 4, 1)
    assert np.array_equal(out[1].view(np.uint32), np.zeros((1, 3), np.uint32))
    assert np.array_equal(out[3].view(np.uint32), np.zeros((1, 3), np.uint32))
    assert np.array_equal(out[2, 0], ws[0][3] + ws[0][0])


def pin_rejects_bad_input(orc):
    """Offsets out of order or range, indices outside [0, rows), bad shapes."""
    from oracle import BAD_ARG, BAD_OFFSETS, INDEX_OOB

    ws = [np.zeros((5, 2), np.float32), np.zeros((3, 2), np.float32)]
    good_idx = np.array([[0, 1, 2, 3], [0, 1, 2, 0]], np.int32)
    offs = _fixed_offsets(2, 2, 2)
    orc.embbag_sum_multi(ws, good_idx, offs, 2, 2)
    for bad in ([[2, 1], [0, 2]], [[-1, 2], [0, 2]], [[0, 5], [0, 2]], [[0, 2], [3, 2]]):
        _expect_code(lambda: orc.embbag_sum_multi(ws, good_idx, np.array(bad, np.int32), 2, 2),
                     BAD_OFFSETS)
    for bad in ([[0, 1, 2, 5], [0, 1, 2, 0]], [[0, 1, 2, 3], [0, 3, 2, 0]],
                [[0, -1, 2, 3], [0, 1, 2, 0]]):
        _expect_code(lambda: orc.embbag_sum_multi(ws, np.array(bad, np.int32), offs, 2, 2),
                     INDEX_OOB)
    _expect_code(lambda: orc.embbag_sum_multi(ws, good_idx, offs, 2, -1), BAD_ARG)
    dense = np.zeros((2, 2), np.float32)
    _expect_code(lambda: orc.interact_lower_tri(dense, np.zeros((2, 257, 2), np.float32)),
                 BAD_ARG)


# --------------------------------------------------------------------------- general pooling

def _ragged(rng, F, B, T, ilo):
    off = np.sort(rng.integers(0, T + 1, (F, B + (1 if ilo else 0))), axis=1).astype(np.int32)
    off[:, 0] = 0
    if ilo:
        off[:, -1] = T
    return off


def _torch_bag(idx_k, w_k, off_k, mode, psw_k=None, ilo=False):
    return torch.nn.functional.embedding_bag(
        torch.from_numpy(idx_k).long(), torch.from_numpy(w_k), torch.from_numpy(off_k).long(),
        mode=mode, per_sample_weights=None if psw_k is None else torch.from_numpy(psw_k),
        include_last_offset=ilo).numpy()


def pin_pool_modes_vs_torch(orc):
    """sum / mean / max, ragged bags, both offset conventions, against torch.

    Sums and means are compared with torch in fp64 within the f32 error of a
    sequential sum; max is exact in any precision, so it is compared bit for
    bit with torch's f32 max mode.
    """
    rng = np.random.default_rng(21)
    B, F, N, D, T = 9, 3, 40, 6, 50
    ws = [rng.normal(0, 0.1, (N, D)).astype(np.float32) for _ in range(F)]
    idx = rng.integers(0, N, (F, T)).astype(np.int32)
    for ilo in (False, True):
        off = _ragged(rng, F, B, T, ilo)
        for mode in ("sum", "mean", "max"):
            out = orc.embbag_pool_multi(ws, idx, off, B, mode=mode, include_last_offset=ilo)
            for k in range(F):
                if mode == "max":
                    ref = _torch_bag(idx[k], ws[k], off[k], "max", ilo=ilo)
                    assert np.array_equal(out[:, k], ref), (ilo, mode, k)
                    continue
                ref = _torch_bag(idx[k], ws[k].astype(np.float64), off[k], mode, ilo=ilo)
                ends = off[k, 1:] if ilo else np.append(off[k, 1:], T)
                n = (ends - off[k, :B]).astype(np.float64)
                absum = _torch_bag(idx[k], np.abs(ws[k]).astype(np.float64), off[k], "sum",
                                   ilo=ilo)
                scale = absum / np.maximum(n, 1)[:, None] if mode == "mean" else absum
                tol = (n[:, None] + 1) * U32 * scale
                assert np.all(np.abs(out[:, k] - ref) <= tol), (ilo, mode, k)


def pin_weighted_sum_vs_torch(orc):
    """per_sample_weights: sum_t w_t * W[idx_t] against torch in fp64."""
    rng = np.random.default_rng(22)
    B, F, N, D, T = 7, 2, 30, 5, 40
    ws = [rng.normal(0, 0.1, (N, D)).astype(np.float32) for _ in range(F)]
    idx = rng.integers(0, N, (F, T)).astype(np.int32)
    psw = rng.normal(1.0, 0.5, (F, T)).astype(np.float32)
    off = _ragged(rng, F, B, T, False)
    out = orc.embbag_pool_multi(ws, idx, off, B, per_sample_weights=psw)
    for k in range(F):
        ref = _torch_bag(idx[k], ws[k].astype(np.float64), off[k], "sum",
                         psw[k].astype(np.float64))
        absum = _torch_bag(idx[k], np.abs(ws[k]).astype(np.float64), off[k], "sum",
                           np.abs(psw[k]).astype(np.float64))
        n = np.diff(np.append(off[k], T)).astype(np.float64)
        assert np.all(np.abs(out[:, k] - ref) <= (n[:, None] + 1) * U32 * absum), k


def pin_weighted_sum_exact_cases(orc):
    """Unit weights give the plain sum bit for bit; dyadic weights are exact."""
    rng = np.random.default_rng(23)
    B, F, N, D, L = 6, 2, 20, 4, 5
    ws = [rng.normal(0, 0.1, (N, D)).astype(np.float32) for _ in range(F)]
    idx = rng.integers(0, N, (F, B * L)).astype(np.int32)
    off = _fixed_offsets(F, B, L)
    plain = orc.embbag_pool_multi(ws, idx, off, B)
    ones = orc.embbag_pool_multi(ws, idx, off, B, per_sample_weights=np.ones((F, B * L)))
    assert np.array_equal(plain.view(np.uint32), ones.view(np.uint32))
    assert np.array_equal(plain, orc.embbag_sum_multi(ws, idx, off, B, L))
    dy = [_dyadic_table(rng, N, D) for _ in range(F)]
    wts = (2.0 ** rng.integers(-3, 4, (F, B * L))).astype(np.float32)
    out = orc.embbag_pool_multi(dy, idx, off, B, per_sample_weights=wts)
    for b in range(B):
        for k in range(F):
            sl = slice(b * L, (b + 1) * L)
            exact = sum(Fraction(float(wt)) * np.vectorize(Fraction)(dy[k][r].astype(np.float64))
                        for wt, r in zip(wts[k, sl], idx[k, sl]))
            assert all(Fraction(float(o)) == e for o, e in zip(out[b, k], exact)), (b, k)


def pin_weighted_sum_rounds_once_per_entry(orc):
    """Each weighted entry is one fused multiply-add: with w = x = 1 + 2^-12 after a
    -1, the exact w*x - 1 = 2^-11 + 2^-24 is an f32 and must come out whole (a
    rounded product first would lose the 2^-24)."""
    a = 1.0 + 2.0 ** -12
    tab = np.array([[-1.0], [a]], np.float32)
    idx = np.array([[0, 1]], np.int32)
    off = np.zeros((1, 1), np.int32)
    wts = np.array([[1.0, a]], np.float32)
    out = orc.embbag_pool_multi([tab], idx, off, 1, per_sample_weights=wts)
    exact = Fraction(a) * Fraction(a) - 1
    assert exact == Fraction(2) ** -11 + Fraction(2) ** -24
    assert Fraction(float(out[0, 0, 0])) == exact


def pin_mean_divides_once(orc):
    """Mean is the f32 sum divided once by the count: entries 2, 2, 1 give the
    f32 nearest 5/3 (0x3FD55555), not 5 times the f32 nearest 1/3."""
    tab = np.array([[2.0], [1.0]], np.float32)
    idx = np.array([[0, 0, 1]], np.int32)
    off = np.zeros((1, 1), np.int32)
    out = orc.embbag_pool_multi([tab], idx, off, 1, mode="mean")
    assert out.view(np.uint32)[0, 0, 0] == 0x3FD55555
    assert np.float32(5.0) * np.float32(1.0 / 3.0) != out[0, 0, 0]  # the case tells them apart


def pin_mean_and_max_closed_forms(orc):
    """Mean of L copies of a dyadic row is the row; max equals numpy's maximum."""
    rng = np.random.default_rng(24)
    B, F, N, D, L = 5, 3, 12, 7, 6
    dy = [_dyadic_table(rng, N, D) for _ in range(F)]
    r = rng.integers(0, N, (F, B))
    idx = np.repeat(r, L, axis=1).astype(np.int32)
    off = _fixed_offsets(F, B, L)
    mean = orc.embbag_pool_multi(dy, idx, off, B, mode="mean")
    for k in range(F):
        assert np.array_equal(mean[:, k], dy[k][r[k]]), k
    ws = [rng.normal(0, 1, (N, D)).astype(np.float32) for _ in range(F)]
    idx = rng.integers(0, N, (F, B * L)).astype(np.int32)
    mx = orc.embbag_pool_multi(ws, idx, off, B, mode="max")
    for k in range(F):
        ref = ws[k][idx[k]].reshape(B, L, D).max(axis=1)
        assert np.array_equal(mx[:, k], ref), k
    # empty bags give 0 in every mode
    zoff = np.zeros((F, B), np.int32)
    for mode in ("sum", "mean", "max"):
        z = orc.embbag_pool_multi(ws, np.zeros((F, 0), np.int32), zoff, B, mode=mode)
        assert np.array_equal(z.view(np.uint32), np.zeros_like(z).view(np.uint32)), mode


def pin_max_ties_keep_the_earlier_entry(orc):
    """Max pooling keeps the first entry, then takes x only when x > acc, so a
    tie keeps the entry seen first: of -0.0 and +0.0 the earlier survives."""
    tab = np.array([[-0.0, 0.0, 1.0], [0.0, -0.0, 1.0]], np.float32)
    idx = np.array([[0, 1, 1, 0]], np.int32)      # bag 0: rows 0, 1; bag 1: rows 1, 0
    off = np.array([[0, 2]], np.int32)
    mx = orc.embbag_pool_multi([tab], idx, off, 2, mode="max")
    bits = mx.view(np.uint32)
    assert bits[0, 0, 0] == 0x80000000 and bits[0, 0, 1] == 0          # -0 then +0 -> -0
    assert bits[1, 0, 0] == 0 and bits[1, 0, 1] == 0x80000000          # +0 then -0 -> +0
    assert mx[0, 0, 2] == 1.0 and mx[1, 0, 2] == 1.0


def pin_bf16_tables_widen_exactly(orc):
    """bf16 tables pool exactly like their f32 widening (done by torch)."""
    rng = np.random.default_rng(25)
    B, F, N, D, T = 8, 2, 25, 6, 30
    tb = [torch.from_numpy(rng.normal(0, 0.3, (N, D)).astype(np.float32)).bfloat16()
          for _ in range(F)]
    bits = [t.view(torch.int16).numpy().view(np.uint16) for t in tb]
    wide = [t.float().numpy() for t in tb]
    idx = rng.integers(0, N, (F, T)).astype(np.int32)
    off = _ragged(rng, F, B, T, False)
    psw = rng.normal(0, 1, (F, T)).astype(np.float32)
    for mode, p in (("sum", None), ("sum", psw), ("mean", None), ("max", None)):
        a = orc.embbag_pool_multi(bits, idx, off, B, mode=mode, per_sample_weights=p)
        b = orc.embbag_pool_multi(wide, idx, off, B, mode=mode, per_sample_weights=p)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), mode


def pin_general_pooling_rejects(orc):
    """Weights outside sum mode, bad offsets and covered out-of-range indices."""
    from oracle import BAD_ARG, BAD_OFFSETS, INDEX_OOB

    ws = [np.zeros((5, 2), np.float32)]
    idx = np.array([[0, 1, 2, 3, 99]], np.int32)  # entry 4 lies in no bag
    off = np.array([[0, 2, 4]], np.int32)
    orc.embbag_pool_multi(ws, idx, off, 2, include_last_offset=True)
    _expect_code(lambda: orc.embbag_pool_multi(ws, idx, off[:, :2], 2), INDEX_OOB)
    _expect_code(lambda: orc.embbag_pool_multi(ws, np.array([[0, 5, 2, 3, 0]], np.int32), off, 2,
                                               include_last_offset=True), INDEX_OOB)
    _expect_code(lambda: orc.embbag_pool_multi(ws, np.array([[0, 1, -1, 3, 0]], np.int32), off,
                                               2, include_last_offset=True), INDEX_OOB)
    _expect_code(lambda: orc.embbag_pool_multi(ws, idx, np.array([[0, 3, 2]], np.int32), 2,
                                               include_last_offset=True), BAD_OFFSETS)
    _expect_code(lambda: orc.embbag_pool_multi(ws, idx, off, 2, include_last_offset=True,
                                               mode="mean",
                                               per_sample_weights=np.ones((1, 5))), BAD_ARG)


# ---------------------------------------------------------------------------
# The MLP layer: act(A W^T + bias) over bf16 operands (matmul2d.rs page,
# linear_bias / _relu / _sigmoid and the split-A forms).


def _bf16_bits(x):
    """bf16 bit patterns of an array (torch's round-to-nearest-even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _bf16_values(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def pin_linear_exact_integers(orc):
    """Small-integer operands: the layer is an exact integer matmul (numpy int64)."""
    rng = np.random.default_rng(71)
    for (M, N, K) in [(1, 1, 1), (3, 5, 7), (17, 9, 40)]:
        a = rng.integers(-8, 9, size=(M, K))
        w = rng.integers(-8, 9, size=(N, K))
        b = rng.integers(-50, 51, size=N)
        out, pre, bound = orc.linear_bf16(_bf16_bits(a), _bf16_bits(w), b.astype(np.float32))
        want = a.astype(np.int64) @ w.astype(np.int64).T + b
        assert np.array_equal(pre, want.astype(np.float64))
        assert np.array_equal(out, want.astype(np.float64))
        wantb = np.abs(a).astype(np.int64) @ np.abs(w).astype(np.int64).T + np.abs(b)
        assert np.array_equal(bound, wantb.astype(np.float64))


def pin_linear_vs_torch_fp64(orc):
    """Random bf16 operands against torch.nn.functional.linear in fp64."""
    rng = np.random.default_rng(72)
    for (M, N, K) in [(4, 3, 16), (33, 20, 100)]:
        a = _bf16_bits(rng.normal(0, 1, size=(M, K)))
        w = _bf16_bits(rng.normal(0, 0.1, size=(N, K)))
        b = rng.normal(0, 0.1, size=N).astype(np.float32)
        ta = torch.from_numpy(_bf16_values(a).astype(np.float64))
        tw = torch.from_numpy(_bf16_values(w).astype(np.float64))
        tb = torch.from_numpy(b.astype(np.float64))
        want = torch.nn.functional.linear(ta, tw, tb).numpy()
        out, _, bound = orc.linear_bf16(a, w, b, 0)
        assert np.all(np.abs(out - want) <= 1e-12 * bound + 1e-300)
        out, _, _ = orc.linear_bf16(a, w, None, 0)
        want0 = torch.nn.functional.linear(ta, tw).numpy()
        assert np.all(np.abs(out - want0) <= 1e-12 * bound + 1e-300)


def pin_linear_activations(orc):
    """ReLU is torch.relu and sigmoid is scipy's expit of the pre-activation."""
    from scipy.special import expit

    rng = np.random.default_rng(73)
    a = _bf16_bits(rng.normal(0, 1, size=(9, 24)))
    w = _bf16_bits(rng.normal(0, 0.5, size=(7, 24)))
    b = rng.normal(0, 0.5, size=7).astype(np.float32)
    _, pre, _ = orc.linear_bf16(a, w, b, 0)
    relu, pre1, _ = orc.linear_bf16(a, w, b, 1)
    sig, pre2, _ = orc.linear_bf16(a, w, b, 2)
    assert np.array_equal(pre, pre1) and np.array_equal(pre, pre2)
    assert (pre < 0).any() and (pre > 0).any()
    assert np.array_equal(relu, torch.relu(torch.from_numpy(pre)).numpy())
    assert np.allclose(sig, expit(pre), rtol=1e-15, atol=0)


def pin_linear_split_equals_concat(orc):
    """Split A (columns from two sources) equals the layer on the concatenation,
    and the weight's column k_lo + k multiplies a_hi's column k."""
    rng = np.random.default_rng(74)
    M, N, k_lo, k_hi = 6, 5, 3, 11
    a_lo = _bf16_bits(rng.normal(0, 1, size=(M, k_lo)))
    a_hi = _bf16_bits(rng.normal(0, 1, size=(M, k_hi)))
    w = _bf16_bits(rng.normal(0, 1, size=(N, k_lo + k_hi)))
    b = rng.normal(0, 1, size=N).astype(np.float32)
    cat = np.concatenate([a_lo, a_hi], axis=1)
    for act in (0, 1, 2):
        want = orc.linear_bf16(cat, w, b, act)
        got = orc.linear_bf16(a_lo, w, b, act, a_hi=a_hi)
        for x, y in zip(want, got):
            assert np.array_equal(x, y)
    # one-hot probes: a_hi = e_k picks weight column k_lo + k
    for k in range(k_hi):
        e = np.zeros((1, k_hi), np.float32)
        e[0, k] = 1.0
        _, pre, _ = orc.linear_bf16(np.zeros((1, k_lo), np.uint16), w, None, 0,
                                    a_hi=_bf16_bits(e))
        assert np.array_equal(pre[0], _bf16_values(w[:, k_lo + k]).astype(np.float64))


def pin_linear_row_pitch(orc):
    """Only the first k columns of each pitched row enter the layer."""
    rng = np.random.default_rng(75)
    M, N, K, pad = 4, 3, 5, 3
    a = _bf16_bits(rng.normal(0, 1, size=(M, K)))
    w = _bf16_bits(rng.normal(0, 1, size=(N, K)))
    junk = _bf16_bits(np.full((M, pad), 1e30))
    wjunk = _bf16_bits(np.full((N, pad), -1e30))
    want = orc.linear_bf16(a, w, None, 0)
    got = orc.linear_bf16(np.concatenate([a, junk], 1), np.concatenate([w, wjunk], 1), None, 0,
                          k_lo=K)
    for x, y in zip(want, got):
        assert np.array_equal(x, y)


def pin_linear_rejects(orc):
    from oracle import BAD_ARG

    a = np.zeros((2, 4), np.uint16)
    w = np.zeros((3, 4), np.uint16)
    _expect_code(lambda: orc.linear_bf16(a, w, None, 3), BAD_ARG)
    _expect_code(lambda: orc.linear_bf16(a, np.zeros((3, 3), np.uint16), None, 0), BAD_ARG)
    _expect_code(lambda: orc.linear_bf16(a, w, None, 0, k_lo=5), BAD_ARG)


# ---------------------------------------------------------------------------
# The MLP layer with f32 activations, the pages' own arithmetic (matmul2d.rs:
# A F32 (M, K) times weights BF16 or F32 (N, K), result F32).


def pin_linear_f32a_exact_integers(orc):
    """Integer operands of up to 12 bits (exact in f32 and, for the weights,
    in bf16): the layer is an exact integer matmul, with f32 and bf16 weights."""
    rng = np.random.default_rng(81)
    for (M, N, K) in [(1, 1, 1), (3, 5, 7), (17, 9, 40)]:
        a = rng.integers(-2048, 2049, size=(M, K))
        w = rng.integers(-128, 129, size=(N, K))
        b = rng.integers(-500, 501, size=N)
        want = a.astype(np.int64) @ w.astype(np.int64).T + b
        wantb = np.abs(a).astype(np.int64) @ np.abs(w).astype(np.int64).T + np.abs(b)
        for wt in (w.astype(np.float32), _bf16_bits(w)):
            out, pre, bound = orc.linear_f32a(a.astype(np.float32), wt, b.astype(np.float32))
            assert np.array_equal(pre, want.astype(np.float64))
            assert np.array_equal(out, want.astype(np.float64))
            assert np.array_equal(bound, wantb.astype(np.float64))


def pin_linear_f32a_keeps_every_bit_of_a(orc):
    """Activations with all 24 significant bits enter unrounded, and so do
    f32 weights: (1 + 2^-23)(1 + 2^-7) = 1 + 2^-7 + 2^-23 + 2^-30 exactly (a
    bf16 activation would drop the 2^-23 and 2^-30 terms, an f32 product the
    2^-30 term)."""
    a = np.array([[1.0 + 2.0 ** -23, 3.0 * (1.0 + 2.0 ** -22)]], np.float32)
    w = np.array([[1.0 + 2.0 ** -7, 0.0], [0.0, 1.0 + 2.0 ** -20]], np.float32)
    assert float(a[0, 0]) == 1.0 + 2.0 ** -23
    _, pre, _ = orc.linear_f32a(a, w)
    assert pre[0, 0] == 1.0 + 2.0 ** -7 + 2.0 ** -23 + 2.0 ** -30
    assert pre[0, 1] == 3.0 * (1.0 + 2.0 ** -22) * (1.0 + 2.0 ** -20)
    # the same with the weights' bf16 bit patterns (1 + 2^-7 is a bf16 value)
    _, pre16, _ = orc.linear_f32a(a, _bf16_bits(w[:1]))
    assert pre16[0, 0] == 1.0 + 2.0 ** -7 + 2.0 ** -23 + 2.0 ** -30


def pin_linear_f32a_vs_torch_fp64(orc):
    """Random f32 activations, f32 and bf16 weights, against torch's linear in fp64."""
    rng = np.random.default_rng(82)
    for (M, N, K) in [(4, 3, 16), (33, 20, 100)]:
        a = rng.normal(0, 1, size=(M, K)).astype(np.float32)
        wf = rng.normal(0, 0.1, size=(N, K)).astype(np.float32)
        wb = _bf16_bits(wf)
        b = rng.normal(0, 0.1, size=N).astype(np.float32)
        ta = torch.from_numpy(a.astype(np.float64))
        tb = torch.from_numpy(b.astype(np.float64))
        for w, wvals in ((wf, wf), (wb, _bf16_values(wb))):
            tw = torch.from_numpy(wvals.astype(np.float64))
            want = torch.nn.functional.linear(ta, tw, tb).numpy()
            out, _, bound = orc.linear_f32a(a, w, b, 0)
            assert np.all(np.abs(out - want) <= 1e-12 * bound + 1e-300)
            want0 = torch.nn.functional.linear(ta, tw).numpy()
            out0, _, _ = orc.linear_f32a(a, w, None, 0)
            assert np.all(np.abs(out0 - want0) <= 1e-12 * bound + 1e-300)


def pin_linear_f32a_bf16_weights_are_their_widening(orc):
    """bf16 weight patterns give the layer of their exact f32 widening, and on
    bf16-valued activations the layer equals the bf16-operand layer."""
    rng = np.random.default_rng(83)
    a16 = _bf16_bits(rng.normal(0, 1, size=(7, 12)))
    w16 = _bf16_bits(rng.normal(0, 1, size=(5, 12)))
    b = rng.normal(0, 1, size=5).astype(np.float32)
    for act in (0, 1, 2):
        x = orc.linear_f32a(_bf16_values(a16), w16, b, act)
        y = orc.linear_f32a(_bf16_values(a16), _bf16_values(w16), b, act)
        z = orc.linear_bf16(a16, w16, b, act)
        for u, v, t in zip(x, y, z):
            assert np.array_equal(u, v) and np.array_equal(u, t)


def pin_linear_f32a_activations(orc):
    """ReLU is torch.relu and sigmoid is scipy's expit of the pre-activation."""
    from scipy.special import expit

    rng = np.random.default_rng(84)
    a = rng.normal(0, 1, size=(9, 24)).astype(np.float32)
    w = rng.normal(0, 0.5, size=(7, 24)).astype(np.float32)
    b = rng.normal(0, 0.5, size=7).astype(np.float32)
    _, pre, _ = orc.linear_f32a(a, w, b, 0)
    relu, pre1, _ = orc.linear_f32a(a, w, b, 1)
    sig, pre2, _ = orc.linear_f32a(a, w, b, 2)
    assert np.array_equal(pre, pre1) and np.array_equal(pre, pre2)
    assert (pre < 0).any() and (pre > 0).any()
    assert np.array_equal(relu, torch.relu(torch.from_numpy(pre)).numpy())
    assert np.allclose(sig, expit(pre), rtol=1e-15, atol=0)


def pin_linear_f32a_split_equals_concat(orc):
    """Split A equals the layer on the concatenation; weight column k_lo + k
    multiplies a_hi's column k; only the first k columns of pitched rows count."""
    rng = np.random.default_rng(85)
    M, N, k_lo, k_hi = 6, 5, 3, 11
    a_lo = rng.normal(0, 1, size=(M, k_lo)).astype(np.float32)
    a_hi = rng.normal(0, 1, size=(M, k_hi)).astype(np.float32)
    w = rng.normal(0, 1, size=(N, k_lo + k_hi)).astype(np.float32)
    b = rng.normal(0, 1, size=N).astype(np.float32)
    cat = np.concatenate([a_lo, a_hi], axis=1)
    for act in (0, 1, 2):
        want = orc.linear_f32a(cat, w, b, act)
        got = orc.linear_f32a(a_lo, w, b, act, a_hi=a_hi)
        for x, y in zip(want, got):
            assert np.array_equal(x, y)
    for k in range(k_hi):
        e = np.zeros((1, k_hi), np.float32)
        e[0, k] = 1.0
        _, pre, _ = orc.linear_f32a(np.zeros((1, k_lo), np.float32), w, None, 0, a_hi=e)
        assert np.array_equal(pre[0], w[:, k_lo + k].astype(np.float64))
    junk = np.full((M, 3), 1e30, np.float32)
    wjunk = np.full((N, 3), -1e30, np.float32)
    want = orc.linear_f32a(cat, w, None, 0)
    got = orc.linear_f32a(np.concatenate([cat, junk], 1), np.concatenate([w, wjunk], 1), None, 0,
                          k_lo=k_lo + k_hi)
    for x, y in zip(want, got):
        assert np.array_equal(x, y)


def pin_linear_f32a_rejects(orc):
    from oracle import BAD_ARG

    a = np.zeros((2, 4), np.float32)
    w = np.zeros((3, 4), np.float32)
    _expect_code(lambda: orc.linear_f32a(a, w, None, 3), BAD_ARG)
    _expect_code(lambda: orc.linear_f32a(a, np.zeros((3, 3), np.float32), None, 0), BAD_ARG)
    _expect_code(lambda: orc.linear_f32a(a, w, None, 0, k_lo=5), BAD_ARG)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


def run_all(orc) -> int:
    """Run every pin; print the failures; return how many failed."""
    failed = 0
    for pin in ALL_PINS:
        try:
            pin(orc)
        except Exception as e:  # noqa: BLE001 - a mutant may fail in any way
            failed += 1
            print(f"FAIL {pin.__name__}: {type(e).__name__}: {e}", file=sys.stderr)
    return failed
