"""GPU parity: the CUDA path through the C ABI against the oracle.

Every test here needs a B200 and is marked ``gpu``. Pooled sums, the dense
part of concatenated rows and all index work are compared bit for bit; dots
within 1e-5 * S_ij (see ``gpu_cases``).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from dlrm_embedding_bag_b200 import synthetic as syn
from gpu_cases import (assert_bits_equal, assert_dots_close, check_inter, host_tables,
                       oracle_stage, sampled_oracle)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def ops():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from dlrm_embedding_bag_b200 import ops as _ops

    return _ops


def _inputs(w: syn.Workload):
    weights = syn.make_weights(w, DEV)
    idx = syn.make_indices(w)
    off = syn.make_offsets(w)
    dense = syn.make_dense(w, DEV)
    return weights, idx, off, dense


def _dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(DEV)


def _run_all_paths(ops, weights, idx, off, dense, B, L, concat):
    """Gather, interaction and fused (with/without pooled) on the same input."""
    idx_d, off_d = _dev_i32(idx), _dev_i32(off)
    pooled = ops.embbag_sum_multi(weights, idx_d, off_d, L)
    inter_sep = ops.interact_lower_tri(dense, pooled)
    fp, fi = ops.sparse_interact(weights, idx_d, off_d, dense, L, concat_dense=concat)
    _, fi2 = ops.sparse_interact(weights, idx_d, off_d, dense, L, concat_dense=concat,
                                 want_pooled=False)
    torch.cuda.synchronize()
    return pooled, inter_sep, fp, fi, fi2


def _check_against_oracle(ops, weights, idx, off, dense, B, L, concat, what):
    pooled, inter_sep, fp, fi, fi2 = _run_all_paths(ops, weights, idx, off, dense, B, L, concat)
    ref_p, ref_i, bound = oracle_stage(host_tables(weights), idx, off, dense.cpu().numpy(), B, L,
                                       concat)
    D = dense.shape[1]
    assert_bits_equal(pooled, ref_p, what + " embbag_sum_multi")
    assert_bits_equal(fp, ref_p, what + " fused pooled")
    ref_plain = ref_i[:, D:] if concat else ref_i
    check_inter(inter_sep, ref_plain, bound, D, False, what + " interact_lower_tri")
    check_inter(fi, ref_i, bound, D, concat, what + " fused")
    check_inter(fi2, ref_i, bound, D, concat, what + " fused without pooled")


# ------------------------------------------------------------------ configurations

def test_tiny_config(ops):
    w = syn.TINY
    weights, idx, off, dense = _inputs(w)
    _check_against_oracle(ops, weights, idx, off, dense, w.B, w.L, False, w.name)
    _check_against_oracle(ops, weights, idx, off, dense, w.B, w.L, True, w.name + " concat")


def test_b2048_f8_concat_config(ops):
    w = syn.C2_CONCAT
    weights, idx, off, dense = _inputs(w)
    _check_against_oracle(ops, weights, idx, off, dense, w.B, w.L, w.concat_dense, w.name)


def test_batch_by_table_count_sweep(ops):
    cells = list(syn.sweep())
    w0 = cells[0]
    all_weights = syn.make_weights(w0.scaled(F=max(c.F for c in cells)), DEV)
    for w in cells:
        weights = all_weights[: w.F]
        idx, off = syn.make_indices(w), syn.make_offsets(w)
        dense = syn.make_dense(w, DEV)
        _check_against_oracle(ops, weights, idx, off, dense, w.B, w.L, False, w.name)


@pytest.mark.parametrize("cfg", ["c3", "c3u", "c5"])
def test_full_size_sampled(ops, cfg):
    """Full-size launch (as the benchmark runs it), checked on sampled samples."""
    w = syn.CONFIGS[cfg]
    torch.cuda.empty_cache()
    weights, idx, off, dense = _inputs(w)
    idx_d, off_d = _dev_i32(idx), _dev_i32(off)
    fp, fi = ops.sparse_interact(weights, idx_d, off_d, dense, w.L, concat_dense=w.concat_dense)
    pooled = ops.embbag_sum_multi(weights, idx_d, off_d, w.L)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    samples = np.unique(np.concatenate([[0, w.B - 1], rng.integers(0, w.B, 62)]))
    ref_p, ref_i, bound = sampled_oracle(weights, idx, off, dense, w.B, w.L, samples,
                                         w.concat_dense)
    sel = torch.from_numpy(samples).to(DEV)
    assert_bits_equal(fp[sel], ref_p, w.name + " fused pooled (sampled)")
    assert_bits_equal(pooled[sel], ref_p, w.name + " embbag_sum_multi (sampled)")
    check_inter(fi[sel], ref_i, bound, w.D, w.concat_dense, w.name + " fused (sampled)")
    # the interaction alone on the full-size pooled vectors, same samples
    inter_sep = ops.interact_lower_tri(dense, pooled)
    torch.cuda.synchronize()
    ref_plain = ref_i[:, w.D:] if w.concat_dense else ref_i
    check_inter(inter_sep[sel], ref_plain, bound, w.D, False,
                w.name + " interact_lower_tri (sampled)")
    # properties over every sample: finite, and both paths pool identically
    assert torch.isfinite(fi).all() and torch.isfinite(inter_sep).all()
    assert torch.equal(fp.view(torch.int32), pooled.view(torch.int32))
    del weights, fp, fi, pooled, inter_sep
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,F,D", [(20000, 8, 64), (12000, 8, 128), (70001, 26, 128),
                                   (1500, 32, 64), (37, 59, 64), (3, 25, 128)])
def test_interact_batches_and_table_counts(ops, B, F, D):
    """The interaction alone on batches of many samples per block (a partial
    last group), about one sample per block, F = 59 and a batch smaller than
    one block; checked against the oracle on sampled rows, with the first and
    the last sample always among them."""
    g = torch.Generator(device=DEV)
    g.manual_seed(B + F + D)
    dense = torch.empty((B, D), device=DEV).normal_(0, 1, generator=g)
    emb = torch.empty((B, F, D), device=DEV).normal_(0, 1, generator=g)
    out = ops.interact_lower_tri(dense, emb)
    torch.cuda.synchronize()
    rng = np.random.default_rng(B)
    samples = np.unique(np.concatenate([[0, B - 1], rng.integers(0, B, min(B, 96))]))
    sel = torch.from_numpy(samples).to(DEV)
    ref, _, bound = oracle.interact_lower_tri(dense[sel].cpu().numpy(), emb[sel].cpu().numpy(),
                                              with_f64=True)
    assert_dots_close(out[sel], ref, bound, f"interact B={B} F={F} D={D}")
    assert torch.isfinite(out).all()


# ------------------------------------------------------------------ shapes and edge cases

def _random_case(seed, B, F, N, D, L, ragged=False, empty_frac=0.0):
    rng = np.random.default_rng(seed)
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    weights = [torch.empty((N, D), device=DEV).normal_(0, 0.1, generator=g) for _ in range(F)]
    idx = rng.integers(0, N, (F, B * L)).astype(np.int32)
    if ragged:
        off = np.sort(rng.integers(0, B * L + 1, (F, B)), axis=1).astype(np.int32)
        off[:, 0] = 0
        if empty_frac:
            # repeat some offsets to make empty bags
            rep = rng.random((F, B)) < empty_frac
            for k in range(F):
                for b in range(1, B):
                    if rep[k, b]:
                        off[k, b] = off[k, b - 1]
    else:
        off = np.broadcast_to((np.arange(B) * L).astype(np.int32), (F, B)).copy()
    dense = torch.empty((B, D), device=DEV).normal_(0, 1, generator=g)
    return weights, idx, off, dense


SHAPES = [
    # (B, F, N, D, L, ragged)  -- several tiles and a ragged tail in each dimension
    (1, 1, 10, 64, 8, False),
    (3, 1, 7, 4, 1, False),
    (33, 5, 100, 64, 16, False),
    (130, 7, 500, 128, 20, False),
    (257, 3, 64, 16, 3, False),
    (65, 32, 1000, 64, 16, True),
    (19, 4, 50, 1, 5, False),          # D = 1, scalar path
    (23, 3, 60, 6, 7, False),          # D % 4 != 0
    (17, 2, 40, 33, 9, True),          # odd D, ragged bags
    (9, 3, 30, 36, 40, False),         # 9 float4 per row, L > 32
    (12, 2, 80, 256, 10, False),       # 64 float4 per row: two chunks per lane
    (7, 2, 40, 260, 6, False),         # 65 float4 per row: two column windows
    (5, 3, 20, 100, 4, True),          # 25 float4 per row, ragged
    (41, 9, 200, 64, 32, True),
    (300, 26, 1000, 128, 20, False),
    (64, 2, 100, 16, 4, True),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}_F{}_N{}_D{}_L{}{}".format(
    *s[:5], "_ragged" if s[5] else ""))
@pytest.mark.parametrize("concat", [False, True])
def test_shapes(ops, shape, concat):
    B, F, N, D, L, ragged = shape
    weights, idx, off, dense = _random_case(hash(shape) % 1000, B, F, N, D, L, ragged, 0.2)
    _check_against_oracle(ops, weights, idx, off, dense, B, L, concat, str(shape))


def test_empty_bags_and_zero_length(ops):
    B, F, N, D = 40, 3, 30, 64
    weights, idx, off, dense = _random_case(1, B, F, N, D, 4, ragged=True, empty_frac=0.5)
    _check_against_oracle(ops, weights, idx, off, dense, B, 4, False, "many empty bags")
    # L = 0: every bag empty, no indices at all
    empty = np.zeros((F, 0), dtype=np.int32)
    zoff = np.zeros((F, B), dtype=np.int32)
    idx_d = torch.zeros(0, dtype=torch.int32, device=DEV)
    pooled = ops.embbag_sum_multi(weights, idx_d, _dev_i32(zoff), 0)
    fp, fi = ops.sparse_interact(weights, idx_d, _dev_i32(zoff), dense, 0)
    torch.cuda.synchronize()
    ref_p, ref_i, bound = oracle_stage(host_tables(weights), empty, zoff, dense.cpu().numpy(), B,
                                       0, False)
    assert_bits_equal(pooled, ref_p, "L=0 pooled")
    assert_bits_equal(fp, ref_p, "L=0 fused pooled")
    check_inter(fi, ref_i, bound, D, False, "L=0 fused")


def test_tables_with_different_row_counts(ops):
    rng = np.random.default_rng(2)
    B, D, L = 50, 64, 6
    rows = [10, 1000, 3, 77]
    weights = [torch.randn(n, D, device=DEV) * 0.1 for n in rows]
    idx = np.stack([rng.integers(0, n, B * L) for n in rows]).astype(np.int32)
    off = np.broadcast_to((np.arange(B) * L).astype(np.int32), (4, B)).copy()
    dense = torch.randn(B, D, device=DEV)
    _check_against_oracle(ops, weights, idx, off, dense, B, L, True, "ragged row counts")


def test_max_tables_and_large_shared_memory(ops):
    """F = 256 tables: the interaction block needs > 48 KB of shared memory."""
    B, F, N, D, L = 9, 256, 64, 128, 2
    weights, idx, off, dense = _random_case(4, B, F, N, D, L)
    _check_against_oracle(ops, weights, idx, off, dense, B, L, True, "F=256 D=128")


def test_shared_memory_limit_is_reported(ops):
    B, F, D = 2, 256, 256  # 260 rows x 260 floats x 4 B = 270 KB > 227 KB
    weights = [torch.zeros(4, D, device=DEV) for _ in range(F)]
    dense = torch.zeros(B, D, device=DEV)
    emb = torch.zeros(B, F, D, device=DEV)
    with pytest.raises(ops.DlrmError, match="DLRM_ERR_SHAPE"):
        ops.interact_lower_tri(dense, emb)
    off = torch.zeros(F, B, dtype=torch.int32, device=DEV)
    idx = torch.zeros(F * B, dtype=torch.int32, device=DEV)
    with pytest.raises(ops.DlrmError, match="DLRM_ERR_SHAPE"):
        ops.sparse_interact(weights, idx, off, dense, 1)
    # the gather alone has no shared-memory limit
    pooled = ops.embbag_sum_multi(weights, idx, off, 1)
    torch.cuda.synchronize()
    assert torch.count_nonzero(pooled) == 0


def test_misaligned_pointers_take_the_scalar_path(ops):
    B, F, N, D, L = 21, 3, 50, 64, 5
    weights, idx, off, dense = _random_case(6, B, F, N, D, L)
    # views that start 4 bytes into their storage: not 16-byte aligned
    wmis = []
    for w in weights:
        buf = torch.empty(w.numel() + 1, device=DEV)
        buf[1:].copy_(w.reshape(-1))
        wmis.append(buf[1:].view(N, D))
    dbuf = torch.empty(dense.numel() + 1, device=DEV)
    dbuf[1:].copy_(dense.reshape(-1))
    dmis = dbuf[1:].view(B, D)
    assert wmis[0].data_ptr() % 16 == 4
    _check_against_oracle(ops, wmis, idx, off, dmis, B, L, True, "misaligned")


def test_checked_entry_points_flag_and_skip(ops):
    rng = np.random.default_rng(8)
    B, F, N, D, L = 30, 3, 20, 64, 4
    weights, idx, off, dense = _random_case(8, B, F, N, D, L)
    bad_idx = idx.copy()
    planted = [(0, 5, N), (1, 17, -1), (2, 100, N + 1000)]
    for k, t, v in planted:
        bad_idx[k, t] = v
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx_d, off_d = _dev_i32(bad_idx), _dev_i32(off)
    pooled = ops.embbag_sum_multi(weights, idx_d, off_d, L, status=status, checked=True)
    torch.cuda.synchronize()
    assert int(status.item()) == ops.FLAG_INDEX_OOB
    assert ops.status_from_flags(int(status.item())) == -5
    # expected: the oracle on the same bags with the planted entries removed
    new_idx, new_off = [], []
    for k in range(F):
        keep = np.ones(B * L, bool)
        for kk, t, _ in planted:
            if kk == k:
                keep[t] = False
        starts = off[k]
        cum = np.concatenate([[0], np.cumsum(keep)])
        new_off.append(cum[starts])
        new_idx.append(bad_idx[k][keep])
    seg = max(len(x) for x in new_idx)
    Lp = -(-seg // (B + 1))
    idx2 = np.zeros((F, (B + 1) * Lp), np.int32)
    off2 = np.zeros((F, B + 1), np.int32)
    for k in range(F):
        idx2[k, :len(new_idx[k])] = new_idx[k]
        off2[k, :B] = new_off[k]
        off2[k, B] = len(new_idx[k])
    ref = oracle.embbag_sum_multi(host_tables(weights), idx2, off2, B + 1, Lp)[:B]
    assert_bits_equal(pooled, ref, "checked gather with planted bad indices")
    fp, fi = ops.sparse_interact(weights, idx_d, off_d, dense, L, status=status, checked=True)
    torch.cuda.synchronize()
    assert int(status.item()) == ops.FLAG_INDEX_OOB
    assert_bits_equal(fp, ref, "checked fused with planted bad indices")
    # clean input: status cleared to 0 by the call
    ops.embbag_sum_multi(weights, _dev_i32(idx), off_d, L, status=status, checked=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # bad offsets: the bag pools as empty and the flag is raised
    off_bad = off.copy()
    off_bad[1, 7] = off_bad[1, 8] + 1  # bag 7 of table 1: start > end
    pooled = ops.embbag_sum_multi(weights, _dev_i32(idx), _dev_i32(off_bad), L, status=status,
                                  checked=True)
    torch.cuda.synchronize()
    assert int(status.item()) & ops.FLAG_OFFSETS
    assert torch.count_nonzero(pooled[7, 1]) == 0
    # the unchecked entry point pools the same bag as empty too (no out-of-range read)
    pooled_u = ops.embbag_sum_multi(weights, _dev_i32(idx), _dev_i32(off_bad), L)
    torch.cuda.synchronize()
    assert torch.equal(pooled_u.view(torch.int32), pooled.view(torch.int32))


# ------------------------------------------------------------------ integer work

def test_pair_decoder_exhaustive(ops):
    """Every flat index p < 2^24 through pair_from_flat_small, the decoder the
    interaction and fused kernels run on their pair-tile index (tile indices
    stay below 2145 at 256 tables), against the oracle's nested-loop
    enumeration of the triangle of 5794 features, bit-exact."""
    n = 1 << 24
    pi, pj = oracle.pair_list(5794)
    assert len(pi) >= n
    gi, gj = ops.pair_decode(0, n)
    torch.cuda.synchronize()
    assert np.array_equal(gi.cpu().numpy(), pi[:n])
    assert np.array_equal(gj.cpu().numpy(), pj[:n])
    # across the switch to the 64-bit decoder at 2^24
    gi, gj = ops.pair_decode(n - 4096, 8192)
    torch.cuda.synchronize()
    assert np.array_equal(gi.cpu().numpy(), pi[n - 4096:n + 4096])
    assert np.array_equal(gj.cpu().numpy(), pj[n - 4096:n + 4096])


def test_pair_decoder_near_int32_limit(ops):
    """The last 2^20 flat indices below 2^31, against exact integer square roots."""
    import math

    p0 = (1 << 31) - (1 << 20)
    gi, gj = ops.pair_decode(p0, 1 << 20)
    torch.cuda.synchronize()
    gi, gj = gi.cpu().numpy().astype(np.int64), gj.cpu().numpy().astype(np.int64)
    for e in list(range(0, 1 << 20, 997)) + [(1 << 20) - 1]:
        p = p0 + e
        i = (1 + math.isqrt(1 + 8 * p)) // 2
        assert (gi[e], gj[e]) == (i, p - i * (i - 1) // 2), p
    # (i, j) is a bijection onto the lower triangle: consistent with p everywhere
    p = p0 + np.arange(1 << 20, dtype=np.int64)
    assert np.array_equal(gi * (gi - 1) // 2 + gj, p)
    assert np.all((gj >= 0) & (gj < gi))


# ------------------------------------------------------------------ API behaviour

def test_host_stage_matches_device_path(ops):
    w = syn.C2_CONCAT.scaled(B=300)
    weights, idx, off, dense = _inputs(w)
    stage = ops.HostStage(weights, w.B, w.L, concat_dense=True, want_pooled=True)
    ih = torch.from_numpy(idx.reshape(-1)).pin_memory()
    oh = torch.from_numpy(off).pin_memory()
    dh = dense.cpu().pin_memory()
    inter_h = torch.empty((w.B, w.D + w.P)).pin_memory()
    pooled_h = torch.empty((w.B, w.F, w.D)).pin_memory()
    stage(ih, oh, dh, inter_h, pooled_h)
    torch.cuda.synchronize()
    fp, fi = ops.sparse_interact(weights, _dev_i32(idx), _dev_i32(off), dense, w.L,
                                 concat_dense=True)
    torch.cuda.synchronize()
    assert torch.equal(inter_h.view(torch.int32), fi.cpu().view(torch.int32))
    assert torch.equal(pooled_h.view(torch.int32), fp.cpu().view(torch.int32))
    assert stage.h2d_bytes() == 4 * (w.F * w.B * w.L + w.F * w.B + w.B * w.D)
    # a packed batch (one host block, one copy) gives the same bits
    pi, po, pd = stage.pack(ih, oh, dh)
    inter2 = torch.empty_like(inter_h).pin_memory()
    pooled2 = torch.empty_like(pooled_h).pin_memory()
    stage(pi, po, pd, inter2, pooled2)
    torch.cuda.synchronize()
    assert torch.equal(inter2.view(torch.int32), inter_h.view(torch.int32))
    assert torch.equal(pooled2.view(torch.int32), pooled_h.view(torch.int32))


def test_host_stage_matches_the_oracle(ops):
    """The host-buffer entry point against the oracle directly (not only
    against the device entry point)."""
    w = syn.C2_CONCAT.scaled(B=300)
    weights, idx, off, dense = _inputs(w)
    stage = ops.HostStage(weights, w.B, w.L, concat_dense=True, want_pooled=True)
    inter_h = torch.empty((w.B, w.D + w.P)).pin_memory()
    pooled_h = torch.empty((w.B, w.F, w.D)).pin_memory()
    stage(torch.from_numpy(idx.reshape(-1)).pin_memory(), torch.from_numpy(off).pin_memory(),
          dense.cpu().pin_memory(), inter_h, pooled_h)
    torch.cuda.synchronize()
    ref_p, ref_i, bound = oracle_stage(host_tables(weights), idx, off, dense.cpu().numpy(), w.B,
                                       w.L, True)
    assert_bits_equal(pooled_h, ref_p, "host stage pooled")
    check_inter(inter_h, ref_i, bound, w.D, True, "host stage")


def test_one_hot_tables_are_exact(ops):
    """Tables W_k[r, :] = e_(r mod D): every pooled value is an entry count and
    every dot an integer, so both sides agree bit for bit, dots included."""
    B, F, N, D, L = 67, 6, 200, 64, 9
    w = syn.Workload("one_hot", B=B, F=F, N=N, D=D, L=L)
    eye = torch.zeros((N, D), device=DEV)
    eye[torch.arange(N), torch.arange(N) % D] = 1.0
    weights = [eye.clone() for _ in range(F)]
    idx, off = syn.make_indices(w), syn.make_offsets(w)
    dense = torch.randint(-3, 4, (B, D), device=DEV).float()
    pooled, inter_sep, fp, fi, fi2 = _run_all_paths(ops, weights, idx, off, dense, B, L, False)
    ref_p, ref_i, _ = oracle_stage(host_tables(weights), idx, off, dense.cpu().numpy(), B, L,
                                   False)
    counts = np.zeros((B, F, D))
    for k in range(F):
        for b in range(B):
            for r in idx[k, b * L:(b + 1) * L]:
                counts[b, k, r % D] += 1
    assert np.array_equal(ref_p, counts)
    for got, what in ((pooled, "gather"), (fp, "fused pooled")):
        assert_bits_equal(got, ref_p, "one-hot " + what)
    for got, what in ((inter_sep, "interact"), (fi, "fused"), (fi2, "fused, no pooled")):
        assert_bits_equal(got, ref_i.astype(np.float32), "one-hot dots " + what)


def test_bag_of_copies_is_exact(ops):
    """A bag of L copies of one row r pools to exactly L * W[r] when the rows
    hold k/256 values (|k| < 256): every partial sum is representable."""
    B, F, N, D, L = 45, 5, 300, 64, 12
    rng = np.random.default_rng(23)
    weights = [torch.from_numpy((rng.integers(-255, 256, (N, D)) / 256.0).astype(np.float32))
               .to(DEV) for _ in range(F)]
    rows = rng.integers(0, N, (F, B))
    idx = np.repeat(rows, L, axis=1).astype(np.int32)
    off = syn.make_offsets(syn.Workload("copies", B=B, F=F, N=N, D=D, L=L))
    dense = torch.zeros((B, D), device=DEV)
    pooled, _, fp, _, _ = _run_all_paths(ops, weights, idx, off, dense, B, L, False)
    want = np.stack([np.stack([L * weights[k][rows[k, b]].cpu().numpy().astype(np.float64)
                               for k in range(F)]) for b in range(B)])
    ref_p, _, _ = oracle_stage(host_tables(weights), idx, off, dense.cpu().numpy(), B, L, False)
    assert np.array_equal(ref_p, want)
    assert_bits_equal(pooled, want.astype(np.float32), "copies gather")
    assert_bits_equal(fp, want.astype(np.float32), "copies fused")


def test_repeat_runs_are_bit_identical_and_launch_once(ops):
    w = syn.C2_CONCAT.scaled(B=512)
    weights, idx, off, dense = _inputs(w)
    idx_d, off_d = _dev_i32(idx), _dev_i32(off)
    n0 = ops.launch_count()
    a = ops.sparse_interact(weights, idx_d, off_d, dense, w.L, concat_dense=True)
    assert ops.launch_count() == n0 + 1
    b = ops.sparse_interact(weights, idx_d, off_d, dense, w.L, concat_dense=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0].view(torch.int32), b[0].view(torch.int32))
    assert torch.equal(a[1].view(torch.int32), b[1].view(torch.int32))


def test_cuda_graph_capture_and_replay(ops):
    w = syn.C2_CONCAT.scaled(B=256)
    weights, idx, off, dense = _inputs(w)
    idx_d, off_d = _dev_i32(idx), _dev_i32(off)
    pooled = torch.empty((w.B, w.F, w.D), device=DEV)
    inter = torch.empty((w.B, w.D + w.P), device=DEV)
    ref_p, ref_i = ops.sparse_interact(weights, idx_d, off_d, dense, w.L, concat_dense=True)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        ops.sparse_interact(weights, idx_d, off_d, dense, w.L, concat_dense=True,
                            pooled_out=pooled, inter_out=inter)  # warm-up outside capture
        s.synchronize()
        pooled.zero_()
        inter.zero_()
        with torch.cuda.graph(g, stream=s):
            ops.sparse_interact(weights, idx_d, off_d, dense, w.L, concat_dense=True,
                                pooled_out=pooled, inter_out=inter)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(pooled.view(torch.int32), ref_p.view(torch.int32))
    assert torch.equal(inter.view(torch.int32), ref_i.view(torch.int32))
    del g


def test_nondefault_stream_ordering(ops):
    w = syn.TINY.scaled(B=200)
    weights, idx, off, dense = _inputs(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        idx_d, off_d = _dev_i32(idx), _dev_i32(off)
        fp, fi = ops.sparse_interact(weights, idx_d, off_d, dense, w.L)
    s.synchronize()
    ref_p, ref_i, bound = oracle_stage(host_tables(weights), idx, off, dense.cpu().numpy(), w.B,
                                       w.L, False)
    assert_bits_equal(fp, ref_p, "side stream pooled")
    check_inter(fi, ref_i, bound, w.D, False, "side stream")


def test_host_pipeline_overlapped_batches(ops):
    w = syn.C2_CONCAT.scaled(B=257)
    weights = syn.make_weights(w, DEV)
    dense = syn.make_dense(w, DEV)
    off = syn.make_offsets(w)
    pipe = ops.HostPipeline(weights, w.B, w.L, concat_dense=True, depth=2)
    batches = [syn.make_indices(w, replica=r) for r in range(5)]
    outs = [torch.empty((w.B, w.D + w.P)).pin_memory() for _ in range(5)]
    events = [pipe.submit(torch.from_numpy(b.reshape(-1)).pin_memory(),
                          torch.from_numpy(off).pin_memory(), dense.cpu().pin_memory(), o)
              for b, o in zip(batches, outs)]
    for ev, b, o in zip(events, batches, outs):
        pipe.wait(ev)
        _, ref = ops.sparse_interact(weights, _dev_i32(b), _dev_i32(off), dense, w.L,
                                     concat_dense=True)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int32), ref.cpu().view(torch.int32))
    pipe.drain()


def test_path_choice(ops):
    """Every call runs the per-block register-load path; the retired path
    numbers are rejected."""
    prev = ops.set_gather_path("auto")
    try:
        for D in (6, 16, 64, 128, 512):
            weights, idx, off, dense = _random_case(D, 5, 3, 40, D, 4)
            ops.embbag_sum_multi(weights, _dev_i32(idx), _dev_i32(off), 4)
            assert ops.last_gather_path() == "ldg"
            ops.sparse_interact(weights, _dev_i32(idx), _dev_i32(off), dense, 4)
            assert ops.last_gather_path() == "ldg"
        for retired in (2, 3, 4):
            assert ops._lib.dlrm_set_gather_path(retired) == -9
        torch.cuda.synchronize()
    finally:
        ops.set_gather_path(prev)


def test_prepared_call_matches_plain_call(ops):
    w = syn.C2_CONCAT.scaled(B=333)
    weights, idx, off, dense = _inputs(w)
    idx_d, off_d = _dev_i32(idx), _dev_i32(off)
    call = ops.SparseInteractCall(weights, idx_d, off_d, dense, w.L, concat_dense=True)
    p1, i1 = call()
    p2, i2 = ops.sparse_interact(weights, idx_d, off_d, dense, w.L, concat_dense=True)
    torch.cuda.synchronize()
    assert torch.equal(p1.view(torch.int32), p2.view(torch.int32))
    assert torch.equal(i1.view(torch.int32), i2.view(torch.int32))


@pytest.mark.parametrize("row_bytes", [16, 128, 256, 512])
def test_probe_row_gather_runs(ops, row_bytes):
    """The random-row read probe: one launch, no error, and on a table of
    zeros the folded value is zero, so the sink keeps its content."""
    table = torch.zeros(1 << 20, dtype=torch.float32, device=DEV)  # 4 MB
    sink = torch.full((1,), 12345, dtype=torch.int32, device=DEV)
    n0 = ops.launch_count()
    ops.probe_row_gather(table, row_bytes, 100_000, sink, seed=7)
    torch.cuda.synchronize()
    assert ops.launch_count() == n0 + 1
    assert int(sink.item()) == 12345
