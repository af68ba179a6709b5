"""GPU parity of the general pooling entry points against the oracle.

Ragged bags, include_last_offset, per-sample weights, sum / mean / max and
bf16 tables, through ``embbag_pool_multi`` and the fused
``dlrm_sparse_interact_pool``. Pooled values are compared bit for bit; dots
within 1e-5 * S_ij.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from dlrm_embedding_bag_b200 import synthetic as syn
from gpu_cases import assert_bits_equal, assert_dots_close

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def ops():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from dlrm_embedding_bag_b200 import ops as _ops

    return _ops


def _host_bits(t: torch.Tensor) -> np.ndarray:
    """Host copy of a table: f32 values, or bf16 bit patterns as uint16."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def _case(seed, B, F, N, D, T, dtype, ilo, empty_frac=0.2):
    rng = np.random.default_rng(seed)
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    weights = [torch.empty((N, D), device=DEV).normal_(0, 0.3, generator=g).to(dtype)
               for _ in range(F)]
    idx = rng.integers(0, N, (F, T)).astype(np.int32)
    nb = B + (1 if ilo else 0)
    off = np.sort(rng.integers(0, T + 1, (F, nb)), axis=1).astype(np.int32)
    off[:, 0] = 0
    if ilo:
        off[:, -1] = rng.integers(T // 2, T + 1, F)  # entries past the last bag are unused
        off = np.minimum(off, off[:, -1:])
    rep = rng.random((F, nb)) < empty_frac
    for k in range(F):
        for b in range(1, nb - (1 if ilo else 0)):
            if rep[k, b]:
                off[k, b] = off[k, b - 1]
    psw = rng.normal(1.0, 0.5, (F, T)).astype(np.float32)
    dense = torch.empty((B, D), device=DEV).normal_(0, 1, generator=g)
    return weights, idx, off, psw, dense


SHAPES = [  # (B, F, N, D, T)
    (37, 3, 50, 64, 300),
    (16, 8, 200, 128, 900),
    (9, 5, 40, 16, 60),
    (21, 2, 30, 24, 90),      # bf16: D % 8 == 0; f32: D % 4 == 0
    (13, 4, 30, 20, 70),      # bf16 scalar path (D % 8 != 0), f32 vector path
    (11, 3, 25, 7, 40),       # both scalar
    (6, 2, 20, 264, 30),      # two column windows
    (70, 26, 500, 64, 2000),
    (10, 100, 30, 16, 120),   # fused: 3 samples x 100 bags per block, > 256 bags to order
]
VARIANTS = [("sum", False), ("sum", True), ("mean", False), ("max", False)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}_F{}_N{}_D{}_T{}".format(*s))
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
@pytest.mark.parametrize("ilo", [False, True], ids=["", "last_offset"])
def test_general_pooling(ops, shape, dtype, ilo):
    B, F, N, D, T = shape
    weights, idx, off, psw, dense = _case(sum(shape) + (7 if ilo else 0), B, F, N, D, T, dtype,
                                          ilo)
    ws = [_host_bits(w) for w in weights]
    idx_d = torch.from_numpy(idx).to(DEV)
    off_d = torch.from_numpy(off).to(DEV)
    psw_d = torch.from_numpy(psw).to(DEV)
    for mode, weighted in VARIANTS:
        p = psw if weighted else None
        ref = oracle.embbag_pool_multi(ws, idx, off, B, mode=mode, per_sample_weights=p,
                                       include_last_offset=ilo)
        what = f"{shape} {dtype} ilo={ilo} {mode}{' weighted' if weighted else ''}"
        out = ops.embbag_pool_multi(weights, idx_d, off_d, mode=mode,
                                    per_sample_weights=psw_d if weighted else None,
                                    include_last_offset=ilo)
        fp, fi = ops.sparse_interact_pool(weights, idx_d, off_d, dense, mode=mode,
                                          per_sample_weights=psw_d if weighted else None,
                                          include_last_offset=ilo, concat_dense=True)
        torch.cuda.synchronize()
        assert_bits_equal(out, ref, what + " embbag_pool_multi")
        assert_bits_equal(fp, ref, what + " fused pooled")
        ref_i, _, bound = oracle.interact_lower_tri(dense.cpu().numpy(), ref, concat_dense=True,
                                                    with_f64=True)
        assert_bits_equal(fi[:, :D], ref_i[:, :D], what + " fused dense part")
        assert_dots_close(fi[:, D:], ref_i[:, D:], bound, what + " fused dots")


def test_plain_entry_points_equal_general_sum(ops):
    w = syn.C2_CONCAT.scaled(B=200)
    weights = syn.make_weights(w, DEV)
    idx = torch.from_numpy(syn.make_indices(w)).to(DEV)
    off = torch.from_numpy(syn.make_offsets(w)).to(DEV)
    dense = syn.make_dense(w, DEV)
    a = ops.embbag_sum_multi(weights, idx, off, w.L)
    b = ops.embbag_pool_multi(weights, idx, off)
    pa, ia = ops.sparse_interact(weights, idx, off, dense, w.L, concat_dense=True)
    pb, ib = ops.sparse_interact_pool(weights, idx, off, dense, concat_dense=True)
    torch.cuda.synchronize()
    for x, y in ((a, b), (pa, pb), (ia, ib)):
        assert torch.equal(x.view(torch.int32), y.view(torch.int32))


@pytest.mark.parametrize("mode", ["sum", "mean", "max"])
def test_checked_general_pooling_skips_bad_indices(ops, mode):
    B, F, N, D, T = 20, 3, 15, 64, 100
    weights, idx, off, _, dense = _case(31, B, F, N, D, T, torch.float32, False, 0.0)
    bad = idx.copy()
    planted = [(0, 3, N), (1, 50, -7), (2, 99, 1 << 30)]
    for k, t, v in planted:
        bad[k, t] = v
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = ops.embbag_pool_multi(weights, torch.from_numpy(bad).to(DEV),
                                torch.from_numpy(off).to(DEV), mode=mode, checked=True,
                                status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == ops.FLAG_INDEX_OOB
    # expected: the same bags with the planted entries removed (include_last_offset form)
    new_idx = np.zeros_like(bad)
    new_off = np.zeros((F, B + 1), np.int32)
    for k in range(F):
        keep = np.ones(T, bool)
        keep[[t for kk, t, _ in planted if kk == k]] = False
        cum = np.concatenate([[0], np.cumsum(keep)])
        new_off[k, :B] = cum[off[k]]
        new_off[k, B] = cum[T]
        kept = bad[k][keep]
        new_idx[k, :kept.size] = kept
    ref = oracle.embbag_pool_multi([w.cpu().numpy() for w in weights], new_idx, new_off, B,
                                   mode=mode, include_last_offset=True)
    assert_bits_equal(out, ref, f"checked {mode}")


@pytest.mark.parametrize("mode", ["sum", "mean"])
def test_general_bad_offsets_flagged(ops, mode):
    """Bags whose bounds break start <= end, start >= 0 or end <= T pool as
    empty and raise FLAG_OFFSETS, through the gather and the fused entry
    points; every other bag (and every dot) is exact."""
    B, F, N, D, T = 40, 5, 60, 64, 300
    weights, idx, off, _, dense = _case(41, B, F, N, D, T, torch.float32, False, 0.0)
    off_bad = off.copy()
    off_bad[1, 7] = off_bad[1, 8] + 1   # bag 7 of table 1: start > end
    off_bad[3, 0] = -1                  # bag 0 of table 3: start < 0
    off_bad[4, B - 1] = T + 1           # last bag of table 4: start > T
    # expected: each valid bag's entries, laid out again back to back
    idx2 = np.zeros((F, T + 1), np.int32)
    off2 = np.zeros((F, B + 1), np.int32)
    bad_bags = []
    for k in range(F):
        pos = 0
        for b in range(B):
            st = int(off_bad[k, b])
            en = int(off_bad[k, b + 1]) if b + 1 < B else T
            off2[k, b] = pos
            if st < 0 or st > en or en > T:
                bad_bags.append((b, k))
                continue
            idx2[k, pos:pos + en - st] = idx[k, st:en]
            pos += en - st
        off2[k, B] = pos
    assert len(bad_bags) >= 3
    ws = [_host_bits(w) for w in weights]
    ref = oracle.embbag_pool_multi(ws, idx2, off2, B, mode=mode, include_last_offset=True)
    idx_d = torch.from_numpy(idx).to(DEV)
    off_d = torch.from_numpy(off_bad).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = ops.embbag_pool_multi(weights, idx_d, off_d, mode=mode, checked=True, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == ops.FLAG_OFFSETS
    assert_bits_equal(out, ref, f"gather, bad offsets, {mode}")
    status.zero_()
    fp, fi = ops.sparse_interact_pool(weights, idx_d, off_d, dense, mode=mode, checked=True,
                                      status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == ops.FLAG_OFFSETS
    assert_bits_equal(fp, ref, f"fused, bad offsets, {mode}")
    for b, k in bad_bags:
        assert torch.count_nonzero(fp[b, k]) == 0
    ref_i, _, bound = oracle.interact_lower_tri(dense.cpu().numpy(), ref, with_f64=True)
    assert_dots_close(fi, ref_i, bound, f"fused dots, bad offsets, {mode}")


def test_bf16_full_size_sampled(ops):
    """The c3 workload with bf16 tables (half the gathered bytes), sampled check."""
    w = syn.C3_ZIPF
    torch.cuda.empty_cache()
    weights = [t.to(torch.bfloat16) for t in syn.make_weights(w, DEV)]
    torch.cuda.empty_cache()
    idx = syn.make_indices(w)
    off = syn.make_offsets(w)
    dense = syn.make_dense(w, DEV)
    pooled, inter = ops.sparse_interact_pool(weights, torch.from_numpy(idx).to(DEV),
                                             torch.from_numpy(off).to(DEV), dense)
    torch.cuda.synchronize()
    rng = np.random.default_rng(9)
    samples = np.unique(np.concatenate([[0, w.B - 1], rng.integers(0, w.B, 30)]))
    tables, sub_idx = [], []
    for k in range(w.F):
        rows = np.concatenate([idx[k, s * w.L:(s + 1) * w.L] for s in samples])
        uniq, inv = np.unique(rows, return_inverse=True)
        t = weights[k].index_select(0, torch.from_numpy(uniq.astype(np.int64)).to(DEV))
        tables.append(_host_bits(t))
        sub_idx.append(inv.astype(np.int32))
    sub_off = np.broadcast_to((np.arange(len(samples)) * w.L).astype(np.int32),
                              (w.F, len(samples))).copy()
    ref = oracle.embbag_pool_multi(tables, np.stack(sub_idx), sub_off, len(samples))
    sel = torch.from_numpy(samples).to(DEV)
    assert_bits_equal(pooled[sel], ref, "bf16 c3 pooled (sampled)")
    ref_i, _, bound = oracle.interact_lower_tri(dense[sel].cpu().numpy(), ref, with_f64=True)
    assert_dots_close(inter[sel], ref_i, bound, "bf16 c3 dots (sampled)")
    del weights, pooled, inter
    torch.cuda.empty_cache()


@pytest.mark.parametrize("weighted", [False, True], ids=["sum", "weighted"])
def test_ragged_full_size_sampled(ops, weighted):
    """The c3 workload with ragged bags (the benchmark's ragged input: sorted
    uniform cut points, mean length L) and optionally per-sample weights,
    through the fused general entry point; sampled check of pooled rows (bit
    for bit) and dots."""
    w = syn.C3_ZIPF
    torch.cuda.empty_cache()
    weights = syn.make_weights(w, DEV)
    idx = syn.make_indices(w)
    off = syn.make_ragged_offsets(w)
    psw = syn.make_sample_weights(w) if weighted else None
    dense = syn.make_dense(w, DEV)
    pooled, inter = ops.sparse_interact_pool(
        weights, torch.from_numpy(idx).to(DEV), torch.from_numpy(off).to(DEV), dense,
        per_sample_weights=torch.from_numpy(psw).to(DEV) if weighted else None)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    samples = np.unique(np.concatenate([[0, w.B - 1], rng.integers(0, w.B, 30)]))
    T = w.B * w.L
    tables, sub_idx, sub_w = [], [], []
    sub_off = np.zeros((w.F, len(samples) + 1), np.int32)
    for k in range(w.F):
        ends = np.append(off[k, 1:], T)
        spans = [(int(off[k, s]), int(ends[s])) for s in samples]
        rows = np.concatenate([idx[k, a:b] for a, b in spans])
        uniq, inv = np.unique(rows, return_inverse=True)
        if uniq.size == 0:  # every sampled bag of this table is empty
            uniq = np.zeros(1, np.int32)
        t = weights[k].index_select(0, torch.from_numpy(uniq.astype(np.int64)).to(DEV))
        tables.append(t.cpu().numpy())
        sub_idx.append(inv.astype(np.int32))
        if weighted:
            sub_w.append(np.concatenate([psw[k, a:b] for a, b in spans]))
        sub_off[k, 1:] = np.cumsum([b - a for a, b in spans])
    seg = max(1, max(x.size for x in sub_idx))
    idx_pad = np.zeros((w.F, seg), np.int32)
    w_pad = np.zeros((w.F, seg), np.float32)
    for k in range(w.F):
        idx_pad[k, :sub_idx[k].size] = sub_idx[k]
        if weighted:
            w_pad[k, :sub_w[k].size] = sub_w[k]
    ref = oracle.embbag_pool_multi(tables, idx_pad, sub_off, len(samples),
                                   per_sample_weights=w_pad if weighted else None,
                                   include_last_offset=True)
    sel = torch.from_numpy(samples).to(DEV)
    what = "ragged c3" + (" weighted" if weighted else "")
    assert_bits_equal(pooled[sel], ref, what + " pooled (sampled)")
    ref_i, _, bound = oracle.interact_lower_tri(dense[sel].cpu().numpy(), ref, with_f64=True)
    assert_dots_close(inter[sel], ref_i, bound, what + " dots (sampled)")
    del weights, pooled, inter
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_max_ties_keep_the_earlier_entry(ops, dtype):
    """Max pooling keeps the first entry and then takes x only when x > acc, so
    of two tied entries the earlier survives: -0.0 then +0.0 gives -0.0, +0.0
    then -0.0 gives +0.0, bit for bit, on every path and in the fused kernel."""
    B, F, D = 48, 3, 64
    tab = np.zeros((4, D), np.float32)
    tab[0] = -0.0
    tab[2] = -1.0
    tab[3, ::2] = -0.0
    pairs = np.array([[0, 1], [1, 0], [2, 0], [0, 2], [3, 1], [1, 3]], np.int32)
    rng = np.random.default_rng(5)
    idx = np.stack([pairs[rng.integers(0, len(pairs), B)].reshape(-1) for _ in range(F)])
    off = np.broadcast_to(np.arange(B, dtype=np.int32) * 2, (F, B)).copy()
    weights = [torch.from_numpy(tab).to(DEV).to(dtype) for _ in range(F)]
    ref = oracle.embbag_pool_multi([_host_bits(w) for w in weights], idx, off, B, mode="max")
    assert (ref.view(np.uint32) == 0x80000000).any() and (ref.view(np.uint32) == 0).any()
    idx_d = torch.from_numpy(idx).to(DEV)
    off_d = torch.from_numpy(off).to(DEV)
    out = ops.embbag_pool_multi(weights, idx_d, off_d, mode="max")
    dense = torch.zeros((B, D), device=DEV)
    fp, _ = ops.sparse_interact_pool(weights, idx_d, off_d, dense, mode="max")
    torch.cuda.synchronize()
    assert_bits_equal(out, ref, "max ties, embbag_pool_multi")
    assert_bits_equal(fp, ref, "max ties, fused pooled")


def test_ordering_dropped_when_its_shared_memory_does_not_fit(ops):
    """A shape whose features fill the block's shared memory to within the
    768 bytes the bag ordering would add: the general (ragged) entry point
    still runs, without the ordering, and matches the oracle."""
    dev = torch.cuda.current_device()
    limit = torch.cuda.get_device_properties(dev).shared_memory_per_block_optin

    def per_sample(F, D):
        f1p = 4 * ((F + 1 + 3) // 4)
        return f1p * (4 * ((D + 3) // 4) + 4) * 4

    shape = next(((F, D) for F in range(200, 257) for D in range(200, 600)
                  if limit - 768 < per_sample(F, D) <= limit), None)
    assert shape is not None, limit
    F, D = shape
    B, N, T = 3, 20, 12
    weights, idx, off, psw, dense = _case(5, B, F, N, D, T, torch.float32, False, 0.3)
    ws = [_host_bits(w) for w in weights]
    ref = oracle.embbag_pool_multi(ws, idx, off, B)
    fp, fi = ops.sparse_interact_pool(weights, torch.from_numpy(idx).to(DEV),
                                      torch.from_numpy(off).to(DEV), dense, concat_dense=True)
    torch.cuda.synchronize()
    what = f"F={F} D={D} shared memory {per_sample(F, D)} of {limit}"
    assert_bits_equal(fp, ref, what + " pooled")
    ref_i, _, bound = oracle.interact_lower_tri(dense.cpu().numpy(), ref, concat_dense=True,
                                                with_f64=True)
    assert_bits_equal(fi[:, :D], ref_i[:, :D], what + " dense part")
    assert_dots_close(fi[:, D:], ref_i[:, D:], bound, what + " dots")
