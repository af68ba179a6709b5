"""Helpers of the GPU parity tests: run the oracle on the same seeded inputs and
compare. Pooled sums and every integer result must match bit for bit; a dot
must satisfy |gpu - oracle| <= 1e-5 * S_ij (S_ij = sum_d |v_i[d] v_j[d]|),
the relative form of the 1e-5 bound, taken against the magnitudes summed so
that dots that cancel to near zero are compared on the scale of their terms.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

DOT_RTOL = 1e-5
DOT_ATOL = 1e-30


def assert_bits_equal(gpu: torch.Tensor, ref: np.ndarray, what: str):
    g = gpu.detach().cpu().contiguous().numpy()
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    gb = g.view(np.uint32)
    rb = np.ascontiguousarray(ref, dtype=np.float32).view(np.uint32)
    bad = np.flatnonzero(gb.ravel() != rb.ravel())
    assert bad.size == 0, (
        f"{what}: {bad.size} of {gb.size} values differ in their bits; first at flat index "
        f"{bad[0]}: gpu {g.ravel()[bad[0]]!r} oracle {ref.ravel()[bad[0]]!r}")


def assert_dots_close(gpu: torch.Tensor, ref: np.ndarray, bound: np.ndarray, what: str):
    g = gpu.detach().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref.astype(np.float64))
    tol = DOT_RTOL * bound + DOT_ATOL
    bad = np.flatnonzero(~(err <= tol))
    assert bad.size == 0, (
        f"{what}: {bad.size} of {err.size} dots off; worst ratio "
        f"{np.nanmax(err / tol):.3g}, first at {bad[0]}: gpu {g.ravel()[bad[0]]!r} "
        f"oracle {ref.ravel()[bad[0]]!r} bound {bound.ravel()[bad[0]]!r}")


def check_inter(gpu_inter: torch.Tensor, ref_inter: np.ndarray, bound: np.ndarray, D: int,
                concat: bool, what: str):
    if concat:
        assert_bits_equal(gpu_inter[:, :D], ref_inter[:, :D], what + " dense part")
        assert_dots_close(gpu_inter[:, D:], ref_inter[:, D:], bound, what + " dots")
    else:
        assert_dots_close(gpu_inter, ref_inter, bound, what)


def host_tables(weights):
    return [w.detach().cpu().numpy() for w in weights]


def oracle_stage(weights_np, idx_np, off_np, dense_np, B, L, concat):
    pooled = oracle.embbag_sum_multi(weights_np, idx_np, off_np, B, L)
    inter, _, bound = oracle.interact_lower_tri(dense_np, pooled, concat_dense=concat,
                                                with_f64=True)
    return pooled, inter, bound


def sampled_oracle(weights, idx_np, off_np, dense: torch.Tensor, B: int, L: int,
                   samples: np.ndarray, concat: bool):
    """Oracle on a subset of samples of a large launch.

    Only the table rows that the sampled bags reference are copied to the host;
    their indices are renumbered into those compact tables and the bags are
    re-based onto a batch of just the sampled samples.
    """
    F = len(weights)
    BL = B * L
    sub_B = len(samples)
    starts = off_np[:, samples].astype(np.int64)
    nxt = np.where(samples + 1 < B, off_np[:, np.minimum(samples + 1, B - 1)], BL)
    ends = nxt.astype(np.int64)
    lens = ends - starts
    sub_idx_rows = []
    sub_offs = np.zeros((F, sub_B), dtype=np.int64)
    tables = []
    maxlen = int(lens.sum(axis=1).max()) if lens.size else 0
    for k in range(F):
        pieces = [idx_np[k, s:e] for s, e in zip(starts[k], ends[k])]
        flat = np.concatenate(pieces) if pieces else np.zeros(0, np.int32)
        uniq, inv = np.unique(flat, return_inverse=True)
        if uniq.size == 0:  # every sampled bag of this table is empty
            uniq = np.zeros(1, dtype=flat.dtype)
        rows_t = torch.from_numpy(uniq.astype(np.int64)).to(weights[k].device)
        tables.append(weights[k].index_select(0, rows_t).cpu().numpy())
        sub_offs[k] = np.concatenate([[0], np.cumsum(lens[k])[:-1]])
        sub_idx_rows.append(inv.astype(np.int32))
    # the oracle takes one B*L segment per table: pad every segment to the same
    # length with entries no bag covers (the last bag ends at the segment end,
    # so the padding goes into an extra trailing bag that is dropped)
    seg = max(maxlen, 1)
    idx_sub = np.zeros((F, seg), dtype=np.int32)
    for k in range(F):
        idx_sub[k, :len(sub_idx_rows[k])] = sub_idx_rows[k]
    # add one trailing sample per table to absorb the padding
    off_sub = np.zeros((F, sub_B + 1), dtype=np.int32)
    off_sub[:, :sub_B] = sub_offs
    off_sub[:, sub_B] = [len(r) for r in sub_idx_rows]
    dense_np = dense[torch.from_numpy(samples.astype(np.int64)).to(dense.device)].cpu().numpy()
    dense_ext = np.concatenate([dense_np, np.zeros((1, dense_np.shape[1]), np.float32)])
    # segment length must be (sub_B + 1) * L' for some L': choose L' = seg / (sub_B + 1) when it
    # divides, else widen the segment
    nb = sub_B + 1
    Lp = -(-seg // nb)
    idx_full = np.zeros((F, nb * Lp), dtype=np.int32)
    idx_full[:, :seg] = idx_sub
    pooled, inter, bound = oracle_stage(tables, idx_full, off_sub, dense_ext, nb, Lp, concat)
    return pooled[:sub_B], inter[:sub_B], bound[:sub_B]
