"""Python binding of the DLRMv1 MLP layers (the C ABI in ``include/dlrm_mlp.h``).

Argument marshalling only, as in :mod:`.ops`: pointers, row pitches and the
current stream go to ``dlrm_linear_f32a`` / ``dlrm_linear_bf16`` /
``dlrm_split_f32_bf16x3`` / ``dlrm_f32_to_bf16``; every layer runs in the
library's tcgen05 kernel. bf16 tensors are ``torch.bfloat16``
views whose row pitch is a multiple of 8 elements (16 bytes), as the layer's
TMA loads require; :func:`bf16_empty` makes such buffers.

Two arithmetics are offered (``mode``). ``"f32"`` (the default) is the pages' own: f32
activations times bf16 (or f32) weights with f32 results, through
``dlrm_linear_f32a``; each f32 activation travels between layers as three
bf16 planes that sum to it exactly (:func:`planes_empty`,
:func:`split_bf16x3`). ``"bf16"`` rounds activations to bf16 (one plane,
``dlrm_linear_bf16``), a third of the tensor work.

A DLRMv1 forward (:func:`dlrm_forward`) is: bottom MLP on the dense features
-> ``dense`` (B, D); the sparse stage (pooled embeddings and the interaction
z, :func:`.ops.sparse_interact`); the top MLP whose first layer reads
``[dense | z]`` through the split-A form, ending in a sigmoid CTR head.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import ops

ACTS = {"none": 0, "relu": 1, "sigmoid": 2}


def _round8(n: int) -> int:
    return (n + 7) // 8 * 8


def bf16_empty(rows: int, cols: int, device="cuda") -> torch.Tensor:
    """A ``(rows, cols)`` bf16 view whose row pitch is ``cols`` rounded up to 8."""
    return torch.empty((rows, _round8(cols)), dtype=torch.bfloat16, device=device)[:, :cols]


def _pitched(t: torch.Tensor, name: str, dtype: torch.dtype) -> Tuple[int, int]:
    """(pointer, row pitch in elements) of a 2-D CUDA tensor with unit column stride."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (got {t.device})")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError(f"{name} must be 2-D with unit column stride")
    return t.data_ptr(), (t.stride(0) if t.shape[0] > 1 else max(t.stride(0), t.shape[1]))


def to_bf16(x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Round an f32 ``(rows, cols)`` tensor to bf16 (nearest even) into a pitched buffer."""
    px, ldx = _pitched(x, "x", torch.float32)
    rows, cols = x.shape
    if out is None:
        out = bf16_empty(rows, cols, x.device)
    py, ldy = _pitched(out, "out", torch.bfloat16)
    ops._check(ops._lib.dlrm_f32_to_bf16(px, ldx, rows, cols, py, ldy, ops._stream()),
               "dlrm_f32_to_bf16")
    return out


def linear_bf16(a_lo: torch.Tensor, w: torch.Tensor, bias: Optional[torch.Tensor] = None,
                act: str = "none", *, a_hi: Optional[torch.Tensor] = None, f32: bool = True,
                bf16: bool = False, out_f32: Optional[torch.Tensor] = None,
                out_bf16: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None):
    """One layer ``act([a_lo | a_hi] w^T + bias)``; returns ``(y_f32, y_bf16)``.

    ``a_lo`` ``(M, K_lo)``, ``a_hi`` ``(M, K_hi)`` (optional) and ``w``
    ``(N, K_lo + K_hi)`` are bf16; ``bias`` is ``(N,)`` f32 or None. The f32
    and/or bf16 result is written to ``out_*`` or to new buffers (``f32`` /
    ``bf16`` select which are made); the one not requested is None.
    """
    if act not in ACTS:
        raise ValueError(f"act must be one of {sorted(ACTS)}")
    pa, lda = _pitched(a_lo, "a_lo", torch.bfloat16)
    M, k_lo = a_lo.shape
    if a_hi is not None:
        ph, ldh = _pitched(a_hi, "a_hi", torch.bfloat16)
        if a_hi.shape[0] != M:
            raise ValueError("a_hi must have as many rows as a_lo")
        k_hi = a_hi.shape[1]
    else:
        ph, ldh, k_hi = None, 0, 0
    pw, ldw = _pitched(w, "w", torch.bfloat16)
    N = w.shape[0]
    if w.shape[1] != k_lo + k_hi:
        raise ValueError(f"w must be (N, {k_lo + k_hi})")
    pb = None
    if bias is not None:
        pb = ops._dev(bias, "bias", torch.float32)
        if bias.numel() != N:
            raise ValueError(f"bias must have {N} elements")
    if out_f32 is None and f32:
        out_f32 = torch.empty((M, N), dtype=torch.float32, device=a_lo.device)
    if out_bf16 is None and bf16:
        out_bf16 = bf16_empty(M, N, a_lo.device)
    pf, ldf = _pitched(out_f32, "out_f32", torch.float32) if out_f32 is not None else (None, 0)
    pbf, ldbf = (_pitched(out_bf16, "out_bf16", torch.bfloat16) if out_bf16 is not None
                 else (None, 0))
    ps = ops._dev(status, "status", torch.int32) if status is not None else None
    ops._check(ops._lib.dlrm_linear_bf16(pa, lda, k_lo, ph, ldh, k_hi, pw, ldw, pb, M, N,
                                         ACTS[act], pf, ldf, pbf, ldbf, ps, ops._stream()),
               "dlrm_linear_bf16")
    return out_f32, out_bf16


def planes_empty(rows: int, cols: int, device="cuda") -> torch.Tensor:
    """A ``(3, rows, cols)`` bf16 view: three planes whose row pitch is ``cols``
    rounded up to 8 (16-byte rows, as the layers' TMA loads require)."""
    return torch.empty((3, rows, _round8(cols)), dtype=torch.bfloat16,
                       device=device)[:, :, :cols]


def _planes(t: torch.Tensor, name: str) -> Tuple[int, int, int]:
    """(pointer, row pitch, plane stride) in elements of a ``(3, rows, cols)`` bf16 tensor."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda" or t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
    if t.dim() != 3 or t.shape[0] != 3 or (t.shape[2] > 1 and t.stride(2) != 1):
        raise ValueError(f"{name} must be (3, rows, cols) with unit column stride")
    ld = t.stride(1) if t.shape[1] > 1 else max(t.stride(1), t.shape[2])
    return t.data_ptr(), ld, t.stride(0)


def split_bf16x3(x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The exact three-plane split of an f32 ``(rows, cols)`` tensor:
    ``x == p[0] + p[1] + p[2]`` with every plane a bf16 value."""
    px, ldx = _pitched(x, "x", torch.float32)
    rows, cols = x.shape
    if out is None:
        out = planes_empty(rows, cols, x.device)
    py, ldy, sp = _planes(out, "out")
    ops._check(ops._lib.dlrm_split_f32_bf16x3(px, ldx, rows, cols, py, ldy, sp, ops._stream()),
               "dlrm_split_f32_bf16x3")
    return out


def linear_f32a(a_lo: torch.Tensor, w: torch.Tensor, bias: Optional[torch.Tensor] = None,
                act: str = "none", *, a_hi: Optional[torch.Tensor] = None, f32: bool = True,
                planes: bool = False, out_f32: Optional[torch.Tensor] = None,
                out_planes: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None):
    """One layer ``act([a_lo | a_hi] w^T + bias)`` on f32 activations; returns
    ``(y_f32, y_planes)``.

    ``a_lo`` ``(3, M, K_lo)`` and ``a_hi`` ``(3, M, K_hi)`` (optional) are the
    activations' bf16 planes (:func:`split_bf16x3`); ``w`` is bf16 ``(N, K)``
    weights or the ``(3, N, K)`` planes of f32 weights; ``bias`` ``(N,)`` f32 or
    None. The f32 result and/or its planes (the next layer's input) are
    written to ``out_*`` or to new buffers (``f32`` / ``planes`` select which).
    """
    if act not in ACTS:
        raise ValueError(f"act must be one of {sorted(ACTS)}")
    pa, lda, spa = _planes(a_lo, "a_lo")
    M, k_lo = a_lo.shape[1], a_lo.shape[2]
    if a_hi is not None:
        ph, ldh, sph = _planes(a_hi, "a_hi")
        if a_hi.shape[1] != M:
            raise ValueError("a_hi must have as many rows as a_lo")
        k_hi = a_hi.shape[2]
    else:
        ph, ldh, sph, k_hi = None, 0, 0, 0
    if w.dim() == 3:
        pw, ldw, spw = _planes(w, "w")
        w_planes, N, kw = 3, w.shape[1], w.shape[2]
    else:
        pw, ldw = _pitched(w, "w", torch.bfloat16)
        spw, w_planes, N, kw = 0, 1, w.shape[0], w.shape[1]
    if kw != k_lo + k_hi:
        raise ValueError(f"w must have {k_lo + k_hi} columns")
    pb = None
    if bias is not None:
        pb = ops._dev(bias, "bias", torch.float32)
        if bias.numel() != N:
            raise ValueError(f"bias must have {N} elements")
    if out_f32 is None and f32:
        out_f32 = torch.empty((M, N), dtype=torch.float32, device=a_lo.device)
    if out_planes is None and planes:
        out_planes = planes_empty(M, N, a_lo.device)
    pf, ldf = _pitched(out_f32, "out_f32", torch.float32) if out_f32 is not None else (None, 0)
    pp, ldp, spp = _planes(out_planes, "out_planes") if out_planes is not None else (None, 0, 0)
    ps = ops._dev(status, "status", torch.int32) if status is not None else None
    ops._check(ops._lib.dlrm_linear_f32a(pa, lda, spa, k_lo, ph, ldh, sph, k_hi, pw, ldw, spw,
                                         w_planes, pb, M, N, ACTS[act], pf, ldf, pp, ldp, spp,
                                         ps, ops._stream()),
               "dlrm_linear_f32a")
    return out_f32, out_planes


class MLP:
    """A stack of layers ``(w, bias, act)``.

    ``w`` is a bf16 ``(N, K)`` tensor (pitched, see :func:`bf16_empty`), or in
    ``"f32"`` mode also the ``(3, N, K)`` planes of f32 weights; ``bias``
    ``(N,)`` f32, ``act`` one of ``"none" | "relu" | "sigmoid"``. In ``"bf16"``
    mode activations between layers are bf16; in ``"f32"`` mode they are f32,
    carried as three exact bf16 planes, and the input is given as planes.
    """

    def __init__(self, layers: Sequence[Tuple[torch.Tensor, torch.Tensor, str]],
                 mode: str = "f32"):
        if not layers:
            raise ValueError("an MLP needs at least one layer")
        if mode not in ("bf16", "f32"):
            raise ValueError("mode must be 'bf16' or 'f32'")
        self.layers: List[Tuple[torch.Tensor, torch.Tensor, str]] = list(layers)
        self.mode = mode

    @property
    def out_features(self) -> int:
        return self.layers[-1][0].shape[0]

    def forward(self, x: torch.Tensor, *, a_hi: Optional[torch.Tensor] = None,
                last_f32: bool = True, last_bf16: bool = False, keep: bool = False):
        """Run the layers on ``x`` (and ``a_hi`` for the first layer's split form):
        bf16 tensors in ``"bf16"`` mode, three-plane tensors in ``"f32"`` mode.

        Returns ``(y_f32, y_next)`` of the last layer -- ``y_next`` is its bf16
        output (``"bf16"``) or its planes (``"f32"``) when ``last_bf16`` is set
        -- plus the list of every layer's inputs when ``keep`` is set.
        """
        inputs = []
        h, hi = x, a_hi
        n = len(self.layers)
        layer = linear_bf16 if self.mode == "bf16" else linear_f32a
        for i, (w, b, act) in enumerate(self.layers):
            inputs.append((h, hi))
            last = i == n - 1
            nxt = (not last) or last_bf16
            if self.mode == "bf16":
                y32, y_n = layer(h, w, b, act, a_hi=hi, f32=last and last_f32, bf16=nxt)
            else:
                y32, y_n = layer(h, w, b, act, a_hi=hi, f32=last and last_f32, planes=nxt)
            h, hi = y_n, None
        return ((y32, y_n), inputs) if keep else (y32, y_n)


def dlrm_forward(bottom: MLP, top: MLP, dense_x: torch.Tensor, weights: Sequence[torch.Tensor],
                 indices: torch.Tensor, offsets: torch.Tensor, L: int, *, keep: bool = False):
    """DLRMv1 forward: CTR ``(B, 1)`` f32 from the dense features and the tables.

    ``"bf16"`` MLPs: ``dense_x`` is bf16; bottom MLP -> ``dense`` (f32 for the
    interaction, bf16 for the top MLP); sparse stage -> z ``(B, P)`` f32 ->
    bf16; top MLP with ``[dense | z]`` as its split first-layer input.
    ``"f32"`` MLPs: ``dense_x`` is f32 and every activation stays f32: the
    bottom MLP's output goes to the interaction as f32 and to the top MLP as
    its exact planes, and z is split into planes. With ``keep`` it also
    returns a dict of the intermediate tensors.
    """
    if bottom.mode != top.mode:
        raise ValueError("the bottom and top MLPs must use the same mode")
    if bottom.mode == "f32":
        x_in = split_bf16x3(dense_x)
        dense32, dense_next = bottom.forward(x_in, last_f32=True, last_bf16=True)
        pooled, z = ops.sparse_interact(weights, indices, offsets, dense32, L)
        z_next = split_bf16x3(z)
    else:
        dense32, dense_next = bottom.forward(dense_x, last_f32=True, last_bf16=True)
        pooled, z = ops.sparse_interact(weights, indices, offsets, dense32, L)
        z_next = to_bf16(z)
    (ctr, _), top_inputs = top.forward(dense_next, a_hi=z_next, keep=True)
    if keep:
        return ctr, dict(dense32=dense32, dense16=dense_next, pooled=pooled, z=z, z16=z_next,
                         top_inputs=top_inputs)
    return ctr
