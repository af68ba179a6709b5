"""Python binding of the DLRMv1 MLP layers (the C ABI in ``include/dlrm_mlp.h``).

Argument marshalling only, as in :mod:`.ops`: pointers, row pitches and the
current stream go to ``dlrm_linear_bf16`` / ``dlrm_f32_to_bf16``; every layer
runs in the library's tcgen05 kernel. bf16 tensors are ``torch.bfloat16``
views whose row pitch is a multiple of 8 elements (16 bytes), as the layer's
TMA loads require; :func:`bf16_empty` makes such buffers.

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


class MLP:
    """A stack of bf16 layers ``(w, bias, act)``; intermediate activations are bf16.

    ``w`` is a bf16 ``(N, K)`` tensor (pitched, see :func:`bf16_empty`), ``bias``
    ``(N,)`` f32, ``act`` one of ``"none" | "relu" | "sigmoid"``.
    """

    def __init__(self, layers: Sequence[Tuple[torch.Tensor, torch.Tensor, str]]):
        if not layers:
            raise ValueError("an MLP needs at least one layer")
        self.layers: List[Tuple[torch.Tensor, torch.Tensor, str]] = list(layers)

    @property
    def out_features(self) -> int:
        return self.layers[-1][0].shape[0]

    def forward(self, x: torch.Tensor, *, a_hi: Optional[torch.Tensor] = None,
                last_f32: bool = True, last_bf16: bool = False, keep: bool = False):
        """Run the layers on bf16 ``x`` (and ``a_hi`` for the first layer's split form).

        Returns ``(y_f32, y_bf16)`` of the last layer, plus the list of every
        layer's bf16 input when ``keep`` is set.
        """
        inputs = []
        h, hi = x, a_hi
        n = len(self.layers)
        for i, (w, b, act) in enumerate(self.layers):
            inputs.append((h, hi))
            last = i == n - 1
            y32, y16 = linear_bf16(h, w, b, act, a_hi=hi, f32=last and last_f32,
                                   bf16=(not last) or last_bf16)
            h, hi = y16, None
        return ((y32, y16), inputs) if keep else (y32, y16)


def dlrm_forward(bottom: MLP, top: MLP, dense_x: torch.Tensor, weights: Sequence[torch.Tensor],
                 indices: torch.Tensor, offsets: torch.Tensor, L: int, *, keep: bool = False):
    """DLRMv1 forward: CTR ``(B, 1)`` f32 from bf16 dense features and the tables.

    bottom MLP -> ``dense`` (f32 for the interaction, bf16 for the top MLP);
    sparse stage -> z ``(B, P)`` f32 -> bf16; top MLP with ``[dense | z]`` as
    its split first-layer input. With ``keep`` it also returns a dict of the
    intermediate tensors.
    """
    dense32, dense16 = bottom.forward(dense_x, last_f32=True, last_bf16=True)
    pooled, z = ops.sparse_interact(weights, indices, offsets, dense32, L)
    z16 = to_bf16(z)
    (ctr, _), top_inputs = top.forward(dense16, a_hi=z16, keep=True)
    if keep:
        return ctr, dict(dense32=dense32, dense16=dense16, pooled=pooled, z=z, z16=z16,
                         top_inputs=top_inputs)
    return ctr
