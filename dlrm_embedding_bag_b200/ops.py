"""Python binding of ``libdlrm_sparse.so`` (the C ABI in ``include/dlrm_sparse.h``;
the MLP layers of ``include/dlrm_mlp.h`` are bound in :mod:`.mlp`).

Argument marshalling only: every function checks tensor placement, dtype and
contiguity, passes raw pointers and the current CUDA stream to the C entry
point of the same name, and raises :class:`DlrmError` on a non-zero status.
All arithmetic happens in the library's CUDA kernels. If the library is
missing, importing this module raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_HERE, "libdlrm_sparse.so")

DLRM_MAX_TABLES = 256
STATUS = {
    0: "DLRM_OK",
    -1: "DLRM_ERR_NULL",
    -2: "DLRM_ERR_SHAPE",
    -3: "DLRM_ERR_ALIGN",
    -4: "DLRM_ERR_TOO_MANY_TABLES",
    -5: "DLRM_ERR_INDEX_OOB",
    -6: "DLRM_ERR_OFFSETS",
    -7: "DLRM_ERR_CUDA",
    -8: "DLRM_ERR_TIMEOUT",
    -9: "DLRM_ERR_ARG",
    -10: "DLRM_ERR_SCRATCH",
}
# Bytes of the library's own device staging (dlrm_sparse_interact_host_static).
STATIC_SCRATCH_BYTES = 32 << 20
GATHER_PATHS = {"auto": 0, "ldg": 1}
FLAG_INDEX_OOB = 1
FLAG_OFFSETS = 2
FLAG_TIMEOUT = 4

# Every symbol the header declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
SIGNATURES = {
    "embbag_sum_multi": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "embbag_sum_multi_ex": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "interact_lower_tri": (_I, [_P, _P, _I, _I, _I, _P, _P]),
    "dlrm_sparse_interact": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _I, _P]),
    "dlrm_sparse_interact_ex": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _P]),
    "dlrm_sparse_interact_host": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                                       _P, _P, _P]),
    "embbag_pool_multi": (_I, [_P, _I, _P, _P, _I, _I, _I, _P, _P, _P]),
    "dlrm_sparse_interact_pool": (_I, [_P, _I, _P, _P, _P, _I, _I, _I, _P, _P, _I, _P, _P]),
    "dlrm_sparse_interact_host_static": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "dlrm_pair_decode": (_I, [_I64, _I64, _P, _P, _P]),
    "dlrm_set_gather_path": (_I, [_I]),
    "dlrm_last_gather_path": (_I, []),
    "dlrm_status_from_flags": (_I, [ctypes.c_int32]),
    "dlrm_status_string": (ctypes.c_char_p, [_I]),
    "dlrm_last_cuda_error": (_I, []),
    "dlrm_launch_count": (_I64, []),
    "dlrm_probe_bounded_wait": (_I, [_I64, _P, _P]),
    "dlrm_probe_row_gather": (_I, [_P, _I64, _I, _I64, ctypes.c_uint64, _P, _P]),
    # include/dlrm_mlp.h
    "dlrm_linear_bf16": (_I, [_P, _I64, _I64, _P, _I64, _I64, _P, _I64, _P, _I64, _I64, _I, _P,
                              _I64, _P, _I64, _P, _P]),
    "dlrm_linear_f32a": (_I, [_P, _I64, _I64, _I64, _P, _I64, _I64, _I64, _P, _I64, _I64, _I,
                              _P, _I64, _I64, _I, _P, _I64, _P, _I64, _I64, _P, _P]),
    "dlrm_split_f32_bf16x3": (_I, [_P, _I64, _I64, _I64, _P, _I64, _I64, _P]),
    "dlrm_f32_to_bf16": (_I, [_P, _I64, _I64, _I64, _P, _I64, _P]),
}


class DlrmError(RuntimeError):
    """A library call returned a non-zero ``dlrm_status_t``."""

    def __init__(self, status: int, what: str, detail: str = ""):
        name = STATUS.get(status, str(status))
        msg = f"{what}: {name} ({_lib.dlrm_status_string(status).decode()})"
        if status == -7:
            msg += f", cudaError {_lib.dlrm_last_cuda_error()}"
        super().__init__(msg + (f"; {detail}" if detail else ""))
        self.status = status


def load_library(path: str = LIBRARY) -> ctypes.CDLL:
    """Load the CUDA library and bind every declared symbol; raise if absent."""
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m dlrm_embedding_bag_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library()


def _check(rc: int, what: str):
    if rc != 0:
        raise DlrmError(rc, what)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device (got {t.device})")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _table_ptrs(weights: Sequence[torch.Tensor]):
    F = len(weights)
    if not 1 <= F <= DLRM_MAX_TABLES:
        raise ValueError(f"table count must be in [1, {DLRM_MAX_TABLES}] (got {F})")
    D = weights[0].shape[1]
    for k, w in enumerate(weights):
        _dev(w, f"weights[{k}]", torch.float32)
        if w.dim() != 2 or w.shape[1] != D:
            raise ValueError(f"weights[{k}] must be (rows, {D})")
    arr = (ctypes.c_void_p * F)(*[w.data_ptr() for w in weights])
    rows = (ctypes.c_int64 * F)(*[w.shape[0] for w in weights])
    return arr, rows, F, D


def _bag_args(weights, indices, offsets, L):
    arr, rows, F, D = _table_ptrs(weights)
    if offsets.dim() != 2 or offsets.shape[0] != F:
        raise ValueError(f"offsets must be (F={F}, B)")
    B = offsets.shape[1]
    if indices.numel() != F * B * L:
        raise ValueError(f"indices must hold F*B*L = {F * B * L} entries (got {indices.numel()})")
    ip = _dev(indices, "indices", torch.int32) if indices.numel() else 0
    op = _dev(offsets, "offsets", torch.int32)
    return arr, rows, F, D, B, ip, op


def embbag_sum_multi(weights: Sequence[torch.Tensor], indices: torch.Tensor,
                     offsets: torch.Tensor, L: int, out: Optional[torch.Tensor] = None,
                     status: Optional[torch.Tensor] = None, checked: bool = False) -> torch.Tensor:
    """Pooled ``(B, F, D)`` sums of F EmbeddingBag(sum) tables in one launch.

    ``indices`` is ``(F, B*L)`` int32, ``offsets`` ``(F, B)`` int32. With
    ``checked`` the ``_ex`` entry point runs (indices checked against each
    table's rows; flags OR-ed into ``status``, a 1-element int32 tensor).
    """
    arr, rows, F, D, B, ip, op = _bag_args(weights, indices, offsets, L)
    if out is None:
        out = torch.empty((B, F, D), dtype=torch.float32, device=weights[0].device)
    outp = _dev(out, "out", torch.float32)
    if out.numel() != B * F * D:
        raise ValueError("out must be (B, F, D)")
    if checked:
        sp = _dev(status, "status", torch.int32) if status is not None else None
        _check(_lib.embbag_sum_multi_ex(arr, rows, ip, op, B, F, L, D, outp, sp, _stream()),
               "embbag_sum_multi_ex")
    else:
        _check(_lib.embbag_sum_multi(arr, ip, op, B, F, L, D, outp, _stream()),
               "embbag_sum_multi")
    return out


def interact_lower_tri(dense: torch.Tensor, emb: torch.Tensor,
                       out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """``(B, (F+1)F/2)`` strict-lower-triangle dots over ``[dense, emb_0..emb_{F-1}]``."""
    if emb.dim() != 3:
        raise ValueError("emb must be (B, F, D)")
    B, F, D = emb.shape
    if tuple(dense.shape) != (B, D):
        raise ValueError(f"dense must be ({B}, {D})")
    P = (F + 1) * F // 2
    if out is None:
        out = torch.empty((B, P), dtype=torch.float32, device=emb.device)
    if out.numel() != B * P:
        raise ValueError("out must be (B, P)")
    _check(_lib.interact_lower_tri(_dev(dense, "dense", torch.float32),
                                   _dev(emb, "emb", torch.float32), B, F, D,
                                   _dev(out, "out", torch.float32), _stream()),
           "interact_lower_tri")
    return out


def sparse_interact(weights: Sequence[torch.Tensor], indices: torch.Tensor,
                    offsets: torch.Tensor, dense: torch.Tensor, L: int, *,
                    concat_dense: bool = False, pooled_out=None, inter_out=None,
                    want_pooled: bool = True, status: Optional[torch.Tensor] = None,
                    checked: bool = False):
    """Fused stage: returns ``(pooled or None, inter)``.

    ``inter`` is ``(B, P)``, or ``(B, D+P)`` with ``concat_dense``.
    ``want_pooled=False`` skips writing the pooled vectors to memory.
    """
    arr, rows, F, D, B, ip, op = _bag_args(weights, indices, offsets, L)
    if tuple(dense.shape) != (B, D):
        raise ValueError(f"dense must be ({B}, {D})")
    P = (F + 1) * F // 2
    dev = weights[0].device
    if want_pooled and pooled_out is None:
        pooled_out = torch.empty((B, F, D), dtype=torch.float32, device=dev)
    if inter_out is None:
        inter_out = torch.empty((B, D + P if concat_dense else P), dtype=torch.float32,
                                device=dev)
    pp = _dev(pooled_out, "pooled_out", torch.float32) if pooled_out is not None else None
    if pooled_out is not None and pooled_out.numel() != B * F * D:
        raise ValueError("pooled_out must be (B, F, D)")
    if inter_out.numel() != B * (D + P if concat_dense else P):
        raise ValueError("inter_out has the wrong size")
    dp = _dev(dense, "dense", torch.float32)
    xp = _dev(inter_out, "inter_out", torch.float32)
    if checked:
        sp = _dev(status, "status", torch.int32) if status is not None else None
        _check(_lib.dlrm_sparse_interact_ex(arr, rows, ip, op, dp, B, F, L, D, pp, xp,
                                            1 if concat_dense else 0, sp, _stream()),
               "dlrm_sparse_interact_ex")
    else:
        _check(_lib.dlrm_sparse_interact(arr, ip, op, dp, B, F, L, D, pp, xp,
                                         1 if concat_dense else 0, _stream()),
               "dlrm_sparse_interact")
    return pooled_out, inter_out


POOL_MODES = {"sum": 0, "mean": 1, "max": 2}
TABLE_DTYPES = {torch.float32: 0, torch.bfloat16: 1}


class Bags(ctypes.Structure):
    """``dlrm_bags_t``: where the bags are and how they pool."""

    _fields_ = [("indices", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("per_sample_weights", ctypes.c_void_p), ("T", ctypes.c_int64),
                ("include_last_offset", ctypes.c_int), ("mode", ctypes.c_int)]


def _general_args(weights, indices, offsets, mode, per_sample_weights, include_last_offset,
                  checked):
    F = len(weights)
    if not 1 <= F <= DLRM_MAX_TABLES:
        raise ValueError(f"table count must be in [1, {DLRM_MAX_TABLES}] (got {F})")
    dtype = weights[0].dtype
    if dtype not in TABLE_DTYPES:
        raise TypeError(f"tables must be float32 or bfloat16 (got {dtype})")
    D = weights[0].shape[1]
    for k, w in enumerate(weights):
        _dev(w, f"weights[{k}]", dtype)
        if w.dim() != 2 or w.shape[1] != D:
            raise ValueError(f"weights[{k}] must be (rows, {D})")
    arr = (ctypes.c_void_p * F)(*[w.data_ptr() for w in weights])
    rows = (ctypes.c_int64 * F)(*[w.shape[0] for w in weights]) if checked else None
    if offsets.dim() != 2 or offsets.shape[0] != F:
        raise ValueError(f"offsets must be (F={F}, B{' + 1' if include_last_offset else ''})")
    B = offsets.shape[1] - (1 if include_last_offset else 0)
    T = indices.numel() // F if F else 0
    if indices.numel() != F * T:
        raise ValueError("indices must hold F equal segments")
    bags = Bags(_dev(indices, "indices", torch.int32) if indices.numel() else None,
                _dev(offsets, "offsets", torch.int32),
                _dev(per_sample_weights, "per_sample_weights", torch.float32)
                if per_sample_weights is not None else None,
                T, 1 if include_last_offset else 0, POOL_MODES[mode])
    if per_sample_weights is not None and per_sample_weights.numel() != F * T:
        raise ValueError("per_sample_weights must match indices")
    return arr, TABLE_DTYPES[dtype], rows, bags, F, D, B


def embbag_pool_multi(weights: Sequence[torch.Tensor], indices: torch.Tensor,
                      offsets: torch.Tensor, *, mode: str = "sum",
                      per_sample_weights: Optional[torch.Tensor] = None,
                      include_last_offset: bool = False, checked: bool = False,
                      status: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """General multi-table EmbeddingBag ``(B, F, D)`` f32 in one launch.

    ``weights``: F float32 or bfloat16 tables; ``indices`` (and
    ``per_sample_weights``) ``(F, T)``; ``offsets`` ``(F, B)`` or ``(F, B+1)``
    with ``include_last_offset``; ``mode`` sum/mean/max. ``checked`` checks
    indices against the table sizes (flags in ``status``).
    """
    arr, dt, rows, bags, F, D, B = _general_args(weights, indices, offsets, mode,
                                                 per_sample_weights, include_last_offset,
                                                 checked)
    if out is None:
        out = torch.empty((B, F, D), dtype=torch.float32, device=weights[0].device)
    if out.numel() != B * F * D:
        raise ValueError("out must be (B, F, D)")
    sp = _dev(status, "status", torch.int32) if status is not None else None
    _check(_lib.embbag_pool_multi(arr, dt, rows, ctypes.byref(bags), B, F, D,
                                  _dev(out, "out", torch.float32), sp, _stream()),
           "embbag_pool_multi")
    return out


def sparse_interact_pool(weights: Sequence[torch.Tensor], indices: torch.Tensor,
                         offsets: torch.Tensor, dense: torch.Tensor, *, mode: str = "sum",
                         per_sample_weights: Optional[torch.Tensor] = None,
                         include_last_offset: bool = False, checked: bool = False,
                         status: Optional[torch.Tensor] = None, concat_dense: bool = False,
                         want_pooled: bool = True, pooled_out=None, inter_out=None):
    """Fused stage over the general bag description: ``(pooled or None, inter)``."""
    arr, dt, rows, bags, F, D, B = _general_args(weights, indices, offsets, mode,
                                                 per_sample_weights, include_last_offset,
                                                 checked)
    if tuple(dense.shape) != (B, D):
        raise ValueError(f"dense must be ({B}, {D})")
    P = (F + 1) * F // 2
    dev = weights[0].device
    if want_pooled and pooled_out is None:
        pooled_out = torch.empty((B, F, D), dtype=torch.float32, device=dev)
    if inter_out is None:
        inter_out = torch.empty((B, D + P if concat_dense else P), dtype=torch.float32,
                                device=dev)
    pp = _dev(pooled_out, "pooled_out", torch.float32) if pooled_out is not None else None
    sp = _dev(status, "status", torch.int32) if status is not None else None
    _check(_lib.dlrm_sparse_interact_pool(arr, dt, rows, ctypes.byref(bags),
                                          _dev(dense, "dense", torch.float32), B, F, D, pp,
                                          _dev(inter_out, "inter_out", torch.float32),
                                          1 if concat_dense else 0, sp, _stream()),
           "dlrm_sparse_interact_pool")
    return pooled_out, inter_out


class SparseInteractCall:
    """A prepared ``dlrm_sparse_interact`` call on fixed buffers.

    All arguments are checked and marshalled once; each ``__call__`` is a
    single C call on the current stream (what a serving loop or a CUDA-graph
    capture wants). The object keeps the tensors alive; their contents may
    change between calls, their storage must not.
    """

    def __init__(self, weights: Sequence[torch.Tensor], indices: torch.Tensor,
                 offsets: torch.Tensor, dense: torch.Tensor, L: int, *,
                 concat_dense: bool = False, pooled_out=None, inter_out=None,
                 want_pooled: bool = True):
        arr, _, F, D, B, ip, op = _bag_args(weights, indices, offsets, L)
        if tuple(dense.shape) != (B, D):
            raise ValueError(f"dense must be ({B}, {D})")
        P = (F + 1) * F // 2
        dev = weights[0].device
        if want_pooled and pooled_out is None:
            pooled_out = torch.empty((B, F, D), dtype=torch.float32, device=dev)
        if inter_out is None:
            inter_out = torch.empty((B, D + P if concat_dense else P), dtype=torch.float32,
                                    device=dev)
        if pooled_out is not None and pooled_out.numel() != B * F * D:
            raise ValueError("pooled_out must be (B, F, D)")
        if inter_out.numel() != B * (D + P if concat_dense else P):
            raise ValueError("inter_out has the wrong size")
        pp = _dev(pooled_out, "pooled_out", torch.float32) if pooled_out is not None else None
        self._keep = (list(weights), indices, offsets, dense)
        self.pooled, self.inter = pooled_out, inter_out
        self._args = (arr, ip, op, _dev(dense, "dense", torch.float32), B, F, L, D, pp,
                      _dev(inter_out, "inter_out", torch.float32), 1 if concat_dense else 0)
        self._fn = _lib.dlrm_sparse_interact

    def __call__(self, stream: Optional[int] = None):
        rc = self._fn(*self._args, _stream() if stream is None else stream)
        if rc != 0:
            raise DlrmError(rc, "dlrm_sparse_interact")
        return self.pooled, self.inter


class PoolInteractCall:
    """A prepared ``dlrm_sparse_interact_pool`` call (general bags, modes, bf16
    tables) on fixed buffers: checked and marshalled once, one C call each time."""

    def __init__(self, weights: Sequence[torch.Tensor], indices: torch.Tensor,
                 offsets: torch.Tensor, dense: torch.Tensor, *, mode: str = "sum",
                 per_sample_weights: Optional[torch.Tensor] = None,
                 include_last_offset: bool = False, concat_dense: bool = False,
                 pooled_out=None, inter_out=None, want_pooled: bool = True):
        arr, dt, rows, bags, F, D, B = _general_args(weights, indices, offsets, mode,
                                                     per_sample_weights, include_last_offset,
                                                     False)
        if tuple(dense.shape) != (B, D):
            raise ValueError(f"dense must be ({B}, {D})")
        P = (F + 1) * F // 2
        dev = weights[0].device
        if want_pooled and pooled_out is None:
            pooled_out = torch.empty((B, F, D), dtype=torch.float32, device=dev)
        if inter_out is None:
            inter_out = torch.empty((B, D + P if concat_dense else P), dtype=torch.float32,
                                    device=dev)
        pp = _dev(pooled_out, "pooled_out", torch.float32) if pooled_out is not None else None
        self._keep = (list(weights), indices, offsets, dense, per_sample_weights, bags)
        self.pooled, self.inter = pooled_out, inter_out
        self._args = (arr, dt, rows, ctypes.byref(bags), _dev(dense, "dense", torch.float32), B,
                      F, D, pp, _dev(inter_out, "inter_out", torch.float32),
                      1 if concat_dense else 0, None)
        self._fn = _lib.dlrm_sparse_interact_pool

    def __call__(self, stream: Optional[int] = None):
        rc = self._fn(*self._args, _stream() if stream is None else stream)
        if rc != 0:
            raise DlrmError(rc, "dlrm_sparse_interact_pool")
        return self.pooled, self.inter


def _host(t: torch.Tensor, name: str, dtype: torch.dtype) -> int:
    if t.device.type != "cpu" or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} CPU tensor")
    return t.data_ptr()


class HostStage:
    """The whole stage fed from host memory, through ``dlrm_sparse_interact_host``.

    Holds the device staging buffers (allocated once, by torch) for batches of
    a fixed shape; each :meth:`__call__` enqueues the host-to-device copies,
    the fused launch and the device-to-host copies on the current stream.
    """

    def __init__(self, weights: Sequence[torch.Tensor], B: int, L: int, *,
                 concat_dense: bool = False, want_pooled: bool = False):
        """``want_pooled``: the kernel also writes the pooled vectors (to a
        device staging buffer; they reach the host only if ``pooled_host`` is
        passed to the call)."""
        self.arr, _, self.F, self.D = _table_ptrs(weights)
        self.weights = list(weights)
        self.B, self.L, self.concat = B, L, concat_dense
        dev = weights[0].device
        self.P = (self.F + 1) * self.F // 2
        self.row = self.D + self.P if concat_dense else self.P
        # one device staging block [indices | offsets | dense], so a packed host
        # batch (see pack) crosses PCIe in one copy
        n_idx, n_off, n_dense = self.F * B * L, self.F * B, B * self.D
        self._staging = torch.empty(n_idx + n_off + n_dense, dtype=torch.int32, device=dev)
        self.idx_dev = self._staging[:n_idx]
        self.off_dev = self._staging[n_idx:n_idx + n_off].view(self.F, B)
        self.dense_dev = self._staging[n_idx + n_off:].view(torch.float32).view(B, self.D)
        self.inter_dev = torch.empty((B, self.row), dtype=torch.float32, device=dev)
        self.pooled_dev = (torch.empty((B, self.F, self.D), dtype=torch.float32, device=dev)
                           if want_pooled else None)

    def pack(self, indices_host: torch.Tensor, offsets_host: torch.Tensor,
             dense_host: torch.Tensor):
        """One page-locked host block ``[indices | offsets | dense]`` holding a
        batch, and the three views into it to pass to a call: the library then
        moves the batch with a single host-to-device copy."""
        F, B, L, D = self.F, self.B, self.L, self.D
        n_idx, n_off = F * B * L, F * B
        block = torch.empty(n_idx + n_off + B * D, dtype=torch.int32).pin_memory()
        idx = block[:n_idx]
        off = block[n_idx:n_idx + n_off].view(F, B)
        dense = block[n_idx + n_off:].view(torch.float32).view(B, D)
        idx.copy_(indices_host.reshape(-1))
        off.copy_(offsets_host.reshape(F, B))
        dense.copy_(dense_host.reshape(B, D))
        return idx, off, dense

    def h2d_bytes(self) -> int:
        return 4 * (self.F * self.B * self.L + self.F * self.B + self.B * self.D)

    def d2h_bytes(self, with_pooled: bool = False) -> int:
        n = self.B * self.row
        if with_pooled:
            n += self.B * self.F * self.D
        return 4 * n

    def __call__(self, indices_host, offsets_host, dense_host, inter_host, pooled_host=None):
        F, B, L, D = self.F, self.B, self.L, self.D
        ip = _host(indices_host, "indices_host", torch.int32) if F * B * L else None
        rc = _lib.dlrm_sparse_interact_host(
            self.arr, ip, _host(offsets_host, "offsets_host", torch.int32),
            _host(dense_host, "dense_host", torch.float32), B, F, L, D,
            1 if self.concat else 0, self.idx_dev.data_ptr(), self.off_dev.data_ptr(),
            self.dense_dev.data_ptr(),
            self.pooled_dev.data_ptr() if self.pooled_dev is not None else None,
            self.inter_dev.data_ptr(),
            _host(pooled_host, "pooled_host", torch.float32) if pooled_host is not None else None,
            _host(inter_host, "inter_host", torch.float32), _stream())
        _check(rc, "dlrm_sparse_interact_host")


def sparse_interact_host_static(weights: Sequence[torch.Tensor], indices_host: torch.Tensor,
                                offsets_host: torch.Tensor, dense_host: torch.Tensor, L: int,
                                inter_host: torch.Tensor, *, concat_dense: bool = False,
                                pooled_host: Optional[torch.Tensor] = None) -> None:
    """The whole stage from host buffers through ``dlrm_sparse_interact_host_static``:
    the device staging is the library's own fixed array, so nothing is
    allocated on the device (for callers that cannot allocate device memory).

    Enqueued on the current stream; the host outputs are valid once the
    stream has reached this point. Calls that overlap on the GPU share the
    array and race: keep them on one stream. Staging beyond
    ``STATIC_SCRATCH_BYTES`` raises ``DLRM_ERR_SCRATCH``.
    """
    arr, _, F, D = _table_ptrs(weights)
    if offsets_host.dim() != 2 or offsets_host.shape[0] != F:
        raise ValueError(f"offsets_host must be (F={F}, B)")
    B = offsets_host.shape[1]
    P = (F + 1) * F // 2
    if indices_host.numel() != F * B * L:
        raise ValueError(f"indices_host must hold F*B*L = {F * B * L} entries")
    if tuple(dense_host.shape) != (B, D):
        raise ValueError(f"dense_host must be ({B}, {D})")
    if inter_host.numel() != B * (D + P if concat_dense else P):
        raise ValueError("inter_host has the wrong size")
    if pooled_host is not None and pooled_host.numel() != B * F * D:
        raise ValueError("pooled_host must be (B, F, D)")
    ip = _host(indices_host, "indices_host", torch.int32) if F * B * L else None
    rc = _lib.dlrm_sparse_interact_host_static(
        arr, ip, _host(offsets_host, "offsets_host", torch.int32),
        _host(dense_host, "dense_host", torch.float32), B, F, L, D, 1 if concat_dense else 0,
        _host(pooled_host, "pooled_host", torch.float32) if pooled_host is not None else None,
        _host(inter_host, "inter_host", torch.float32), _stream())
    _check(rc, "dlrm_sparse_interact_host_static")


class HostPipeline:
    """Batches from host memory, overlapped across ``depth`` CUDA streams.

    Each slot owns a :class:`HostStage` (its own device staging buffers) and a
    stream; batch i goes to slot ``i % depth``, so the host-to-device copies of
    one batch run while another batch's kernel and device-to-host copy run.
    :meth:`submit` returns the slot's completion event; the host outputs of a
    batch are valid once its event has completed (:meth:`wait`). A slot is
    reused only after its previous batch completed, so outputs are never
    overwritten while in flight.
    """

    def __init__(self, weights: Sequence[torch.Tensor], B: int, L: int, *,
                 concat_dense: bool = False, want_pooled: bool = False, depth: int = 2):
        dev = weights[0].device
        self.slots = []
        for _ in range(depth):
            stage = HostStage(weights, B, L, concat_dense=concat_dense, want_pooled=want_pooled)
            self.slots.append((stage, torch.cuda.Stream(device=dev), torch.cuda.Event()))
        self.n = 0

    def h2d_bytes(self) -> int:
        return self.slots[0][0].h2d_bytes()

    def d2h_bytes(self) -> int:
        return self.slots[0][0].d2h_bytes()

    def submit(self, indices_host, offsets_host, dense_host, inter_host, pooled_host=None):
        """Enqueue one batch; returns its completion event. The host inputs
        must stay unchanged, and the host outputs unread, until that event
        has completed."""
        stage, stream, done = self.slots[self.n % len(self.slots)]
        self.n += 1
        done.synchronize()  # the slot's previous batch (and its host outputs) is finished
        # work the caller queued before this call (e.g. writes to the tables)
        # comes first
        stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(stream):
            stage(indices_host, offsets_host, dense_host, inter_host, pooled_host)
            done.record(stream)
        return done

    @staticmethod
    def wait(event: "torch.cuda.Event"):
        event.synchronize()

    def drain(self):
        for _, stream, _ in self.slots:
            stream.synchronize()


def pair_decode(p0: int, count: int, device="cuda"):
    """``(i, j)`` int32 tensors from the kernels' closed-form pair decoder."""
    i = torch.empty(count, dtype=torch.int32, device=device)
    j = torch.empty(count, dtype=torch.int32, device=device)
    _check(_lib.dlrm_pair_decode(p0, count, i.data_ptr() if count else None,
                                 j.data_ptr() if count else None, _stream()),
           "dlrm_pair_decode")
    return i, j


def set_gather_path(path: str) -> str:
    """Choose the gather path for later calls ("auto" or "ldg"); returns the old one."""
    prev = _lib.dlrm_set_gather_path(GATHER_PATHS[path])
    if prev < 0:
        raise DlrmError(prev, "dlrm_set_gather_path")
    return {v: k for k, v in GATHER_PATHS.items()}[prev]


def last_gather_path() -> str:
    """The path that served this thread's last gather or fused launch."""
    return {0: "none", 1: "ldg"}[_lib.dlrm_last_gather_path()]


def status_from_flags(flags: int) -> int:
    return _lib.dlrm_status_from_flags(int(flags))


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(_lib.dlrm_launch_count())


def probe_row_gather(table: torch.Tensor, row_bytes: int, count: int, sink: torch.Tensor,
                     seed: int = 0) -> None:
    """Read ``count`` random rows of ``row_bytes`` bytes from ``table`` (any
    contiguous device tensor, taken as ``numel * itemsize // row_bytes`` rows),
    the device's random-row read ceiling without index loads (see the header);
    ``sink`` is one int32 on the device. Time it with events on the current
    stream."""
    if not table.is_cuda or not table.is_contiguous():
        raise ValueError("table must be a contiguous device tensor")
    rows = table.numel() * table.element_size() // row_bytes
    _check(_lib.dlrm_probe_row_gather(table.data_ptr(), rows, row_bytes, count, seed,
                                      _dev(sink, "sink", torch.int32), _stream()),
           "dlrm_probe_row_gather")


def probe_bounded_wait(status: torch.Tensor, limit_cycles: int = 1_000_000) -> None:
    """Run the library's bounded wait on a barrier nothing completes (see the
    header); DLRM_FLAG_TIMEOUT lands in ``status`` (one int32 on the device)."""
    _check(_lib.dlrm_probe_bounded_wait(limit_cycles, _dev(status, "status", torch.int32),
                                        _stream()), "dlrm_probe_bounded_wait")
