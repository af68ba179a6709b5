"""Oracle for the DLRMv1 sparse/interaction stage (numpy front end).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers. The product path never
imports this package, and this package imports nothing from the product.

The arithmetic lives in ``dlrm_oracle.c`` (plain C loops, built with gcc -O2,
no fast-math, no FMA contraction); this module only compiles it, loads it with
ctypes and marshals numpy arrays. What each function follows on the pages
(luminal compare main...vanilla-pytorch):

* :meth:`Oracle.embbag_sum_multi` -- embedding_bag.rs, module doc comment and
  the multi-table section doc comment (pooled sum over K tables).
* :meth:`Oracle.embbag_pool_multi` -- the same pooling generalised the way
  torch.nn.EmbeddingBag defines it (ragged bags, include_last_offset,
  per-sample weights, mean/max, bf16 tables), which movement.rs
  (translate_embedding_bag_forward_only) names as the extension a later
  model would need.
* :meth:`Oracle.interact_lower_tri` -- dlrm_interact.rs, module doc comment
  (the strict-lower-triangle dot products) and the stacked-kernel doc comment
  (feature 0 = dense vector, features 1..N = pooled embeddings).
* :meth:`Oracle.pair_list` -- dlrm_interact.rs, pair-table comment: row-major
  over i then j, the torch.tril_indices(F, F, -1) order.
* :meth:`Oracle.linear_bf16` / :meth:`Oracle.linear_f32a` -- matmul2d.rs:
  the linear-with-bias layer, its ReLU / sigmoid forms and the split-A form;
  ``linear_f32a`` is the pages' own arithmetic (f32 activations, f32 or bf16
  weights), ``linear_bf16`` the bf16-operand variant.

Every function is pinned by ``tests/test_oracle_pins.py`` to facts fixed by
the pages and by mathematics, not by this code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "dlrm_oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")

OK = 0
BAD_ARG = 1
BAD_OFFSETS = 2
INDEX_OOB = 3

POOL_SUM, POOL_MEAN, POOL_MAX = 0, 1, 2
MODES = {"sum": POOL_SUM, "mean": POOL_MEAN, "max": POOL_MAX}

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


class OracleError(RuntimeError):
    """The oracle rejected its input; ``code`` is one of the codes above."""

    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} rejected its input (code {code})")
        self.code = code


def compile_source(src: str, lib: str) -> str:
    """Compile one C source file into a shared library with the oracle's flags."""
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
    os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """Compile ``dlrm_oracle.c`` into ``liboracle.so`` (if stale) and return its path."""
    if (not force and os.path.exists(LIBRARY)
            and os.path.getmtime(LIBRARY) >= os.path.getmtime(SOURCE)):
        return LIBRARY
    return compile_source(SOURCE, LIBRARY)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


class Oracle:
    """The oracle's functions, bound to one compiled copy of ``dlrm_oracle.c``."""

    def __init__(self, libpath: str):
        lib = ctypes.CDLL(libpath)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_embbag_sum_multi.argtypes = [P, P, P, P, I, I, I, I, P, P, P]
        lib.oracle_embbag_sum_multi.restype = I
        lib.oracle_interact_lower_tri.argtypes = [P, P, I, I, I, P, I, P, P]
        lib.oracle_interact_lower_tri.restype = I
        lib.oracle_embbag_pool_multi.argtypes = [P, I, P, P, P, P, ctypes.c_int64, I, I, I, I,
                                                 I, P]
        lib.oracle_embbag_pool_multi.restype = I
        lib.oracle_pair_list.argtypes = [I, P, P]
        lib.oracle_pair_list.restype = ctypes.c_int64
        L64 = ctypes.c_int64
        lib.oracle_linear_bf16.argtypes = [P, L64, L64, P, L64, L64, P, L64, P, L64, L64, I, P, P,
                                           P]
        lib.oracle_linear_bf16.restype = I
        lib.oracle_linear_f32a.argtypes = [P, L64, L64, P, L64, L64, P, I, L64, P, L64, L64, I, P,
                                           P, P]
        lib.oracle_linear_f32a.restype = I
        self.lib = lib
        self.path = libpath

    def embbag_sum_multi(self, weights: Sequence[np.ndarray], indices: np.ndarray,
                         offsets: np.ndarray, B: int, L: int, *, with_f64: bool = False):
        """Pooled sums ``(B, F, D)`` f32 of F EmbeddingBag(sum) tables.

        ``weights[k]`` is ``(rows_k, D)`` f32; ``indices`` is ``(F, B*L)``
        int32 (table-major); ``offsets`` is ``(F, B)`` int32. With
        ``with_f64`` it also returns the fp64 sums and the per-output sum of
        ``|w|`` over the bag.
        """
        F = len(weights)
        ws = [_f32(w) for w in weights]
        D = int(ws[0].shape[1])
        ptrs = (ctypes.c_void_p * F)(*[w.ctypes.data for w in ws])
        rows = np.array([w.shape[0] for w in ws], dtype=np.int64)
        idx = np.ascontiguousarray(indices, dtype=np.int32).reshape(F, -1)
        off = np.ascontiguousarray(offsets, dtype=np.int32).reshape(F, B)
        out = np.empty((B, F, D), dtype=np.float32)
        o64 = np.empty((B, F, D), dtype=np.float64) if with_f64 else None
        oab = np.empty((B, F, D), dtype=np.float64) if with_f64 else None
        rc = self.lib.oracle_embbag_sum_multi(ctypes.cast(ptrs, ctypes.c_void_p), _ptr(rows),
                                              _ptr(idx), _ptr(off), B, F, L, D, _ptr(out),
                                              _ptr(o64), _ptr(oab))
        if rc != OK:
            raise OracleError(rc, "embbag_sum_multi")
        return (out, o64, oab) if with_f64 else out

    def embbag_pool_multi(self, weights: Sequence[np.ndarray], indices: np.ndarray,
                          offsets: np.ndarray, B: int, *, mode: str = "sum",
                          per_sample_weights: np.ndarray | None = None,
                          include_last_offset: bool = False):
        """General pooling ``(B, F, D)`` f32: ragged bags, weights, sum/mean/max.

        ``weights[k]`` is ``(rows_k, D)`` float32, or uint16 holding bf16 bit
        patterns; ``indices`` (and ``per_sample_weights``) are ``(F, T)``;
        ``offsets`` is ``(F, B)``, or ``(F, B+1)`` with ``include_last_offset``.
        """
        F = len(weights)
        bf16 = weights[0].dtype == np.uint16
        ws = [np.ascontiguousarray(w, dtype=np.uint16 if bf16 else np.float32) for w in weights]
        D = int(ws[0].shape[1])
        ptrs = (ctypes.c_void_p * F)(*[w.ctypes.data for w in ws])
        rows = np.array([w.shape[0] for w in ws], dtype=np.int64)
        idx = np.ascontiguousarray(indices, dtype=np.int32).reshape(F, -1)
        T = idx.shape[1]
        off = np.ascontiguousarray(offsets, dtype=np.int32).reshape(F, B + (1 if include_last_offset else 0))
        psw = None
        if per_sample_weights is not None:
            psw = np.ascontiguousarray(per_sample_weights, dtype=np.float32).reshape(F, T)
        out = np.empty((B, F, D), dtype=np.float32)
        rc = self.lib.oracle_embbag_pool_multi(ctypes.cast(ptrs, ctypes.c_void_p), 1 if bf16 else 0,
                                               _ptr(rows), _ptr(idx), _ptr(off), _ptr(psw), T,
                                               1 if include_last_offset else 0, MODES[mode], B, F,
                                               D, _ptr(out))
        if rc != OK:
            raise OracleError(rc, "embbag_pool_multi")
        return out

    def interact_lower_tri(self, dense: np.ndarray, emb: np.ndarray, *,
                           concat_dense: bool = False, with_f64: bool = False):
        """Strict-lower-triangle dots over ``[dense, emb_0 .. emb_{F-1}]``.

        ``dense`` is ``(B, D)``, ``emb`` is ``(B, F, D)``. Returns ``(B, P)``
        f32 (``(B, D+P)`` with ``concat_dense``), ``P = (F+1)F/2``. With
        ``with_f64`` it also returns the unrounded fp64 dots and the error
        scale ``S_ij = sum_d |v_i v_j|``.
        """
        dn = _f32(dense)
        em = _f32(emb)
        B, F, D = em.shape
        P = (F + 1) * F // 2
        out = np.empty((B, D + P if concat_dense else P), dtype=np.float32)
        o64 = np.empty((B, P), dtype=np.float64) if with_f64 else None
        bnd = np.empty((B, P), dtype=np.float64) if with_f64 else None
        rc = self.lib.oracle_interact_lower_tri(_ptr(dn), _ptr(em), B, F, D, _ptr(out),
                                                1 if concat_dense else 0, _ptr(o64), _ptr(bnd))
        if rc != OK:
            raise OracleError(rc, "interact_lower_tri")
        return (out, o64, bnd) if with_f64 else out

    def sparse_interact(self, weights, indices, offsets, dense, B: int, L: int, *,
                        concat_dense: bool = False, with_bound: bool = False):
        """The whole stage: pooled ``(B,F,D)`` and the interaction row per sample."""
        pooled = self.embbag_sum_multi(weights, indices, offsets, B, L)
        if with_bound:
            inter, _, bound = self.interact_lower_tri(dense, pooled, concat_dense=concat_dense,
                                                      with_f64=True)
            return pooled, inter, bound
        return pooled, self.interact_lower_tri(dense, pooled, concat_dense=concat_dense)

    def pair_list(self, nf: int):
        """``(i, j)`` of the strict lower triangle of ``nf x nf``, nested-loop order."""
        n = nf * (nf - 1) // 2
        pi = np.empty(n, dtype=np.int32)
        pj = np.empty(n, dtype=np.int32)
        got = self.lib.oracle_pair_list(nf, _ptr(pi), _ptr(pj))
        if got != n:
            raise OracleError(-1, "pair_list")
        return pi, pj

    def linear_bf16(self, a_lo: np.ndarray, w: np.ndarray, bias=None, act: int = 0, *,
                    a_hi: Optional[np.ndarray] = None, k_lo: Optional[int] = None,
                    k_hi: Optional[int] = None, k: Optional[int] = None):
        """One MLP layer ``act(A W^T + bias)`` over bf16 operands, exactly (fp64).

        ``a_lo`` ``(M, >=k_lo)``, ``a_hi`` ``(M, >=k_hi)`` (optional) and ``w``
        ``(N, >=k_lo+k_hi)`` are uint16 arrays of bf16 bit patterns (row pitch =
        their second dimension); ``bias`` is ``(N,)`` f32 or None; ``act`` is 0
        (none), 1 (ReLU) or 2 (sigmoid). ``k_lo``/``k_hi`` default to the
        widths of ``a_lo``/``a_hi``. Returns ``(out, pre, bound)``, each
        ``(M, N)`` fp64: the activation, the pre-activation and
        ``sum_k |a_k w_k| + |bias|``.
        """
        a_lo = np.ascontiguousarray(a_lo, dtype=np.uint16)
        w = np.ascontiguousarray(w, dtype=np.uint16)
        M, lda_lo = a_lo.shape
        N, ldw = w.shape
        k_lo = lda_lo if k_lo is None else k_lo
        if a_hi is not None:
            a_hi = np.ascontiguousarray(a_hi, dtype=np.uint16)
            lda_hi = a_hi.shape[1]
            k_hi = lda_hi if k_hi is None else k_hi
        else:
            lda_hi, k_hi = 0, 0
        b = None if bias is None else _f32(bias)
        out = np.empty((M, N), dtype=np.float64)
        pre = np.empty((M, N), dtype=np.float64)
        bnd = np.empty((M, N), dtype=np.float64)
        rc = self.lib.oracle_linear_bf16(_ptr(a_lo), lda_lo, k_lo, _ptr(a_hi), lda_hi, k_hi,
                                         _ptr(w), ldw, _ptr(b), M, N, act, _ptr(out), _ptr(pre),
                                         _ptr(bnd))
        if rc != OK:
            raise OracleError(rc, "linear_bf16")
        return out, pre, bnd


    def linear_f32a(self, a_lo: np.ndarray, w: np.ndarray, bias=None, act: int = 0, *,
                    a_hi: Optional[np.ndarray] = None, k_lo: Optional[int] = None,
                    k_hi: Optional[int] = None):
        """One MLP layer ``act(A W^T + bias)`` with f32 activations, exactly (fp64).

        ``a_lo`` ``(M, >=k_lo)`` and ``a_hi`` ``(M, >=k_hi)`` (optional) are f32;
        ``w`` ``(N, >=k_lo+k_hi)`` is f32 values or uint16 bf16 bit patterns
        (the dtype says which); ``bias`` ``(N,)`` f32 or None; ``act`` as for
        :meth:`linear_bf16`. Returns ``(out, pre, bound)`` like it.
        """
        a_lo = _f32(a_lo)
        w_bf16 = np.asarray(w).dtype == np.uint16
        w = np.ascontiguousarray(w, dtype=np.uint16) if w_bf16 else _f32(w)
        M, lda_lo = a_lo.shape
        N, ldw = w.shape
        k_lo = lda_lo if k_lo is None else k_lo
        if a_hi is not None:
            a_hi = _f32(a_hi)
            lda_hi = a_hi.shape[1]
            k_hi = lda_hi if k_hi is None else k_hi
        else:
            lda_hi, k_hi = 0, 0
        b = None if bias is None else _f32(bias)
        out = np.empty((M, N), dtype=np.float64)
        pre = np.empty((M, N), dtype=np.float64)
        bnd = np.empty((M, N), dtype=np.float64)
        rc = self.lib.oracle_linear_f32a(_ptr(a_lo), lda_lo, k_lo, _ptr(a_hi), lda_hi, k_hi,
                                         _ptr(w), 1 if w_bf16 else 0, ldw, _ptr(b), M, N, act,
                                         _ptr(out), _ptr(pre), _ptr(bnd))
        if rc != OK:
            raise OracleError(rc, "linear_f32a")
        return out, pre, bnd


_default = None


def default() -> Oracle:
    """The oracle built from ``dlrm_oracle.c`` as committed."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def embbag_sum_multi(*a, **k):
    return default().embbag_sum_multi(*a, **k)


def interact_lower_tri(*a, **k):
    return default().interact_lower_tri(*a, **k)


def sparse_interact(*a, **k):
    return default().sparse_interact(*a, **k)


def pair_list(*a, **k):
    return default().pair_list(*a, **k)


def embbag_pool_multi(*a, **k):
    return default().embbag_pool_multi(*a, **k)


def linear_bf16(*a, **k):
    return default().linear_bf16(*a, **k)


def linear_f32a(*a, **k):
    return default().linear_f32a(*a, **k)
