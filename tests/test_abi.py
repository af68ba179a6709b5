"""The C-ABI library on the CPU: it loads, exports exactly what the header
declares, and rejects bad arguments on the host before any CUDA call.

None of these calls reaches a kernel launch: every one fails a host-side check
that runs before the library touches the CUDA runtime.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("dlrm_sparse.h", "dlrm_mlp.h")]


def _declared():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"DLRM_API\s+[\w\s\*]+?\b(\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def ops():
    from dlrm_embedding_bag_b200 import build, ops as _ops

    build.build()
    return _ops


def test_header_declares_the_stage_entry_points():
    names = _declared()
    assert {"embbag_sum_multi", "interact_lower_tri", "dlrm_sparse_interact"} <= names
    assert {"dlrm_linear_bf16", "dlrm_f32_to_bf16"} <= names
    assert len(names) == 22


def test_library_exports_every_declared_symbol(ops):
    names = _declared()
    out = subprocess.run(["nm", "-D", "--defined-only", ops.LIBRARY], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert names == exported
    assert names == set(ops.SIGNATURES)
    for n in names:
        assert getattr(ops._lib, n) is not None


def _declarations():
    """name -> (return type, [parameter types]) from the headers' DLRM_API lines."""
    out = {}
    for h in HEADERS:
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for ret, name, params in re.findall(r"DLRM_API\s+([\w\s\*]+?)\b(\w+)\s*\(([^)]*)\)\s*;",
                                            src):
            plist = [] if params.strip() in ("", "void") else [p.strip() for p in params.split(",")]
            types = [re.sub(r"\s*\b\w+$", "", p) if not p.endswith("*") else p for p in plist]
            out[name] = (" ".join(ret.split()), [" ".join(t.split()) for t in types])
    return out


def _ctype_of(decl):
    if "*" in decl or decl == "dlrm_stream_t":
        return ctypes.c_void_p
    return {"int": ctypes.c_int, "int64_t": ctypes.c_int64, "int32_t": ctypes.c_int32,
            "uint64_t": ctypes.c_uint64}[decl]


def test_binding_signatures_match_the_headers(ops):
    """Every ctypes signature in the binding has the header's arity and, per
    argument, the same kind (pointer, int, int32_t or int64_t)."""
    decls = _declarations()
    assert set(decls) == set(ops.SIGNATURES)
    for name, (ret, params) in decls.items():
        res, args = ops.SIGNATURES[name]
        assert len(args) == len(params), name
        for i, (a, p) in enumerate(zip(args, params)):
            assert a is _ctype_of(p), (name, i, p)
        want_ret = ctypes.c_char_p if ret == "const char*" else _ctype_of(ret)
        assert res is want_ret, (name, ret)


def _ptrs(*vals):
    return (ctypes.c_void_p * len(vals))(*vals)


def test_status_strings_and_flags(ops):
    lib = ops._lib
    for code in ops.STATUS:
        assert lib.dlrm_status_string(code)
    assert lib.dlrm_status_string(12345) == b"unknown status"
    assert lib.dlrm_status_from_flags(0) == 0
    assert lib.dlrm_status_from_flags(1) == -5
    assert lib.dlrm_status_from_flags(2) == -6
    assert lib.dlrm_status_from_flags(3) == -5
    assert lib.dlrm_status_from_flags(4) == -8
    assert lib.dlrm_set_gather_path(7) == -9
    assert lib.dlrm_set_gather_path(1) == 0 and lib.dlrm_set_gather_path(0) == 1
    for retired in (2, 3, 4):
        assert lib.dlrm_set_gather_path(retired) == -9
    assert lib.dlrm_launch_count() == 0


FAKE = 0x10000  # never dereferenced: every call below fails a host check first


@pytest.mark.parametrize("case,expect", [
    (dict(F=0), -4), (dict(F=257), -4), (dict(B=0), -2), (dict(L=-1), -2), (dict(D=0), -2),
    (dict(B=1 << 20, L=1 << 12), -2), (dict(weights=None), -1), (dict(offsets=None), -1),
    (dict(indices=None), -1), (dict(out=None), -1), (dict(w0=0), -1),
    (dict(w0=FAKE + 2), -3), (dict(out=FAKE + 1), -3), (dict(offsets=FAKE + 2), -3),
])
def test_embbag_host_checks(ops, case, expect):
    F = case.get("F", 2)
    w0 = case.get("w0", FAKE)
    weights = case.get("weights", _ptrs(*([w0] + [FAKE] * (max(F, 1) - 1))))
    rc = ops._lib.embbag_sum_multi(weights, case.get("indices", FAKE), case.get("offsets", FAKE),
                                   case.get("B", 4), F, case.get("L", 2), case.get("D", 8),
                                   case.get("out", FAKE), None)
    assert rc == expect


def test_checked_entry_points_need_rows(ops):
    rc = ops._lib.embbag_sum_multi_ex(_ptrs(FAKE), None, FAKE, FAKE, 4, 1, 2, 8, FAKE, None, None)
    assert rc == -1
    rows = (ctypes.c_int64 * 1)(-5)
    rc = ops._lib.embbag_sum_multi_ex(_ptrs(FAKE), rows, FAKE, FAKE, 4, 1, 2, 8, FAKE, None, None)
    assert rc == -9


def test_fused_and_interact_host_checks(ops):
    lib = ops._lib
    w = _ptrs(FAKE, FAKE)
    assert lib.dlrm_sparse_interact(w, FAKE, FAKE, None, 4, 2, 2, 8, None, FAKE, 0, None) == -1
    assert lib.dlrm_sparse_interact(w, FAKE, FAKE, FAKE, 4, 2, 2, 8, None, None, 0, None) == -1
    assert lib.dlrm_sparse_interact(w, FAKE, FAKE, FAKE + 1, 4, 2, 2, 8, None, FAKE, 0,
                                    None) == -3
    assert lib.dlrm_sparse_interact(w, FAKE, FAKE, FAKE, 4, 0, 2, 8, None, FAKE, 0, None) == -4
    assert lib.interact_lower_tri(None, FAKE, 4, 2, 8, FAKE, None) == -1
    assert lib.interact_lower_tri(FAKE, FAKE, 0, 2, 8, FAKE, None) == -2
    assert lib.interact_lower_tri(FAKE, FAKE, 4, 300, 8, FAKE, None) == -4
    assert lib.interact_lower_tri(FAKE, FAKE + 2, 4, 2, 8, FAKE, None) == -3
    assert lib.dlrm_sparse_interact_host(w, FAKE, FAKE, FAKE, 4, 2, 2, 8, 0, FAKE, FAKE, FAKE,
                                         None, FAKE, FAKE, None, None) == -1
    assert lib.dlrm_pair_decode(-1, 5, FAKE, FAKE, None) == -9
    assert lib.dlrm_pair_decode(0, -1, FAKE, FAKE, None) == -9
    assert lib.dlrm_pair_decode((1 << 31) - 2, 5, FAKE, FAKE, None) == -9
    assert lib.dlrm_pair_decode(0, 5, None, FAKE, None) == -1
    assert lib.dlrm_launch_count() == 0


def test_static_staging_host_checks(ops):
    """The host entry point with library-owned staging rejects missing host
    buffers and any call whose staging exceeds its fixed array, before any CUDA
    call."""
    lib = ops._lib
    w = _ptrs(FAKE, FAKE)
    call = lib.dlrm_sparse_interact_host_static
    assert call(w, FAKE, FAKE, FAKE, 4, 2, 2, 8, 0, None, None, None) == -1
    assert call(w, None, FAKE, FAKE, 4, 2, 2, 8, 0, None, FAKE, None) == -1
    assert call(w, FAKE, FAKE, FAKE, 4, 0, 2, 8, 0, None, FAKE, None) == -4
    # 2 tables, B = 1 << 20, L = 4: 32 MiB of indices alone
    assert call(w, FAKE, FAKE, FAKE, 1 << 20, 2, 4, 8, 0, None, FAKE, None) == -10
    # pooled vectors that no longer fit once asked for
    B, D = 1 << 14, 256  # inputs 16.2 MiB, dots 0.2 MiB, pooled 32 MiB
    assert call(w, FAKE, FAKE, FAKE, B, 2, 1, D, 0, FAKE, FAKE, None) == -10
    assert lib.dlrm_status_string(-10).startswith(b"the call needs more device staging")
    assert lib.dlrm_launch_count() == 0


def test_general_pooling_host_checks(ops):
    lib = ops._lib
    w = _ptrs(FAKE, FAKE)
    bags = ops.Bags(FAKE, FAKE, None, 8, 0, 0)
    assert lib.embbag_pool_multi(w, 0, None, None, 4, 2, 8, FAKE, None, None) == -1
    assert lib.embbag_pool_multi(w, 2, None, ctypes.byref(bags), 4, 2, 8, FAKE, None, None) == -9
    bad_mode = ops.Bags(FAKE, FAKE, None, 8, 0, 7)
    assert lib.embbag_pool_multi(w, 0, None, ctypes.byref(bad_mode), 4, 2, 8, FAKE, None,
                                 None) == -9
    psw_mean = ops.Bags(FAKE, FAKE, FAKE, 8, 0, 1)
    assert lib.embbag_pool_multi(w, 0, None, ctypes.byref(psw_mean), 4, 2, 8, FAKE, None,
                                 None) == -9
    neg_t = ops.Bags(FAKE, FAKE, None, -1, 0, 0)
    assert lib.embbag_pool_multi(w, 0, None, ctypes.byref(neg_t), 4, 2, 8, FAKE, None,
                                 None) == -2
    no_idx = ops.Bags(None, FAKE, None, 8, 0, 0)
    assert lib.embbag_pool_multi(w, 0, None, ctypes.byref(no_idx), 4, 2, 8, FAKE, None,
                                 None) == -1
    # bf16 tables need 2-byte alignment, f32 tables 4-byte
    w_odd = _ptrs(FAKE + 2, FAKE)
    assert lib.embbag_pool_multi(w_odd, 0, None, ctypes.byref(bags), 4, 2, 8, FAKE, None,
                                 None) == -3
    assert lib.embbag_pool_multi(w_odd, 1, None, ctypes.byref(bags), 4, 2, 8, None, None,
                                 None) == -1
    rows = (ctypes.c_int64 * 2)(5, -1)
    assert lib.embbag_pool_multi(w, 0, rows, ctypes.byref(bags), 4, 2, 8, FAKE, None,
                                 None) == -9
    assert lib.dlrm_sparse_interact_pool(w, 0, None, ctypes.byref(bags), None, 4, 2, 8, None,
                                         FAKE, 0, None, None) == -1
    assert lib.dlrm_launch_count() == 0


def test_missing_library_fails_loudly(ops, tmp_path):
    with pytest.raises(ImportError, match="no CPU fallback"):
        ops.load_library(str(tmp_path / "libdlrm_sparse.so"))


def test_linear_host_checks(ops):
    """Bad MLP-layer arguments are rejected before any CUDA call."""
    lib = ops._lib
    A = 0x10000  # a 16-byte aligned non-null address that is never dereferenced
    W = 0x20000
    Y = 0x30000

    def call(a_lo=A, lda_lo=64, k_lo=64, a_hi=None, lda_hi=0, k_hi=0, w=W, ldw=64, bias=None,
             M=4, N=8, act=0, y32=Y, ld32=8, y16=None, ld16=0, status=None):
        return lib.dlrm_linear_bf16(a_lo, lda_lo, k_lo, a_hi, lda_hi, k_hi, w, ldw, bias, M, N,
                                    act, y32, ld32, y16, ld16, status, None)

    assert call(a_lo=None) == -1
    assert call(w=None) == -1
    assert call(y32=None) == -1
    assert call(k_hi=8, lda_hi=8, ldw=72) == -1          # a_hi missing
    assert call(act=3) == -9
    assert call(M=0) == -2 and call(N=0) == -2 and call(k_lo=0) == -2
    assert call(lda_lo=56) == -2                          # pitch < k
    assert call(ldw=56) == -2
    assert call(ld32=7) == -2
    assert call(lda_lo=68, k_lo=60, ldw=64) == -3         # pitch not a multiple of 8
    assert call(a_lo=A + 8) == -3                         # 8-byte aligned only
    assert call(k_lo=60, ldw=72, a_hi=A, lda_hi=8, k_hi=8) == -3  # k_lo % 8 with a split
    assert call(y32=Y + 2) == -3
    assert lib.dlrm_f32_to_bf16(None, 4, 1, 4, Y, 4, None) == -1
    assert lib.dlrm_f32_to_bf16(A, 3, 1, 4, Y, 4, None) == -2
    assert lib.dlrm_f32_to_bf16(A + 2, 4, 1, 4, Y, 4, None) == -3


def test_probe_host_checks(ops):
    lib = ops._lib
    assert lib.dlrm_probe_bounded_wait(1000, None, None) == -1
    assert lib.dlrm_probe_bounded_wait(1000, 0x10002, None) == -3
    T, S = 0x10000, 0x20000  # never dereferenced: every call fails its host checks
    assert lib.dlrm_probe_row_gather(None, 10, 256, 5, 0, S, None) == -1
    assert lib.dlrm_probe_row_gather(T, 10, 256, 5, 0, None, None) == -1
    for rb in (0, 8, 48, 100, 1024):
        assert lib.dlrm_probe_row_gather(T, 10, rb, 5, 0, S, None) == -2, rb
    assert lib.dlrm_probe_row_gather(T, 0, 256, 5, 0, S, None) == -2
    assert lib.dlrm_probe_row_gather(T, 10, 256, -1, 0, S, None) == -2
    assert lib.dlrm_probe_row_gather(T + 8, 10, 256, 5, 0, S, None) == -3
    assert lib.dlrm_probe_row_gather(T, 10, 256, 5, 0, S + 2, None) == -3


def test_header_compiles_as_c_and_matches_the_binding(ops, tmp_path):
    """The headers are plain C: a probe built with gcc reports the layout of
    dlrm_bags_t and the constants, which must equal what the binding passes."""
    from dlrm_embedding_bag_b200 import mlp

    probe = tmp_path / "probe.c"
    probe.write_text(r"""
#include <stddef.h>
#include <stdio.h>
#include "dlrm_sparse.h"
#include "dlrm_mlp.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu\n", sizeof(dlrm_bags_t),
         offsetof(dlrm_bags_t, indices), offsetof(dlrm_bags_t, offsets),
         offsetof(dlrm_bags_t, per_sample_weights), offsetof(dlrm_bags_t, T),
         offsetof(dlrm_bags_t, include_last_offset), offsetof(dlrm_bags_t, mode));
  printf("%d %d %d %d %d %d %d\n", DLRM_MAX_TABLES, DLRM_FLAG_INDEX_OOB, DLRM_FLAG_OFFSETS,
         DLRM_FLAG_TIMEOUT, DLRM_POOL_SUM, DLRM_POOL_MEAN, DLRM_POOL_MAX);
  printf("%d %d %d %d\n", DLRM_TABLE_F32, DLRM_TABLE_BF16, DLRM_PATH_AUTO, DLRM_PATH_LDG);
  printf("%d %d %d\n", DLRM_ACT_NONE, DLRM_ACT_RELU, DLRM_ACT_SIGMOID);
  return 0;
}
""")
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(probe), "-o", str(exe)], check=True)
    lines = subprocess.run([str(exe)], capture_output=True, text=True,
                           check=True).stdout.split("\n")
    layout = [int(v) for v in lines[0].split()]
    B = ops.Bags
    assert layout == [ctypes.sizeof(B), B.indices.offset, B.offsets.offset,
                      B.per_sample_weights.offset, B.T.offset, B.include_last_offset.offset,
                      B.mode.offset]
    consts = [int(v) for v in lines[1].split()]
    assert consts == [ops.DLRM_MAX_TABLES, ops.FLAG_INDEX_OOB, ops.FLAG_OFFSETS,
                      ops.FLAG_TIMEOUT, ops.POOL_MODES["sum"], ops.POOL_MODES["mean"],
                      ops.POOL_MODES["max"]]
    paths = [int(v) for v in lines[2].split()]
    import torch
    assert paths[:2] == [ops.TABLE_DTYPES[torch.float32], ops.TABLE_DTYPES[torch.bfloat16]]
    assert paths[2:] == [ops.GATHER_PATHS[p] for p in ("auto", "ldg")]
    assert [int(v) for v in lines[3].split()] == [mlp.ACTS[a] for a in ("none", "relu",
                                                                        "sigmoid")]
