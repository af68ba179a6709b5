"""The MLP layers (tcgen05 GEMM with fused bias/activation, split-A) against
the oracle, on the GPU.

Parity bar: the oracle computes each layer exactly (fp64) from the same bf16
operand bits. The kernel's products are exact and its accumulation is f32, so
the pre-activation may differ by at most (K + 2) * 2^-23 * sum_k |a_k w_k| +
|bias| (K + 1 f32 roundings, each relative to a partial sum bounded by that
magnitude); ReLU keeps that bound, sigmoid (slope <= 1/4) scales it by 1/4
and adds the f32 exp/divide error (a few ulp of the result). The bf16 output
must be exactly the round-to-nearest-even of the kernel's own f32 output.
"""
import numpy as np
import pytest
import torch

import oracle
from dlrm_embedding_bag_b200 import mlp, ops, synthetic as syn

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
ACT_CODE = {"none": 0, "relu": 1, "sigmoid": 2}


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _rand_bf16(g, rows, cols, std=1.0, pitch=None):
    x = torch.empty((rows, cols), device=DEV).normal_(0, std, generator=g)
    buf = mlp.bf16_empty(rows, pitch or cols, DEV)[:, :cols]
    buf.copy_(x.to(torch.bfloat16))
    return buf


def _check_layer(y32, y16, a_lo, w, bias, act, a_hi=None, rows=None, what=""):
    """y32/y16: kernel outputs; rows: optional subset of rows to check."""
    a = a_lo if rows is None else a_lo[rows]
    h = None if a_hi is None else (a_hi if rows is None else a_hi[rows])
    out, pre, bound = oracle.linear_bf16(_bits(a), _bits(w),
                                         None if bias is None else bias.cpu().numpy(),
                                         ACT_CODE[act], a_hi=None if h is None else _bits(h))
    K = w.shape[1]
    slope = 0.25 if act == "sigmoid" else 1.0
    tol = slope * (K + 2) * 2.0 ** -23 * bound + 8 * 2.0 ** -24 * np.abs(out) + 1e-30
    if y32 is not None:
        got = (y32 if rows is None else y32[rows]).double().cpu().numpy()
        err = np.abs(got - out)
        bad = err > tol
        assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside the bound; worst "
                               f"err {err.max():.3e}, tol there {tol.flat[err.argmax()]:.3e}")
    if y16 is not None and y32 is not None:
        want16 = _bits(y32.to(torch.bfloat16))
        assert np.array_equal(_bits(y16), want16), f"{what}: bf16 output is not RNE of f32"


def _run(M, N, K, act="none", bias=True, seed=0, pitch_a=None, pitch_y=None, rows=None,
         bf16=True):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    a = _rand_bf16(g, M, K, 1.0, pitch_a)
    w = _rand_bf16(g, N, K, K ** -0.5)
    b = torch.empty(N, device=DEV).normal_(0, 0.5, generator=g) if bias else None
    y32 = None
    if pitch_y:
        y32 = torch.full((M, pitch_y), float("nan"), device=DEV)[:, :N]
    y32, y16 = mlp.linear_bf16(a, w, b, act, out_f32=y32, bf16=bf16)
    torch.cuda.synchronize()
    _check_layer(y32, y16, a, w, b, act, rows=rows, what=f"M={M} N={N} K={K} {act}")
    return y32, y16


@pytest.mark.parametrize("M,N,K", [(1, 1, 8), (5, 3, 16), (128, 64, 64), (200, 96, 72),
                                   (300, 130, 200), (129, 257, 136), (1000, 512, 592),
                                   (64, 40, 13)])
def test_linear_shapes(M, N, K):
    _run(M, N, K, seed=M + N + K)


@pytest.mark.parametrize("act", ["none", "relu", "sigmoid"])
def test_linear_activations(act):
    y32, _ = _run(333, 200, 96, act=act, seed=7)
    if act == "relu":
        assert (y32 >= 0).all() and (y32 == 0).any()
    if act == "sigmoid":
        assert ((y32 > 0) & (y32 < 1)).all()


def test_linear_no_bias_bf16_only_and_pitched():
    _run(150, 70, 80, bias=False, seed=3)
    _run(150, 70, 80, seed=4, pitch_a=96, pitch_y=75)
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    a = _rand_bf16(g, 77, 40)
    w = _rand_bf16(g, 33, 40)
    y32, _ = mlp.linear_bf16(a, w, None, "relu")
    _, y16 = mlp.linear_bf16(a, w, None, "relu", f32=False, bf16=True)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y16), _bits(y32.to(torch.bfloat16)))


@pytest.mark.parametrize("M,N,K", [(20000, 512, 128), (10000, 256, 192)])
def test_linear_wide_tiles_sampled(M, N, K):
    """Sizes that select 256- and 128-column tiles; the oracle checks 96 rows."""
    rows = torch.from_numpy(np.random.default_rng(M).choice(M, 96, replace=False)).to(DEV)
    _run(M, N, K, act="relu", seed=11, rows=rows)


@pytest.mark.parametrize("M,N,K", [(20000, 512, 592), (10000, 256, 192), (20000, 200, 64),
                                   (300, 130, 200)])
def test_linear_bf16_only_outputs(M, N, K):
    """A layer with only the bf16 output runs the instance without f32 output
    staging (a deeper operand ring at 256-column tiles); its bits are the RNE
    of the f32 results of the instance with staging, checked on sampled rows."""
    g = torch.Generator(device=DEV)
    g.manual_seed(M + N + K)
    a = _rand_bf16(g, M, K)
    w = _rand_bf16(g, N, K, K ** -0.5)
    b = torch.empty(N, device=DEV).normal_(0, 0.5, generator=g)
    y32, _ = mlp.linear_bf16(a, w, b, "relu")
    _, y16 = mlp.linear_bf16(a, w, b, "relu", f32=False, bf16=True)
    torch.cuda.synchronize()
    rows = torch.from_numpy(np.random.default_rng(K).choice(M, min(M, 96),
                                                            replace=False)).to(DEV)
    _check_layer(y32, None, a, w, b, "relu", rows=rows, what=f"M={M} N={N} K={K} f32")
    assert np.array_equal(_bits(y16), _bits(y32.to(torch.bfloat16)))


@pytest.mark.parametrize("k_lo,k_hi", [(64, 528), (128, 351), (24, 40), (8, 8), (64, 0)])
def test_linear_split_a(k_lo, k_hi):
    g = torch.Generator(device=DEV)
    g.manual_seed(k_lo * 1000 + k_hi)
    M, N = 260, 192
    a_lo = _rand_bf16(g, M, k_lo)
    a_hi = _rand_bf16(g, M, k_hi) if k_hi else None
    w = _rand_bf16(g, N, k_lo + k_hi, (k_lo + k_hi) ** -0.5)
    b = torch.empty(N, device=DEV).normal_(0, 0.5, generator=g)
    y32, y16 = mlp.linear_bf16(a_lo, w, b, "relu", a_hi=a_hi, bf16=True)
    torch.cuda.synchronize()
    _check_layer(y32, y16, a_lo, w, b, "relu", a_hi=a_hi, what=f"split {k_lo}+{k_hi}")
    if k_hi and k_lo % 64 == 0:
        # same K blocks as the layer on the concatenation: identical bits
        cat = mlp.bf16_empty(M, k_lo + k_hi, DEV)
        cat[:, :k_lo].copy_(a_lo)
        cat[:, k_lo:].copy_(a_hi)
        c32, _ = mlp.linear_bf16(cat, w, b, "relu")
        torch.cuda.synchronize()
        assert torch.equal(c32.view(torch.int32), y32.view(torch.int32))


def test_f32_to_bf16_matches_torch_rne():
    rng = np.random.default_rng(9)
    bits = rng.integers(0, 2 ** 32, size=(37, 301), dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32).copy()
    x[~np.isfinite(x)] = 0.0
    x[0, :8] = [0.0, -0.0, np.inf, -np.inf, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1e-40, -1e-40]
    xt = torch.from_numpy(x).to(DEV)
    y = mlp.to_bf16(xt)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y), _bits(xt.to(torch.bfloat16)))


def _dlrm_case(seed, B, F, N, D, L, dense_in=13, bot=(64, 32), top=(64, 32)):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    bottom = mlp.MLP(syn.make_mlp_layers(dense_in, list(bot) + [D], seed, DEV), mode="bf16")
    P = (F + 1) * F // 2
    top_m = mlp.MLP(syn.make_mlp_layers(D + P, list(top) + [1], seed + 1, DEV, last="sigmoid"),
                    mode="bf16")
    w = syn.Workload("t", B=B, F=F, N=N, D=D, L=L)
    weights = syn.make_weights(w, DEV)
    idx = torch.from_numpy(syn.make_indices(w)).to(DEV)
    off = torch.from_numpy(syn.make_offsets(w)).to(DEV)
    x = _rand_bf16(g, B, dense_in)
    return bottom, top_m, x, weights, idx, off


def test_mlp_chain_per_layer():
    bottom, _, x, *_ = _dlrm_case(21, 300, 4, 100, 64, 3)
    (y32, _), inputs = bottom.forward(x, keep=True, last_bf16=True)
    torch.cuda.synchronize()
    outs = [inp[0] for inp in inputs[1:]] + [None]
    for i, ((w, b, act), (a, _)) in enumerate(zip(bottom.layers, inputs)):
        if outs[i] is not None:
            # the next layer's bf16 input is this layer's bf16 output; check it
            # against the oracle through its f32 twin recomputed with f32=True
            r32, r16 = mlp.linear_bf16(a, w, b, act, bf16=True)
            torch.cuda.synchronize()
            assert torch.equal(r16.contiguous().view(torch.int16),
                               outs[i].contiguous().view(torch.int16))
            _check_layer(r32, r16, a, w, b, act, what=f"bottom layer {i}")
        else:
            _check_layer(y32, None, a, w, b, act, what=f"bottom layer {i}")


def test_dlrm_forward_chain():
    """Every stage of the forward against the oracle, fed the kernel's own inputs."""
    B, F, N, D, L = 256, 8, 1000, 64, 4
    bottom, top, x, weights, idx, off = _dlrm_case(31, B, F, N, D, L)
    ctr, t = mlp.dlrm_forward(bottom, top, x, weights, idx, off, L, keep=True)
    torch.cuda.synchronize()
    assert ctr.shape == (B, 1) and ((ctr > 0) & (ctr < 1)).all()
    # bottom: last layer's f32 and bf16 outputs agree
    assert np.array_equal(_bits(t["dense16"]), _bits(t["dense32"].to(torch.bfloat16)))
    # sparse stage: pooled bit-exact, z within the dot bound
    wn = [w_.cpu().numpy() for w_ in weights]
    pooled, inter, bound = oracle.sparse_interact(wn, idx.cpu().numpy(), off.cpu().numpy(),
                                                  t["dense32"].cpu().numpy(), B, L,
                                                  with_bound=True)
    assert np.array_equal(t["pooled"].cpu().numpy().view(np.uint32), pooled.view(np.uint32))
    assert np.all(np.abs(t["z"].cpu().numpy().astype(np.float64) - inter) <= 1e-5 * bound + 1e-30)
    assert np.array_equal(_bits(t["z16"]), _bits(t["z"].to(torch.bfloat16)))
    # top: first layer reads [dense | z] through the split form
    (a0, h0) = t["top_inputs"][0]
    w0, b0, act0 = top.layers[0]
    r32, _ = mlp.linear_bf16(a0, w0, b0, act0, a_hi=h0)
    torch.cuda.synchronize()
    _check_layer(r32, None, a0, w0, b0, act0, a_hi=h0, what="top layer 0")
    (a_last, _) = t["top_inputs"][-1]
    wl, bl, actl = top.layers[-1]
    _check_layer(ctr, None, a_last, wl, bl, actl, what="CTR head")


def test_linear_graph_capture_and_launch_count():
    g = torch.Generator(device=DEV)
    g.manual_seed(41)
    a = _rand_bf16(g, 512, 128)
    w = _rand_bf16(g, 256, 128)
    b = torch.zeros(256, device=DEV)
    y = torch.empty((512, 256), device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    n0 = ops.launch_count()
    mlp.linear_bf16(a, w, b, "relu", out_f32=y, status=status)
    assert ops.launch_count() == n0 + 1
    ref = y.clone()
    y.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            mlp.linear_bf16(a, w, b, "relu", out_f32=y, status=status)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    assert int(status.item()) == 0


# ---------------------------------------------------------------------------
# f32 activations (dlrm_linear_f32a): the pages' own arithmetic. Each
# activation is three exact bf16 planes and every product is exact, so the
# only error is the f32 accumulation of the 3K (bf16 weights) or 6K (f32
# weights, whose dropped plane products are below 2^-20 |a w|) products.


def _rand_f32(g, rows, cols, std=1.0):
    return torch.empty((rows, cols), device=DEV).normal_(0, std, generator=g)


def _f32a_tol(bound, out, K, act, w_planes):
    slope = 0.25 if act == "sigmoid" else 1.0
    n = (3 if w_planes == 1 else 6) * K + 2
    rep = 0.0 if w_planes == 1 else 2.0 ** -20
    return slope * (n * 2.0 ** -23 * 1.02 + rep) * bound + 8 * 2.0 ** -24 * np.abs(out) + 1e-30


def _check_f32a(y32, a_lo, w, bias, act, a_hi=None, rows=None, w_planes=1, what=""):
    """a_lo/a_hi: the f32 activations; w: bf16 (N, K) or f32 (N, K) weights."""
    a = a_lo if rows is None else a_lo[rows]
    h = None if a_hi is None else (a_hi if rows is None else a_hi[rows])
    wn = _bits(w) if w.dtype == torch.bfloat16 else w.cpu().numpy()
    out, pre, bound = oracle.linear_f32a(a.cpu().numpy(), wn,
                                         None if bias is None else bias.cpu().numpy(),
                                         ACT_CODE[act],
                                         a_hi=None if h is None else h.cpu().numpy())
    K = w.shape[1]
    tol = _f32a_tol(bound, out, K, act, w_planes)
    got = (y32 if rows is None else y32[rows]).double().cpu().numpy()
    err = np.abs(got - out)
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside the bound; worst "
                           f"err {err.max():.3e}, tol there {tol.flat[err.argmax()]:.3e}")
    return err, bound


def test_split_bf16x3_is_exact():
    """The three planes are bf16 values that sum to the f32 value exactly,
    p0 holds the value's top 8 significant bits and p1 the next 8."""
    rng = np.random.default_rng(19)
    bits = rng.integers(0, 2 ** 32, size=(41, 133), dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32).copy()
    x[~np.isfinite(x)] = 1.0
    x[np.abs(x) < 1e-30] = 0.5  # away from subnormal planes
    x[0, :6] = [0.0, -0.0, 1.0, -3.0, 1.0 + 2 ** -23, -(1.0 + 2 ** -9 + 2 ** -17 + 2 ** -23)]
    xt = torch.from_numpy(x).to(DEV)
    p = mlp.split_bf16x3(xt)
    torch.cuda.synchronize()
    planes = [(_bits(p[i]).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
              for i in range(3)]
    assert np.array_equal(planes[0] + planes[1] + planes[2], x.astype(np.float64))
    assert np.array_equal(_bits(p[0]), (x.view(np.uint32) >> 16).astype(np.uint16))
    r = x.astype(np.float64) - planes[0]
    assert np.array_equal(planes[1], (r.astype(np.float32).view(np.uint32) & 0xffff0000)
                          .view(np.float32).astype(np.float64))


@pytest.mark.parametrize("M,N,K", [(1, 1, 8), (5, 3, 16), (128, 64, 64), (200, 96, 72),
                                   (300, 130, 200), (129, 257, 136), (1000, 512, 592),
                                   (64, 40, 13)])
@pytest.mark.parametrize("wdt", ["bf16", "f32"])
def test_linear_f32a_shapes(M, N, K, wdt):
    g = torch.Generator(device=DEV)
    g.manual_seed(M + N + K)
    a = _rand_f32(g, M, K)
    b = torch.empty(N, device=DEV).normal_(0, 0.5, generator=g)
    if wdt == "bf16":
        w = _rand_bf16(g, N, K, K ** -0.5)
        wk = w
    else:
        w = _rand_f32(g, N, K, K ** -0.5)
        wk = mlp.split_bf16x3(w)
    y32, planes = mlp.linear_f32a(mlp.split_bf16x3(a), wk, b, "none", planes=True)
    torch.cuda.synchronize()
    err, bound = _check_f32a(y32, a, w, b, "none", w_planes=1 if wdt == "bf16" else 3,
                             what=f"M={M} N={N} K={K} {wdt} weights")
    # the planes written for the next layer are the exact split of the f32 result
    p = [(_bits(planes[i]).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
         for i in range(3)]
    assert np.array_equal(p[0] + p[1] + p[2], y32.double().cpu().numpy())
    if wdt == "bf16" and K >= 64:
        # the f32 activations are honoured: the bf16-activation layer is far off
        y16, _ = mlp.linear_bf16(mlp.to_bf16(a), w, b, "none")
        torch.cuda.synchronize()
        e16 = np.abs(y16.double().cpu().numpy() - y32.double().cpu().numpy())
        assert e16.max() > 100 * max(err.max(), 1e-30)


@pytest.mark.parametrize("act", ["none", "relu", "sigmoid"])
def test_linear_f32a_activations(act):
    g = torch.Generator(device=DEV)
    g.manual_seed(77)
    a = _rand_f32(g, 333, 96)
    w = _rand_bf16(g, 200, 96, 96 ** -0.5)
    b = torch.empty(200, device=DEV).normal_(0, 0.5, generator=g)
    y32, _ = mlp.linear_f32a(mlp.split_bf16x3(a), w, b, act)
    torch.cuda.synchronize()
    _check_f32a(y32, a, w, b, act, what=f"f32a {act}")


@pytest.mark.parametrize("k_lo,k_hi", [(64, 528), (128, 351), (24, 40), (8, 8)])
def test_linear_f32a_split_a(k_lo, k_hi):
    g = torch.Generator(device=DEV)
    g.manual_seed(k_lo * 7 + k_hi)
    M, N = 260, 192
    a_lo = _rand_f32(g, M, k_lo)
    a_hi = _rand_f32(g, M, k_hi)
    w = _rand_bf16(g, N, k_lo + k_hi, (k_lo + k_hi) ** -0.5)
    b = torch.empty(N, device=DEV).normal_(0, 0.5, generator=g)
    y32, _ = mlp.linear_f32a(mlp.split_bf16x3(a_lo), w, b, "relu",
                             a_hi=mlp.split_bf16x3(a_hi))
    torch.cuda.synchronize()
    _check_f32a(y32, a_lo, w, b, "relu", a_hi=a_hi, what=f"f32a split {k_lo}+{k_hi}")


@pytest.mark.parametrize("M,N,K", [(20000, 512, 592), (10000, 256, 192)])
def test_linear_f32a_wide_tiles_sampled(M, N, K):
    g = torch.Generator(device=DEV)
    g.manual_seed(M + K)
    a = _rand_f32(g, M, K)
    w = _rand_bf16(g, N, K, K ** -0.5)
    b = torch.empty(N, device=DEV).normal_(0, 0.5, generator=g)
    y32, _ = mlp.linear_f32a(mlp.split_bf16x3(a), w, b, "relu")
    torch.cuda.synchronize()
    rows = torch.from_numpy(np.random.default_rng(M).choice(M, 96, replace=False)).to(DEV)
    _check_f32a(y32, a, w, b, "relu", rows=rows, what=f"f32a M={M} N={N} K={K}")


def test_dlrm_forward_f32_chain():
    """The f32-activation forward, each stage against the oracle on the
    kernel's own f32 inputs: bottom layers, sparse stage, split top layer 0,
    CTR head."""
    B, F, N, D, L = 256, 8, 1000, 64, 4
    g = torch.Generator(device=DEV)
    g.manual_seed(33)
    seed = 41
    bottom = mlp.MLP(syn.make_mlp_layers(13, [64, 32, D], seed, DEV), mode="f32")
    P = (F + 1) * F // 2
    top = mlp.MLP(syn.make_mlp_layers(D + P, [64, 32, 1], seed + 1, DEV, last="sigmoid"),
                  mode="f32")
    w = syn.Workload("t", B=B, F=F, N=N, D=D, L=L)
    weights = syn.make_weights(w, DEV)
    idx = torch.from_numpy(syn.make_indices(w)).to(DEV)
    off = torch.from_numpy(syn.make_offsets(w)).to(DEV)
    x = _rand_f32(g, B, 13).abs()
    ctr, t = mlp.dlrm_forward(bottom, top, x, weights, idx, off, L, keep=True)
    torch.cuda.synchronize()
    assert ctr.shape == (B, 1) and ((ctr > 0) & (ctr < 1)).all()

    def f32_of(planes):
        return sum((_bits(planes[i]).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
                   for i in range(3))

    # the dense features enter as their exact planes
    a_in = torch.from_numpy(f32_of(mlp.split_bf16x3(x)).astype(np.float32)).to(DEV)
    assert torch.equal(a_in, x)
    # the dense vector handed to the top MLP is exactly the f32 one the interaction used
    assert np.array_equal(f32_of(t["dense16"]), t["dense32"].double().cpu().numpy())
    wn = [w_.cpu().numpy() for w_ in weights]
    pooled, inter, bound = oracle.sparse_interact(wn, idx.cpu().numpy(), off.cpu().numpy(),
                                                  t["dense32"].cpu().numpy(), B, L,
                                                  with_bound=True)
    assert np.array_equal(t["pooled"].cpu().numpy().view(np.uint32), pooled.view(np.uint32))
    assert np.all(np.abs(t["z"].cpu().numpy().astype(np.float64) - inter) <= 1e-5 * bound + 1e-30)
    assert np.array_equal(f32_of(t["z16"]), t["z"].double().cpu().numpy())
    (a0, h0) = t["top_inputs"][0]
    w0, b0, act0 = top.layers[0]
    r32, _ = mlp.linear_f32a(a0, w0, b0, act0, a_hi=h0)
    torch.cuda.synchronize()
    _check_f32a(r32, t["dense32"], w0, b0, act0, a_hi=t["z"], what="f32 top layer 0")
    (a_last, _) = t["top_inputs"][-1]
    wl, bl, actl = top.layers[-1]
    a_last32 = torch.from_numpy(f32_of(a_last).astype(np.float32)).to(DEV)
    _check_f32a(ctr, a_last32, wl, bl, actl, what="f32 CTR head")


def _pair_rows(M, n, seed):
    """Sampled rows of a layer run on CTA pairs: random ones plus each half of
    the first and the last 256-row pair (the even and the odd CTA's rows)."""
    rng = np.random.default_rng(seed)
    last = (M - 1) // 256 * 256
    edge = {0, 127, 128, 255, last, min(M - 1, last + 127), min(M - 1, last + 128), M - 1}
    rows = np.unique(np.concatenate([rng.choice(M, n, replace=False),
                                     np.array(sorted(edge))]))
    return torch.from_numpy(rows).to(DEV)


@pytest.mark.parametrize("M,N,k_lo,k_hi", [(65536, 512, 64, 528), (19999, 512, 1024, 0),
                                           (20100, 200, 64, 960), (40000, 256, 512, 0)])
@pytest.mark.parametrize("mode", ["bf16", "f32"])
def test_linear_cta_pair_tiles(M, N, k_lo, k_hi, mode):
    """Layers large enough for 256 x 256 tiles on CTA pairs (cta_group::2,
    every case here, in both activation modes): the DLRMv1 top layer 0 at
    B=65536 (split A), a row count whose last pair has rows only in its even
    CTA, N below one tile with split A, and a 256-wide layer; checked against
    the oracle on sampled rows."""
    g = torch.Generator(device=DEV)
    g.manual_seed(M + N + k_lo + k_hi)
    K = k_lo + k_hi
    b = torch.empty(N, device=DEV).normal_(0, 0.5, generator=g)
    w = _rand_bf16(g, N, K, K ** -0.5)
    rows = _pair_rows(M, 64, M)
    if mode == "bf16":
        a_lo = _rand_bf16(g, M, k_lo)
        a_hi = _rand_bf16(g, M, k_hi) if k_hi else None
        y32, y16 = mlp.linear_bf16(a_lo, w, b, "relu", a_hi=a_hi, bf16=True)
        torch.cuda.synchronize()
        _check_layer(y32, None, a_lo, w, b, "relu", a_hi=a_hi, rows=rows,
                     what=f"pair M={M} N={N} K={k_lo}+{k_hi}")
        assert np.array_equal(_bits(y16), _bits(y32.to(torch.bfloat16)))
    else:
        a_lo = _rand_f32(g, M, k_lo)
        a_hi = _rand_f32(g, M, k_hi) if k_hi else None
        y32, planes = mlp.linear_f32a(mlp.split_bf16x3(a_lo), w, b, "relu",
                                      a_hi=None if a_hi is None else mlp.split_bf16x3(a_hi),
                                      planes=True)
        torch.cuda.synchronize()
        _check_f32a(y32, a_lo, w, b, "relu", a_hi=a_hi, rows=rows,
                    what=f"f32a pair M={M} N={N} K={k_lo}+{k_hi}")
        p = [(_bits(planes[i][rows]).astype(np.uint32) << 16).view(np.float32)
             .astype(np.float64) for i in range(3)]
        assert np.array_equal(p[0] + p[1] + p[2], y32[rows].double().cpu().numpy())


# Layers with K <= 16 (the DLRMv1 bottom MLP reads 13 dense features): one
# zero-filled K block per tile, every output form, the same oracle bounds.
@pytest.mark.parametrize("M,N,K", [(20000, 512, 13), (777, 1000, 16), (513, 9, 5), (3, 1, 1),
                                   (100, 2048, 13), (4099, 64, 7)])
def test_linear_small_k(M, N, K):
    _run(M, N, K, act="relu", seed=M + N + K)


@pytest.mark.parametrize("act", ["none", "relu", "sigmoid"])
def test_linear_small_k_outputs(act):
    # bf16 output alone, pitched outputs, no bias, a column count off the 8-wide groups
    _run(1003, 100, 13, act=act, seed=11, pitch_a=16, pitch_y=104)
    _run(1003, 100, 13, act=act, bias=False, seed=12)
    g = torch.Generator(device=DEV)
    g.manual_seed(13)
    a = _rand_bf16(g, 515, 13, pitch=16)
    w = _rand_bf16(g, 77, 13)
    y32, _ = mlp.linear_bf16(a, w, None, act)
    _, y16 = mlp.linear_bf16(a, w, None, act, f32=False, bf16=True)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y16), _bits(y32.to(torch.bfloat16)))


@pytest.mark.parametrize("M,N,K", [(20000, 512, 13), (300, 1000, 16), (65, 9, 3)])
@pytest.mark.parametrize("wdt", ["bf16", "f32"])
@pytest.mark.parametrize("act", ["relu", "sigmoid"])
def test_linear_f32a_small_k(M, N, K, wdt, act):
    g = torch.Generator(device=DEV)
    g.manual_seed(M + N + K + (wdt == "f32"))
    a = _rand_f32(g, M, K)
    b = torch.empty(N, device=DEV).normal_(0, 0.5, generator=g)
    if wdt == "bf16":
        w = _rand_bf16(g, N, K, K ** -0.5)
        wk = w
    else:
        w = _rand_f32(g, N, K, K ** -0.5)
        wk = mlp.split_bf16x3(w)
    y32, planes = mlp.linear_f32a(mlp.split_bf16x3(a), wk, b, act, planes=True)
    torch.cuda.synchronize()
    _check_f32a(y32, a, w, b, act, w_planes=1 if wdt == "bf16" else 3,
                what=f"M={M} N={N} K={K} {wdt} weights {act}")
    p = [(_bits(planes[i]).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
         for i in range(3)]
    assert np.array_equal(p[0] + p[1] + p[2], y32.double().cpu().numpy())


@pytest.mark.parametrize("M,N,k_lo,k_hi", [(40000, 256, 512, 0), (20100, 200, 64, 960)])
def test_linear_f32a_cta_pairs_f32_weights(M, N, k_lo, k_hi):
    """f32 activations against f32 weights (three weight planes, six plane
    products) on CTA pairs, where each stage holds one A plane: the path the
    bf16-weight layers leave for stages with all three A planes."""
    g = torch.Generator(device=DEV)
    g.manual_seed(M + N + 3)
    K = k_lo + k_hi
    b = torch.empty(N, device=DEV).normal_(0, 0.5, generator=g)
    w = _rand_f32(g, N, K, K ** -0.5)
    a_lo = _rand_f32(g, M, k_lo)
    a_hi = _rand_f32(g, M, k_hi) if k_hi else None
    rows = _pair_rows(M, 64, M + 1)
    y32, _ = mlp.linear_f32a(mlp.split_bf16x3(a_lo), mlp.split_bf16x3(w), b, "relu",
                             a_hi=None if a_hi is None else mlp.split_bf16x3(a_hi))
    torch.cuda.synchronize()
    _check_f32a(y32, a_lo, w, b, "relu", a_hi=a_hi, rows=rows, w_planes=3,
                what=f"f32a pair, f32 weights, M={M} N={N} K={k_lo}+{k_hi}")
