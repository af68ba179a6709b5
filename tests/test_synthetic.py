"""The seeded input generators (CPU only): ranges, laws and determinism."""
import numpy as np
import torch

from dlrm_embedding_bag_b200 import synthetic as syn


def test_configs_have_stated_shapes():
    assert (syn.TINY.B, syn.TINY.F, syn.TINY.N, syn.TINY.D, syn.TINY.L) == (16, 2, 1000, 16, 4)
    assert syn.TINY.P == 3
    assert syn.C2_CONCAT.P == 36 and syn.C2_CONCAT.concat_dense
    assert syn.C3_ZIPF.P == 528 and syn.C3_ZIPF.table_bytes == 32 * 10 ** 6 * 64 * 4
    assert syn.C5_ZIPF.P == 351
    cells = list(syn.sweep())
    assert len(cells) == 55
    assert {c.B for c in cells} == {2 ** i for i in range(11)}
    assert {c.F for c in cells} == {1, 4, 8, 16, 32}


def test_uniform_indices_in_range_and_deterministic():
    w = syn.TINY
    a = syn.make_indices(w)
    b = syn.make_indices(w)
    assert a.dtype == np.int32 and a.shape == (w.F, w.B * w.L)
    assert np.array_equal(a, b)
    assert a.min() >= 0 and a.max() < w.N
    assert not np.array_equal(a[0], a[1])  # tables draw from their own streams


def test_zipf_law_and_scatter():
    w = syn.Workload("z", B=4096, F=1, N=1000, D=4, L=50, dist="zipf", alpha=1.2)
    rng = np.random.Generator(np.random.PCG64(99))
    r = syn.zipf_ranks(rng, 200_000, w.N, w.alpha)
    pmf = np.arange(1, w.N + 1, dtype=np.float64) ** -w.alpha
    pmf /= pmf.sum()
    freq = np.bincount(r, minlength=w.N) / r.size
    # top ranks within 5 standard errors of the law
    se = np.sqrt(pmf[:10] * (1 - pmf[:10]) / r.size)
    assert np.all(np.abs(freq[:10] - pmf[:10]) <= 5 * se)
    idx = syn.table_indices(w, 0)
    top = np.bincount(idx, minlength=w.N).argmax()
    # rank 1 is mapped through the table's permutation, not to row 0
    perm = np.random.Generator(np.random.PCG64(4000)).permutation(w.N)
    assert top == perm[0]
    assert idx.min() >= 0 and idx.max() < w.N


def test_fixed_stride_offsets():
    w = syn.C2_CONCAT.scaled(B=5)
    off = syn.make_offsets(w)
    assert off.dtype == np.int32 and off.shape == (w.F, 5)
    assert np.array_equal(off[3], np.arange(5) * w.L)


def test_weights_and_dense_seeded():
    w = syn.TINY
    t1 = syn.make_weights(w)
    t2 = syn.make_weights(w)
    assert len(t1) == w.F and t1[0].shape == (w.N, w.D) and t1[0].dtype == torch.float32
    assert all(torch.equal(a, b) for a, b in zip(t1, t2))
    assert abs(float(t1[0].std()) - 0.1) < 0.01
    d = syn.make_dense(w)
    assert d.shape == (w.B, w.D) and torch.equal(d, syn.make_dense(w))


def test_ragged_offsets_cover_the_same_entries():
    """Ragged bags: sorted cut points on [0, B*L], first bag at 0, mean length L,
    seeded per table (PCG64(6000 + k))."""
    w = syn.C3_ZIPF.scaled(B=512)
    off = syn.make_ragged_offsets(w)
    T = w.B * w.L
    assert off.dtype == np.int32 and off.shape == (w.F, w.B)
    assert np.array_equal(off, syn.make_ragged_offsets(w))
    assert np.all(off[:, 0] == 0)
    assert np.all(np.diff(off, axis=1) >= 0) and off.max() <= T
    lengths = np.diff(np.concatenate([off, np.full((w.F, 1), T)], axis=1), axis=1)
    assert np.all(lengths.sum(axis=1) == T)          # every entry in exactly one bag
    assert abs(lengths.mean() - w.L) < 1e-9          # mean length L
    assert (lengths == 0).any() and lengths.max() > 3 * w.L   # really ragged
    assert not np.array_equal(off[0], off[1])


def test_sample_weights_seeded_in_unit_interval():
    w = syn.TINY
    a = syn.make_sample_weights(w)
    assert a.dtype == np.float32 and a.shape == (w.F, w.B * w.L)
    assert np.array_equal(a, syn.make_sample_weights(w))
    assert a.min() >= 0.0 and a.max() < 1.0
    assert not np.array_equal(a[0], a[1])


def test_mlp_layers_shapes_and_dtypes():
    layers = syn.make_mlp_layers(13, [512, 256, 64], 7, "cpu")
    assert [tuple(wt.shape) for wt, _, _ in layers] == [(512, 13), (256, 512), (64, 256)]
    assert all(wt.dtype == torch.bfloat16 and b.dtype == torch.float32 for wt, b, _ in layers)
    assert [act for _, _, act in layers] == ["relu", "relu", "relu"]
    top = syn.make_mlp_layers(592, [512, 256, 1], 8, "cpu", last="sigmoid")
    assert top[-1][2] == "sigmoid" and top[0][2] == "relu"
    again = syn.make_mlp_layers(13, [512, 256, 64], 7, "cpu")
    assert all(torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
               for a, b in zip(layers, again))
