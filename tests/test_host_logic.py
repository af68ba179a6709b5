"""Host-side logic of the test and bench harness, on the CPU."""
import numpy as np
import torch

import oracle
from gpu_cases import sampled_oracle


def test_sampled_oracle_matches_full_oracle():
    rng = np.random.default_rng(3)
    B, F, N, D, L = 37, 3, 50, 8, 5
    weights = [torch.from_numpy(rng.normal(0, 0.1, (N, D)).astype(np.float32)) for _ in range(F)]
    idx = rng.integers(0, N, (F, B * L)).astype(np.int32)
    # ragged offsets with some empty bags
    offs = np.sort(rng.integers(0, B * L + 1, (F, B)), axis=1).astype(np.int32)
    offs[:, 0] = 0
    dense = torch.from_numpy(rng.normal(0, 1, (B, D)).astype(np.float32))
    ws = [w.numpy() for w in weights]
    pooled = oracle.embbag_sum_multi(ws, idx, offs, B, L)
    inter = oracle.interact_lower_tri(dense.numpy(), pooled, concat_dense=True)
    samples = np.array([0, 5, 17, 36])
    sp, si, sb = sampled_oracle(weights, idx, offs, dense, B, L, samples, True)
    assert np.array_equal(sp.view(np.uint32), pooled[samples].view(np.uint32))
    assert np.array_equal(si.view(np.uint32), inter[samples].view(np.uint32))
    assert sb.shape == (4, F * (F + 1) // 2)


def test_algorithmic_bytes_model():
    """The roofline's byte model at the benchmark workload: 294,518,784 bytes per
    fused step (268.44 MB of rows, 4.19 MB of row ids, 0.26 MB of offsets,
    0.52 MB of dense rows, 16.78 MB of pooled rows, 4.33 MB of dots)."""
    import bench
    from dlrm_embedding_bag_b200 import synthetic as syn
    w = syn.C3_ZIPF
    assert bench.algorithmic_bytes(w) == 294_518_784
    parts = {"rows": 2048 * 32 * 16 * 64 * 4, "ids": 2048 * 32 * 16 * 4, "offsets": 2048 * 32 * 4,
             "dense": 2048 * 64 * 4, "pooled": 2048 * 32 * 64 * 4, "dots": 2048 * 528 * 4}
    assert sum(parts.values()) == 294_518_784
    # without the pooled output, with 2-byte rows, with a 4-byte weight per entry
    assert bench.algorithmic_bytes(w, write_pooled=False) == 294_518_784 - parts["pooled"]
    assert bench.algorithmic_bytes(w, esz=2) == 294_518_784 - parts["rows"] // 2
    assert bench.algorithmic_bytes(w, weighted=True) == 294_518_784 + parts["ids"]
    # concatenated rows [dense | dots] at c2
    c2 = syn.C2_CONCAT
    assert bench.algorithmic_bytes(c2) == (2048 * 8 * 32 * 64 * 4 + 2048 * 8 * 32 * 4
                                           + 2048 * 8 * 4 + 2048 * 64 * 4
                                           + 2048 * 8 * 64 * 4 + 2048 * (64 + 36) * 4)


def test_recorded_traffic_applies_only_to_unchanged_sources(tmp_path, monkeypatch):
    """The committed DRAM figure is reported only while the fused kernel's
    sources still hash to the digest it was captured with."""
    import json
    import bench
    rec = {"w": {"source_digest": bench.source_digest(), "dram_bytes_per_launch": 123}}
    (tmp_path / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    assert bench.recorded_traffic("w") == 123
    assert bench.recorded_traffic("other") is None
    rec["w"]["source_digest"] = "0" * 16
    (tmp_path / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("w") is None


def test_oracle_and_cuda_path_share_no_code():
    """The oracle (test infrastructure) and the product are independent: the
    package and its CUDA sources never import or include the oracle, and the
    oracle never imports the package or includes its sources."""
    import os
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "dlrm_embedding_bag_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), f
                assert "dlrm_oracle" not in src, f
    for f in os.listdir(os.path.join(root, "oracle")):
        if f.endswith((".py", ".c", ".h")):
            src = open(os.path.join(root, "oracle", f)).read()
            assert not re.search(r"^\s*(import|from)\s+dlrm_embedding_bag_b200\b", src, re.M), f
            assert not re.search(r"#\s*include\s*[<\"].*(csrc|dlrm_sparse|dlrm_mlp)", src), f


def test_fused_bag_rounds_cover_every_bag_once():
    """The fused kernel's round structure (256 threads, lane groups of G lanes,
    slot = round * groups + group, mirrored in odd rounds when the bags are
    ordered): every bag of a block is taken exactly once, and all slots of a
    warp in a round lie in one run of 32 bags -- the property that lets each
    warp sort and keep one run at a time without a block-wide barrier."""
    threads = 256
    for G in (4, 8, 16, 32):
        groups = threads // G
        for S in (1, 2, 3, 4):
            for F in (1, 2, 3, 5, 8, 26, 32, 33, 100, 256):
                if S * F >= 2048:
                    continue
                rounds = -(-S * F // groups)
                for ntasks in {S * F, max(1, S * F - F)}:  # full block and a tail block
                    for ordered in (False, True):
                        seen = []
                        for rd in range(rounds):
                            for warp in range(threads // 32):
                                gs = range(warp * 32 // G, (warp + 1) * 32 // G)
                                slots = [rd * groups + ((groups - 1 - g) if ordered and rd & 1
                                                        else g) for g in gs]
                                assert len({s >> 5 for s in slots}) == 1, (G, S, F, rd, warp)
                                seen += [s for s in slots if s < ntasks]
                        assert sorted(seen) == list(range(ntasks)), (G, S, F, ordered)


def test_warp_bitonic_network_sorts_descending():
    """The 32-lane bitonic network of the fused kernel's bag ordering (phase k,
    step j: the lane keeps the larger of itself and lane ^ j exactly when bit j
    and bit k of its index agree) sorts any keys descending; keys are
    (min(length, 2^21 - 2) + 1) << 11 | bag, so empty slots (key 0) go last and
    keys are unique (ties in length order by bag number, higher first)."""
    def network(keys):
        keys = list(keys)
        k = 2
        while k <= 32:
            j = k >> 1
            while j:
                other = [keys[lane ^ j] for lane in range(32)]
                keys = [max(keys[lane], other[lane]) if ((lane & j) == 0) == ((lane & k) == 0)
                        else min(keys[lane], other[lane]) for lane in range(32)]
                j >>= 1
            k <<= 1
        return keys

    rng = np.random.default_rng(1)
    for trial in range(300):
        n = int(rng.integers(0, 33))
        lengths = rng.integers(0, 40 if trial % 2 else 3, n)
        keys = [((min(int(ln), (1 << 21) - 2) + 1) << 11) | t for t, ln in enumerate(lengths)]
        keys += [0] * (32 - n)
        perm = rng.permutation(32)
        out = network([keys[p] for p in perm])
        assert out == sorted(keys, reverse=True)
        bags = [key & 2047 for key in out[:n]]
        # longest first; among equal lengths the higher bag number first
        assert [(int(lengths[b]), b) for b in bags] == sorted(
            ((int(lengths[b]), b) for b in bags), reverse=True)
