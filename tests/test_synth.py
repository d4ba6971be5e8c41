"""The seeded input generators: rounding, reproducibility, shapes (no GPU)."""
import numpy as np
import torch

import block_draft_synth as syn


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -7e-39], dtype=np.float32)])
    ours = syn.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = syn.bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_streams_are_independent_and_reproducible():
    w = syn.workload(0)
    a = syn.hidden(w)
    E1, M1 = syn.selector_tables(w)
    b = syn.hidden(w)
    np.testing.assert_array_equal(a, b)
    E2, _ = syn.selector_tables(w)
    np.testing.assert_array_equal(E1, E2)
    assert not np.array_equal(syn.hidden(syn.workload(0)), syn._normal_bf16(syn.rng_for(0, "W"), a.shape, 1.0))


def test_shapes_and_distributions_tiny():
    w = syn.workload("tiny")
    H, W = syn.hidden(w), syn.lm_head(w)
    assert H.shape == (4, 256) and W.shape == (4096, 256)
    assert abs(syn.bf16_bits_to_f32(W).std() - 1 / 16) < 2e-3
    a0, a1 = syn.conv_taps(w)
    a0f, a1f = syn.bf16_bits_to_f32(a0), syn.bf16_bits_to_f32(a1)
    assert a0f.min() >= 0.5 and a0f.max() <= 1.0 and a1f.min() >= 0.0 and a1f.max() <= 0.5
    x, prev = syn.conv_input(w)
    assert x.shape == (1, 5, 256) and prev.shape == (1, 256)
    Hn = syn.target_hidden(w, H)
    assert Hn.shape == (5, 256)


def test_synthetic_topk_is_a_valid_list():
    logp, idx = syn.synthetic_topk(10, 7, 5000, 1)
    assert (np.diff(logp, axis=1) <= 0).all() and (logp <= 0).all()
    assert all(len(set(r)) == 16 for r in idx.tolist())
    assert idx.min() >= 0 and idx.max() < 5000


def test_workload_table():
    names = [w.name for w in syn.WORKLOADS]
    assert names == ["tiny", "qwen3-4b-bs1", "qwen3-4b-batched", "27b-class", "throughput"]
    assert [w.M for w in syn.WORKLOADS] == [4, 7, 448, 80, 4096]
