"""Dynamic-tap conv (and the plain tensor-core GEMM it uses) on the GPU
against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import block_draft_synth as syn
from helpers import dev_bf16, bf16_out_to_f64, logits_bound

pytestmark = pytest.mark.gpu


def _bits(a):
    return syn.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


@pytest.mark.parametrize("M,N,K", [(7, 320, 2560), (1, 16, 64), (130, 48, 192), (512, 640, 512), (33, 1000, 128),
                                   (1, 16, 8192), (113, 512, 2560), (100, 2000, 1024)])
def test_gemm_within_bound(M, N, K):
    import block_draft_selection_b200 as bds
    rng = syn.rng_for(M + N + K, "gate")
    A = _bits(rng.standard_normal((M, K)))
    B = _bits(rng.standard_normal((N, K)) / np.sqrt(K))
    C = bds.dflash_gemm_bf16(dev_bf16(A), dev_bf16(B))
    torch.cuda.synchronize()
    ref = oracle.logits(A, B)          # the same contraction, float64
    err = np.abs(C.cpu().numpy().astype(np.float64) - ref)
    assert (err <= logits_bound(A, B)).all(), err.max()


def _run(x, prev, a0, a1, wc):
    import block_draft_selection_b200 as bds
    y = bds.dflash_conv2tap_dynamic(dev_bf16(x), dev_bf16(a0), dev_bf16(a1), dev_bf16(wc),
                                    None if prev is None else dev_bf16(prev))
    torch.cuda.synchronize()
    return bf16_out_to_f64(y)


def test_hand_worked(golden):
    g = golden("conv_dynamic_hand.json")
    d = 128                                  # the smallest supported width: 8 groups
    x = np.zeros((1, 2, d), np.float32); x[0, 0, :4] = g["x_t0"]; x[0, 1, :4] = g["x_t1"]
    prev = np.zeros((1, d), np.float32); prev[0, :4] = g["prev"]
    a0 = np.zeros(d, np.float32); a0[:4] = g["a0"]
    a1 = np.zeros(d, np.float32); a1[:4] = g["a1"]
    G = d // 16
    wc = np.zeros((2 * G, d), np.float32); wc[0, 0] = 0.5; wc[G, 1] = 0.25
    y = _run(_bits(x), _bits(prev), _bits(a0), _bits(a1), _bits(wc))
    np.testing.assert_array_equal(y[0, 0, :4], g["y_t0"])
    np.testing.assert_array_equal(y[0, 1, :4], g["y_t1"])


def test_zero_correction_equals_static_kernel():
    import block_draft_selection_b200 as bds
    w = syn.workload(2)
    x, prev = syn.conv_input(w)
    a0, a1 = syn.conv_taps(w)
    wc = np.zeros((2 * w.d // 16, w.d), np.uint16)
    y = _run(x, prev, a0, a1, wc)
    ys = bds.dflash_conv2tap(dev_bf16(x), dev_bf16(a0), dev_bf16(a1), dev_bf16(prev))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y, bf16_out_to_f64(ys))


@pytest.mark.parametrize("wi", [0, 1, 2, 3, 4])
def test_workloads_within_bound(wi):
    """|y - y_ref| <= 2^-8 |y_ref| + |x| e0 + |x_prev| e1 + 1e-6, where e_j is
    the a priori fp32 bound of the correction GEMM (and the 1e-2 relative
    tolerance of the static conv wherever that is looser)."""
    w = syn.workload(wi)
    x, prev = syn.conv_input(w)
    a0, a1 = syn.conv_taps(w)
    wc = syn.conv_correction(w)
    y = _run(x, prev, a0, a1, wc)
    ref = oracle.conv2tap_dynamic(x, prev, a0, a1, wc)
    G = w.d // 16
    xr = x.reshape(w.B * w.P, w.d)
    e = logits_bound(xr, wc).reshape(w.B, w.P, 2 * G)     # per (b, t, tap-group)
    e0 = np.repeat(e[:, :, :G], 16, axis=2)
    e1 = np.repeat(e[:, :, G:], 16, axis=2)
    xf = np.abs(syn.bf16_bits_to_f32(x).astype(np.float64))
    xp = np.concatenate([np.abs(syn.bf16_bits_to_f32(prev).astype(np.float64))[:, None, :], xf[:, :-1, :]], axis=1)
    bound = np.maximum(1e-2 * np.abs(ref), (2.0 ** -8 + 2.0 ** -22) * np.abs(ref) + xf * e0 + xp * e1) + 1e-6
    err = np.abs(y - ref)
    assert (err <= bound).all(), (err - bound).max()
