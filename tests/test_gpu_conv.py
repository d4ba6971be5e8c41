"""Two-tap conv on the GPU against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import block_draft_synth as syn
from helpers import dev_bf16, bf16_out_to_f64

pytestmark = pytest.mark.gpu


def _run(x, prev, a0, a1):
    import block_draft_selection_b200 as bds
    y = bds.dflash_conv2tap(dev_bf16(x), dev_bf16(a0), dev_bf16(a1),
                            None if prev is None else dev_bf16(prev))
    torch.cuda.synchronize()
    return bf16_out_to_f64(y)


def _bits(a):
    return syn.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def test_hand_worked_bit_exact(golden):
    g = golden("conv_hand.json")
    # d must be a multiple of 8: embed the 2 hand channels in 8 (others zero)
    x = np.zeros((2, 3, 8), np.float32); x[:, :, :2] = g["x"]
    prev = np.zeros((2, 8), np.float32); prev[:, :2] = g["prev"]
    a0 = np.zeros(8, np.float32); a0[:2] = g["a0"]
    a1 = np.zeros(8, np.float32); a1[:2] = g["a1"]
    y = _run(_bits(x), _bits(prev), _bits(a0), _bits(a1))
    np.testing.assert_array_equal(y[:, :, :2], np.asarray(g["y"]))
    y0 = _run(_bits(x), None, _bits(a0), _bits(a1))
    np.testing.assert_array_equal(y0[:, 0, :2], np.asarray(g["y_row0_without_prev"]))


@pytest.mark.parametrize("B,P,d", [(3, 5, 16), (2, 1, 8), (5, 17, 24), (1, 8, 2560)])
def test_identity_and_shift_bit_exact(B, P, d):
    x = (1 + np.arange(B)[:, None, None] * P + np.arange(P)[None, :, None]
         + (np.arange(d) % 5)[None, None, :]).astype(np.float32)
    prev = -(1 + np.arange(B)[:, None] + np.zeros(d)[None, :]).astype(np.float32)
    xb, pb = _bits(x), _bits(prev)
    y = _run(xb, pb, _bits(np.ones(d)), _bits(np.zeros(d)))
    np.testing.assert_array_equal(y, x)
    y = _run(xb, pb, _bits(np.zeros(d)), _bits(np.ones(d)))
    np.testing.assert_array_equal(y[:, 0], prev)
    np.testing.assert_array_equal(y[:, 1:], x[:, :-1])


@pytest.mark.parametrize("wi", [0, 1, 2, 3, 4])
def test_workloads_within_tolerance(wi):
    """|y - y_ref| <= 1e-2 |y_ref| + 1e-6 on every element, at the full conv
    shape of each workload; the same launch the benchmark times."""
    w = syn.workload(wi)
    x, prev = syn.conv_input(w)
    a0, a1 = syn.conv_taps(w)
    y = _run(x, prev, a0, a1)
    ref = oracle.conv2tap(x, prev, a0, a1)
    err = np.abs(y - ref)
    assert (err <= 1e-2 * np.abs(ref) + 1e-6).all(), err.max()
    # output is the exact value rounded to fp32 then to bf16: within half a bf16
    # ulp (2^-8 of |y|) plus the fp32 step (2^-24 of |y|)
    assert (err <= (2.0 ** -8 + 2.0 ** -23) * np.abs(ref)).all()


def test_without_prev():
    w = syn.workload(0)
    x, _ = syn.conv_input(w)
    a0, a1 = syn.conv_taps(w)
    y = _run(x, None, a0, a1)
    ref = oracle.conv2tap(x, None, a0, a1)
    assert (np.abs(y - ref) <= 1e-2 * np.abs(ref) + 1e-6).all()
