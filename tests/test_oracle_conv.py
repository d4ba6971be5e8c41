"""Pins for the oracle's two-tap conv (no GPU)."""
import numpy as np
import oracle
from block_draft_synth import f32_to_bf16_bits


def _bits(a):
    return f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def test_hand_worked(golden):
    g = golden("conv_hand.json")
    y = oracle.conv2tap(_bits(g["x"]), _bits(g["prev"]), _bits(g["a0"]), _bits(g["a1"]))
    np.testing.assert_array_equal(y, np.asarray(g["y"], dtype=np.float64))
    y0 = oracle.conv2tap(_bits(g["x"]), None, _bits(g["a0"]), _bits(g["a1"]))
    np.testing.assert_array_equal(y0[:, 0, :], np.asarray(g["y_row0_without_prev"]))
    np.testing.assert_array_equal(y0[:, 1:, :], np.asarray(g["y"])[:, 1:, :])


def _markers(B, P, d):
    # integer markers, exact in bf16: x[b,t,c] = 1 + b*P + t (+ c % 3), prev[b,c] = -(b+1)
    x = (1 + np.arange(B)[:, None, None] * P + np.arange(P)[None, :, None]
         + (np.arange(d) % 3)[None, None, :]).astype(np.float32)
    prev = -(1 + np.arange(B)[:, None] + 0 * np.arange(d)[None, :]).astype(np.float32)
    return x, prev


def test_identity_taps_reproduce_x():
    B, P, d = 3, 5, 16
    x, prev = _markers(B, P, d)
    y = oracle.conv2tap(_bits(x), _bits(prev), _bits(np.ones(d)), _bits(np.zeros(d)))
    np.testing.assert_array_equal(y, x.astype(np.float64))


def test_shift_taps_read_predecessor_and_prev_only_within_block():
    B, P, d = 3, 5, 16
    x, prev = _markers(B, P, d)
    y = oracle.conv2tap(_bits(x), _bits(prev), _bits(np.zeros(d)), _bits(np.ones(d)))
    np.testing.assert_array_equal(y[:, 0, :], prev)             # first position reads prev
    np.testing.assert_array_equal(y[:, 1:, :], x[:, :-1, :])     # others read t-1, same block
    y0 = oracle.conv2tap(_bits(x), None, _bits(np.zeros(d)), _bits(np.ones(d)))
    np.testing.assert_array_equal(y0[:, 0, :], 0.0)


def test_single_position_block():
    x = np.array([[[2.0, -1.0]]], dtype=np.float32)
    prev = np.array([[4.0, 8.0]], dtype=np.float32)
    y = oracle.conv2tap(_bits(x), _bits(prev), _bits([1.0, 0.5]), _bits([0.25, 0.125]))
    np.testing.assert_array_equal(y, [[[2.0 + 1.0, -0.5 + 1.0]]])

