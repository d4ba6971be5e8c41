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



def _dyn_hand(golden):
    g = golden("conv_dynamic_hand.json")
    d = 16
    x = np.zeros((1, 2, d), np.float32)
    x[0, 0, :4] = g["x_t0"]
    x[0, 1, :4] = g["x_t1"]
    prev = np.zeros((1, d), np.float32)
    prev[0, :4] = g["prev"]
    a0 = np.zeros(d, np.float32); a0[:4] = g["a0"]
    a1 = np.zeros(d, np.float32); a1[:4] = g["a1"]
    wc = np.zeros((2, d), np.float32)
    wc[0, 0] = 0.5
    wc[1, 1] = 0.25
    return g, x, prev, a0, a1, wc


def test_dynamic_hand_worked(golden):
    g, x, prev, a0, a1, wc = _dyn_hand(golden)
    y = oracle.conv2tap_dynamic(_bits(x), _bits(prev), _bits(a0), _bits(a1), _bits(wc))
    np.testing.assert_array_equal(y[0, 0, :4], g["y_t0"])
    np.testing.assert_array_equal(y[0, 1, :4], g["y_t1"])


def test_dynamic_zero_correction_is_static_conv():
    from block_draft_synth import workload, conv_input, conv_taps
    w = workload(0)
    x, prev = conv_input(w)
    a0, a1 = conv_taps(w)
    wc = np.zeros((2 * w.d // 16, w.d), np.uint16)
    np.testing.assert_array_equal(oracle.conv2tap_dynamic(x, prev, a0, a1, wc),
                                  oracle.conv2tap(x, prev, a0, a1))


def test_dynamic_correction_stays_in_its_group():
    """A correction row for group g changes channels 16g..16g+15 only (catches
    a wrong group index or a missing broadcast)."""
    from block_draft_synth import workload, conv_input, conv_taps
    w = workload(0)
    x, prev = conv_input(w)
    a0, a1 = conv_taps(w)
    G = w.d // 16
    base = oracle.conv2tap(x, prev, a0, a1)
    for j, g in ((0, 3), (1, 7)):
        wc = np.zeros((2 * G, w.d), np.float32)
        wc[j * G + g, :] = 0.01
        y = oracle.conv2tap_dynamic(x, prev, a0, a1, _bits(wc))
        changed = np.abs(y - base).max(axis=(0, 1)) > 0
        assert changed[16 * g:16 * g + 16].all()
        changed[16 * g:16 * g + 16] = False
        assert not changed.any()
