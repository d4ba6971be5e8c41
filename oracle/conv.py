"""Two-tap block-local convolution, float64.

"DFlash 2: Keep Drafting Parallel", section "a lightweight local convolution",
formula Conv_k(x)_t = k_{t,0} (.) x_t + k_{t,1} (.) x_{t-1}: one depthwise tap
on the current position and one on the previous; the first position reads the
representation of the last verified token (also Figure 4's caption).  The
static base taps a0, a1 [d] stand for k_{t,0}, k_{t,1}; the content-dependent
correction the section mentions is not part of this function.
"""
import numpy as np

from ._widen import bf16


def conv2tap(x_bits, prev_bits, a0_bits, a1_bits) -> np.ndarray:
    """y[b,t,c] = a0[c]*x[b,t,c] + a1[c]*x[b,t-1,c], with x[b,-1,:] = prev[b,:]
    (zeros when prev_bits is None).  x [B,P,d] bf16 bits -> y [B,P,d] float64."""
    x = bf16(x_bits)
    B, P, d = x.shape
    a0 = bf16(a0_bits).reshape(d)
    a1 = bf16(a1_bits).reshape(d)
    prev = np.zeros((B, d)) if prev_bits is None else bf16(prev_bits).reshape(B, d)
    y = np.empty_like(x)
    for t in range(P):
        before = prev if t == 0 else x[:, t - 1, :]
        y[:, t, :] = a0 * x[:, t, :] + a1 * before
    return y


def conv2tap_dynamic(x_bits, prev_bits, a0_bits, a1_bits, wc_bits) -> np.ndarray:
    """Two-tap conv whose taps get a content-dependent correction.

    "DFlash 2: Keep Drafting Parallel", section "a lightweight local
    convolution": each coefficient is a learnable base kernel plus a small
    correction computed from the current hidden state, one correction shared
    by every 16 channels.  Reading taken here: the correction of tap j at
    position t for channel group g (channels 16g .. 16g+15) is the linear map
        delta_j[b,t,g] = sum_c x[b,t,c] * Wc[j*G + g, c],   G = d / 16,
    of the conv input at that position, and
        y[b,t,c] = (a0[c] + delta_0[b,t,c//16]) * x[b,t,c]
                 + (a1[c] + delta_1[b,t,c//16]) * x[b,t-1,c],
    with x[b,-1,:] = prev[b,:] (zeros when prev_bits is None).
    Wc [2G, d] bf16 bits.  Returns y [B,P,d] float64."""
    x = bf16(x_bits)
    B, P, d = x.shape
    G = d // 16
    a0 = bf16(a0_bits).reshape(d)
    a1 = bf16(a1_bits).reshape(d)
    wc = bf16(wc_bits).reshape(2 * G, d)
    prev = np.zeros((B, d)) if prev_bits is None else bf16(prev_bits).reshape(B, d)
    delta = np.einsum("btc,gc->btg", x, wc)          # [B, P, 2G]
    k0 = a0[None, None, :] + np.repeat(delta[:, :, :G], 16, axis=2)
    k1 = a1[None, None, :] + np.repeat(delta[:, :, G:], 16, axis=2)
    y = np.empty_like(x)
    for t in range(P):
        before = prev if t == 0 else x[:, t - 1, :]
        y[:, t, :] = k0[:, t, :] * x[:, t, :] + k1[:, t, :] * before
    return y
