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
