"""fp64 oracle of the layer's front end (test infrastructure only).

The two steps of the Mamba-2 block that come right before the SSD recurrence, as the
"Engineering Hybrid State-Space Models" page lists them (section 3, the block diagram):
a width-4 1-D convolution followed by SiLU, and the step size
Delta = Softplus(Linear(x) + bias); its session state keeps the convolution's last
dConv - 1 inputs per channel (the convState buffer of shape [dConv - 1, dModel]).

Readings where the page is silent: the convolution is depthwise (one width-4 filter per
channel) and causal (output t sees inputs t-3 .. t), with an optional per-channel bias;
its channels are those of x, B and C together (H*P + 2*G*N, in that order), which the
front end splits into the layouts the SSD layer takes; dt_raw is the output of the
linear projection (given), and dt = softplus(dt_raw + dt_bias) with
softplus(z) = log(1 + exp(z)).  Everything here is a plain definition in float64.
"""
import numpy as np

D_CONV = 4


def softplus(z):
    z = np.asarray(z, dtype=np.float64)
    return np.logaddexp(0.0, z)  # log(1 + exp(z)), without overflow


def silu(v):
    v = np.asarray(v, dtype=np.float64)
    return v / (1.0 + np.exp(-v))


def causal_conv(u, w, bias=None, state=None):
    """Depthwise causal convolution of u [b, L, C] with w [C, 4]:
    out[t, c] = sum_k w[c, k] * u[t - 3 + k, c] (+ bias[c]), where inputs before the
    first token come from `state` [b, 3, C] (the three previous inputs, oldest first)
    or are zero.  Returns (out [b, L, C], new_state [b, 3, C]: the last three inputs)."""
    u = np.asarray(u, dtype=np.float64)
    b, L, C = u.shape
    hist = np.zeros((b, D_CONV - 1, C)) if state is None else np.asarray(state, dtype=np.float64)
    full = np.concatenate([hist, u], axis=1)  # [b, 3 + L, C]
    w = np.asarray(w, dtype=np.float64)
    out = np.zeros((b, L, C))
    for k in range(D_CONV):
        out += w[None, None, :, k] * full[:, k:k + L, :]
    if bias is not None:
        out += np.asarray(bias, dtype=np.float64)[None, None, :]
    return out, full[:, -(D_CONV - 1):, :].copy()


def frontend(xbc, conv_w, conv_b, dt_raw, dt_bias, H, P, G, N, state=None):
    """The whole front end: conv + SiLU over the xBC channels, split into
    x [b, L, H, P], B [b, L, G, N], C [b, L, G, N]; dt [b, L, H]; and the new conv state."""
    conv, new_state = causal_conv(xbc, conv_w, conv_b, state)
    act = silu(conv)
    b, L, _ = act.shape
    x = act[:, :, :H * P].reshape(b, L, H, P)
    B = act[:, :, H * P:H * P + G * N].reshape(b, L, G, N)
    C = act[:, :, H * P + G * N:].reshape(b, L, G, N)
    dt = softplus(np.asarray(dt_raw, dtype=np.float64) + np.asarray(dt_bias, dtype=np.float64)[None, None, :])
    return x, B, C, dt, new_state
