"""A second, vectorised float64 formulation of the selective state update (tests only).

Written independently of the loop oracle: numpy einsum over whole tensors, softplus as
``logaddexp(0, v)``. It follows the formula of the Selective State Update page
(TensorRT-Edge-LLM C++ API, invokeSelectiveStateUpdate):
    new_state = state * exp(A * dt) + B * dt * x
    out       = sum_n new_state * C + D * x, times silu(z) when z is given.
It takes dense per-row state (no pool, no indices) and is used on tiny shapes only.
"""

import numpy as np


def f64(t):
    return None if t is None else t.double().numpy()


def decode_dense(state, x, A, B, C, dt, dt_bias, D, z, G, softplus):
    """state [b,H,Dm,N], x/z [b,H,Dm], B/C [b,G,N], dt [b,H] (all float64 numpy)."""
    H = x.shape[1]
    grp = np.arange(H) // (H // G)
    v = dt + (dt_bias[None, :] if dt_bias is not None else 0.0)
    dte = np.logaddexp(0.0, v) if softplus else v
    decay = np.exp(A[None, :] * dte)
    Bh, Ch = B[:, grp, :], C[:, grp, :]
    new = state * decay[:, :, None, None] + np.einsum("bhn,bh,bhd->bhdn", Bh, dte, x)
    y = np.einsum("bhdn,bhn->bhd", new, Ch)
    if D is not None:
        y = y + D[None, :, None] * x
    if z is not None:
        y = y * z / (1.0 + np.exp(-z))
    return new, y


def prefill_dense(state, x, A, B, C, dt, dt_bias, D, z, G, softplus, lengths=None):
    """Token-by-token over [b,T,...] inputs; returns (final state, out [b,T,H,Dm]) with
    positions t >= lengths[b] left as NaN and the state frozen after lengths[b]."""
    b, T = x.shape[:2]
    out = np.full(x.shape, np.nan)
    s = state.copy()
    for t in range(T):
        new, y = decode_dense(s, x[:, t], A, B[:, t], C[:, t], dt[:, t], dt_bias, D,
                              None if z is None else z[:, t], G, softplus)
        live = np.ones(b, bool) if lengths is None else (t < lengths)
        s[live] = new[live]
        out[live, t] = y[live]
    return s, out
