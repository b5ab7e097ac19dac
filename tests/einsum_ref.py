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


def ancestor_path(parents, i):
    """Root-to-node list of the nodes on node i's path (parents: list, -1 = root)."""
    path = []
    while i != -1:
        path.append(i)
        i = parents[i]
    return path[::-1]


def ddtree_dual(state, x, A, B, C, dt, dt_bias, D, G, softplus, parents):
    """Tree verify in closed form, without any per-path state: for node i with path
    j_0..j_k = i, unrolling the recurrence gives
        s_i = W_i0 * s0 + sum_m W_im * B_jm * dt_jm * x_jm,  W_im = prod_{l>m} dA_jl,
    with W_i0 the product over the whole path, and out_i = C_i . s_i + D * x_i.
    state [b,H,Dm,N]; x [b,T,H,Dm]; B/C [b,T,G,N]; dt [b,T,H]; parents [b,T] (lists)."""
    b, T, H, Dm = x.shape
    grp = np.arange(H) // (H // G)
    v = dt + (dt_bias[None, None, :] if dt_bias is not None else 0.0)
    dte = np.logaddexp(0.0, v) if softplus else v
    logdA = A[None, None, :] * dte                       # [b,T,H]
    Bh, Ch = B[:, :, grp, :], C[:, :, grp, :]            # [b,T,H,N]
    out = np.zeros(x.shape)
    for r in range(b):
        for i in range(T):
            path = ancestor_path(parents[r], i)
            total = sum(logdA[r, j] for j in path)       # [H]
            a = np.einsum("hdn,hn->hd", state[r], Ch[r, i])
            y = np.exp(total)[:, None] * a
            after = np.zeros(H)                          # log of prod_{l>m} dA_jl
            for j in reversed(path):
                cb = np.einsum("hn,hn->h", Ch[r, i], Bh[r, j])
                y = y + (np.exp(after) * dte[r, j] * cb)[:, None] * x[r, j]
                after = after + logdA[r, j]
            if D is not None:
                y = y + D[:, None] * x[r, i]
            out[r, i] = y
    return out


def causal_conv_step(state, xbc, w, bias, silu):
    """One causal conv1d step per channel: window = (state taps oldest first, new input).
    state [b, C, W-1], xbc [b, C], w [C, W], bias [C] or None (float64 numpy). Returns
    (conv output [b, C], shifted state [b, C, W-1])."""
    win = np.concatenate([state, xbc[:, :, None]], axis=2)
    v = np.einsum("bck,ck->bc", win, w)
    if bias is not None:
        v = v + bias[None, :]
    if silu:
        v = v / (1.0 + np.exp(-v))
    return v, win[:, :, 1:]


def gdn_dense(S, q, k, v, a, b, A_log, dt_bias, scale, l2norm, HK):
    """Gated delta-rule decode, vectorised over heads and rows (float64 numpy).
    S [bt, HV, V, K]; q, k [bt, HK, K]; v [bt, HV, V]; a, b [bt, HV]. Returns (S', out)."""
    HV = v.shape[1]
    hk = np.arange(HV) // (HV // HK)
    qh, kh = q[:, hk, :], k[:, hk, :]
    if l2norm:
        qh = qh / np.sqrt((qh * qh).sum(-1, keepdims=True) + 1e-6)
        kh = kh / np.sqrt((kh * kh).sum(-1, keepdims=True) + 1e-6)
    qh = qh * scale
    e = a + (dt_bias[None, :] if dt_bias is not None else 0.0)
    g = -np.exp(A_log)[None, :] * np.logaddexp(0.0, e)
    alpha = np.exp(g)
    beta = 1.0 / (1.0 + np.exp(-b))
    Sd = S * alpha[:, :, None, None]
    u = np.einsum("bhvk,bhk->bhv", Sd, kh)
    d = beta[:, :, None] * (v - u)
    Sn = Sd + np.einsum("bhv,bhk->bhvk", d, kh)
    out = np.einsum("bhvk,bhk->bhv", Sn, qh)
    return Sn, out
