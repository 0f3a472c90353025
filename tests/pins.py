"""Independent checks that pin the fp64 oracle to mathematics it does not share.

Nothing here re-types the oracle's loop.  Each helper reaches the same
quantity another way:

* ``fir_conv_silu``: the causal 4-tap conv through numpy's correlate, SiLU
  through scipy's logistic function;
* ``quadratic_form``: the SSD "attention-like" form of the layer
  ("EP6. 트랜스포머 대체 신경망 연구" §8: Mamba-2 proves SSM == structured
  attention), y_t = sum_{s<=t} (C_t . B_s) * prod_{r=s+1..t} a_r * dt_s * x_s
  + C_t . (prod_{r<=t} a_r) h_0 + D x_t, evaluated as a dense masked matrix
  with decays from sums of dt in the exponent rather than running products;
* closed forms and library routines (cumsum, lfilter) in the tests themselves.
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit


def f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.asarray(a, dtype=np.float64)


def silu_lib(v):
    return v * expit(v)


def softplus_lib(v):
    return np.logaddexp(0.0, v)


def fir_conv_silu(seq, hist, w, b):
    """silu(b + sum_k w[k] * seq[t-3+k]) via numpy.correlate on the padded sequence."""
    pad = np.zeros(3) if hist is None else np.asarray(hist, dtype=np.float64)
    full = np.concatenate([pad, np.asarray(seq, dtype=np.float64)])
    return silu_lib(np.correlate(full, np.asarray(w, dtype=np.float64), mode="valid") + b)


def post_conv(inp, b):
    """Post-conv channels of sequence b: (ux [L, H*P], uB [L, G, N], uC [L, G, N])."""
    x, Bm, Cm = f64(inp["x"])[b], f64(inp["B"])[b], f64(inp["C"])[b]
    L, HP = x.shape
    G, N = Bm.shape[1], Bm.shape[2]
    w, cb = f64(inp["conv_w"]), f64(inp["conv_b"])
    ics = f64(inp.get("init_conv_state"))
    raw = np.concatenate([x, Bm.reshape(L, G * N), Cm.reshape(L, G * N)], axis=1)
    u = np.empty_like(raw)
    for c in range(raw.shape[1]):
        u[:, c] = fir_conv_silu(raw[:, c], None if ics is None else ics[b, c], w[c], cb[c])
    return u[:, :HP], u[:, HP:HP + G * N].reshape(L, G, N), u[:, HP + G * N:].reshape(L, G, N)


def quadratic_form(inp):
    """(y [Bt, L, H*P], final_state [Bt, H, P, N]) from the masked quadratic form."""
    x = f64(inp["x"])
    Bt, L, HP = x.shape
    H = f64(inp["A"]).shape[0]
    P = HP // H
    G, N = f64(inp["B"]).shape[2:]
    A, D, dtb = f64(inp["A"]), f64(inp["D"]), f64(inp["dt_bias"])
    dt_all = softplus_lib(f64(inp["dt"]) + dtb[None, None, :])
    z = f64(inp["z"])
    h0_all = f64(inp.get("init_state"))
    y = np.zeros((Bt, L, HP))
    fs = np.zeros((Bt, H, P, N))
    for b in range(Bt):
        ux, uB, uC = post_conv(inp, b)
        for h in range(H):
            g = h // (H // G)
            dt = dt_all[b, :, h]
            seg = np.zeros((L, L))            # seg[t, s] = sum_{r=s+1..t} dt_r (t >= s)
            for t in range(L):
                for s in range(t + 1):
                    seg[t, s] = dt[s + 1:t + 1].sum()
            mask = np.tril(np.ones((L, L), dtype=bool))
            decay = np.where(mask, np.exp(A[h] * np.where(mask, seg, 0.0)), 0.0)
            CB = uC[:, g, :] @ uB[:, g, :].T  # [t, s]
            M = CB * decay * dt[None, :]
            xs = ux[:, h * P:(h + 1) * P]
            yh = M @ xs
            tot = np.array([dt[:t + 1].sum() for t in range(L)])
            h0 = np.zeros((P, N)) if h0_all is None else h0_all[b, h]
            yh += (uC[:, g, :] @ h0.T) * np.exp(A[h] * tot)[:, None]
            yh += D[h] * xs
            y[b, :, h * P:(h + 1) * P] = yh * silu_lib(z[b, :, h * P:(h + 1) * P])
            w_end = np.exp(A[h] * np.array([dt[s + 1:].sum() for s in range(L)])) * dt
            fs[b, h] = (xs * w_end[:, None]).T @ uB[:, g, :] + np.exp(A[h] * dt.sum()) * h0
    return y, fs


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
