"""Error bounds of the compared stages that cancel.

Several stages of the layer are sums whose terms cancel: B and C sum 3200 products of
x_proj, the state h sums the decayed inputs delta*B*u, y = C.h + D u, the conv sums four
taps and a bias, and the attention output averages values of both signs.  A stage value
near zero then carries an error set by the size of its terms, not by its own size, and a
bound of the form a + r|o| (or one scaled by the stage's rms) either misses large errors
in small elements or fails on correct code.  Such a stage is checked twice:

  * elementwise, every element, no exceptions: |g - o| <= 2e-2 (the bf16 path's relative
    tolerance) times the stage's first-order error *magnitude*, the classical forward
    error bound: every input of the stage perturbed by a relative amount of its own
    magnitude, propagated with the oracle's own functions (plus a floor of a thousandth
    of the stage's rms, below which an element is noise of the fp32 sums making it);
  * as a whole: relative L2 error <= 1e-2, which is tight (bf16 storage rounding alone
    gives 0.1-0.5 %), so a mistake spread over many elements shows even where the
    worst-case elementwise bound is wide.

The magnitudes:
    x_ssm, z, q, k, v : |X~| |W_in|^T
    conv (pre-SiLU)   : |b| + sum_k |w_k| |x_{t-k}|,   u: |u| + 1.1 * that (|SiLU'| <= 1.1)
    B, C, delta_r     : |u| |W_x|^T
    delta             : |delta| + sigmoid(raw) |delta_r|_mag |W_dt|^T   (softplus' = sigmoid)
    h, y              : the recurrence's first-order error magnitude (_scan_magnitude):
                        perturbed inputs delta_mag B_mag u_mag, and the decays' own
                        sensitivity to delta, |A| delta_mag |h|
    y_ssm             : y_mag |SiLU(z)| + 1.1 |y| |z|
    o (attention)     : the attention of (q, k, |v|)  (the weights P are positive)
    f                 : (|beta_1| o_mag / rms(o) + |beta_2| y_ssm_mag / rms(y_ssm)) / 2

The bounds are computed from the oracle's fp64 values only; no CUDA-path value enters
them.  Test infrastructure."""
from __future__ import annotations

import numpy as np

from oracle import hymba_oracle as O

REL = 2e-2


def _conv_mag(xs_mag: np.ndarray, conv_w: np.ndarray, conv_b: np.ndarray,
              history: np.ndarray | None = None) -> np.ndarray:
    T, E = xs_mag.shape
    K = conv_w.shape[1]
    hist = np.zeros((K - 1, E)) if history is None else np.abs(history)
    xx = np.concatenate([hist, xs_mag], axis=0)
    acc = np.broadcast_to(np.abs(conv_b), (T, E)).copy()
    for k in range(K):
        acc += np.abs(conv_w[:, k])[None, :] * xx[k:k + T]
    return acc


def _scan_magnitude(u, u_mag, delta, delta_mag, A, Bm, B_mag, Cm, C_mag, D, h0=None, h0_mag=None):
    """First-order error magnitude of the recurrence h_t = exp(delta_t A) h_{t-1} + delta_t B_t u_t,
    y_t = C_t . h_t + D u_t when every input carries a relative perturbation of its magnitude:
      H_t = d_t H_{t-1} + d_t |A| delta_mag_t |h_{t-1}| + delta_mag_t B_mag_t u_mag_t
      Y_t = sum_n (C_mag_t |h_t| + |C_t| H_t) + |D| u_mag_t
    (d_t = exp(delta_t A); the middle term is the decay's sensitivity to delta).  The initial
    state h0 carries the error magnitude h0_mag (zero when omitted).  Returns (Y, H_final)."""
    T, E = u.shape
    h = np.zeros_like(A) if h0 is None else np.asarray(h0, np.float64).copy()
    H = np.zeros_like(A) if h0_mag is None else np.asarray(h0_mag, np.float64).copy()
    absA, absD = np.abs(A), np.abs(D)
    Y = np.empty((T, E))
    for t in range(T):
        d = np.exp(delta[t][:, None] * A)
        H = d * H + d * absA * delta_mag[t][:, None] * np.abs(h) + (delta_mag[t] * u_mag[t])[:, None] * B_mag[t][None, :]
        h = d * h + (delta[t] * u[t])[:, None] * Bm[t][None, :]
        Y[t] = np.abs(h) @ C_mag[t] + H @ np.abs(Cm[t]) + absD * u_mag[t]
    return Y, H


def ssm_magnitudes(w: dict, s: O.Spec, ref: dict) -> dict:
    """Magnitude companions of the SSM branch's stages of O.layer_prefill (ref: its result)."""
    um = np.abs(ref["u"]) + 1.1 * _conv_mag(np.abs(ref["x_ssm"]), w["conv_w"], w["conv_b"])
    R, N = s.dt_rank, s.d_state
    ua = np.abs(ref["u"])
    xdm = ua @ np.abs(np.asarray(w["w_x"], np.float64)).T
    Bm, Cm = xdm[:, R:R + N], xdm[:, R + N:R + 2 * N]
    w_dt = np.asarray(w["w_dt"], np.float64)
    raw = (ref["u"] @ np.asarray(w["w_x"], np.float64)[:R].T) @ w_dt.T + np.asarray(w["b_dt"], np.float64)
    dm = np.abs(ref["delta"]) + (1.0 / (1.0 + np.exp(-raw))) * (xdm[:, :R] @ np.abs(w_dt).T)
    A = -np.exp(np.asarray(w["a_log"], np.float64))
    ym, hm = _scan_magnitude(ref["u"], um, ref["delta"], dm, A, ref["B"], Bm, ref["C"], Cm,
                             np.asarray(w["d_skip"], np.float64))
    ysm = ym * np.abs(O.silu(ref["z"])) + 1.1 * np.abs(ref["y"]) * np.abs(ref["z"])
    return dict(u=um, B=Bm, C=Cm, delta=dm, h=hm, y=ym, y_ssm=ysm)


def prefill_magnitudes(xt, w: dict, s: O.Spec, ref: dict, kv_from: dict | None = None) -> dict:
    """Magnitude companion of each stage of O.layer_prefill (ref is its result)."""
    xt = np.asarray(xt, dtype=np.float64)
    consumer = kv_from is not None
    qm, km, vm, xsm, zm = O.in_proj(np.abs(xt), np.abs(np.asarray(w["w_in"], np.float64)), s, consumer)
    if consumer:
        km, vm = np.abs(kv_from["k"]), np.abs(kv_from["v"])
    k = kv_from["k"] if consumer else ref["k"]
    v = kv_from["v"] if consumer else ref["v"]
    om = O.attention(ref["q"], k, np.abs(v), s)
    out = ssm_magnitudes(w, s, ref)
    rms = lambda a: np.sqrt(np.mean(a * a, axis=-1, keepdims=True) + s.eps)  # noqa: E731
    fm = (np.abs(w["beta_attn"]) * om / rms(ref["o"]) +
          np.abs(w["beta_ssm"]) * out["y_ssm"] / rms(ref["y_ssm"])) / 2
    out.update(q=qm, k=km, v=vm, x_ssm=xsm, z=zm, o=om, f=fm)
    return out


def decode_state_magnitude(x_t, pos: int, w: dict, s: O.Spec, cache: dict, consumer: bool = False,
                           h0_mag=None) -> np.ndarray:
    """Error magnitude of the SSM state after one decode step.  h0_mag: the error magnitude
    of the state the step starts from when that state was itself computed (a prefill's
    final state); None when both sides start from the same stored state."""
    q, k, v, xs, z = O.in_proj(np.asarray(x_t, np.float64)[None, :], np.asarray(w["w_in"], np.float64), s,
                               consumer)
    u = O.causal_conv_silu(xs, w["conv_w"], w["conv_b"], history=cache["conv"])
    um = np.abs(u) + 1.1 * _conv_mag(np.abs(xs), w["conv_w"], w["conv_b"], history=cache["conv"])
    delta, Bv, Cv = O.ssm_inputs(u, w["w_x"], w["w_dt"], w["b_dt"], s)
    R, N = s.dt_rank, s.d_state
    xdm = np.abs(u) @ np.abs(np.asarray(w["w_x"], np.float64)).T
    w_dt = np.asarray(w["w_dt"], np.float64)
    raw = (u @ np.asarray(w["w_x"], np.float64)[:R].T) @ w_dt.T + np.asarray(w["b_dt"], np.float64)
    dm = np.abs(delta) + (1.0 / (1.0 + np.exp(-raw))) * (xdm[:, :R] @ np.abs(w_dt).T)
    A = -np.exp(np.asarray(w["a_log"], np.float64))
    _, hm = _scan_magnitude(u, um, delta, dm, A, Bv, xdm[:, R:R + N], Cv, xdm[:, R + N:],
                            np.asarray(w["d_skip"], np.float64), h0=cache["ssm"], h0_mag=h0_mag)
    return hm


# Elements below a thousandth of their stage's rms are resolved down to that level only
# (their size is then noise of the fp32 sums that produce them); the relative L2 check
# covers the stage as a whole.
FLOOR = 1e-3


def bound_of(o, mag) -> np.ndarray:
    """The elementwise bound 2e-2 x (magnitude + 1e-3 x rms of the stage)."""
    o = np.asarray(o, dtype=np.float64)
    return REL * (np.asarray(mag, dtype=np.float64) + FLOOR * float(np.sqrt(np.mean(o * o)))) + 1e-300


def close_mag(g, o, mag, what=""):
    """|g - o| <= 2e-2 (magnitude + 1e-3 rms(o)), elementwise, every element."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    err = np.abs(g - o)
    bound = bound_of(o, mag)
    ratio = err / bound
    if (ratio > 1).any():
        idx = np.unravel_index(np.argmax(ratio), ratio.shape)
        raise AssertionError(f"{what}: {(ratio > 1).sum()} of {ratio.size} elements outside 2e-2 x magnitude; "
                             f"worst {ratio.max():.2f}x at {idx} (gpu {g[idx]:.5g}, oracle {o[idx]:.5g}, "
                             f"magnitude {mag[idx]:.3g})")
    return float(ratio.max())
