"""fp64 CPU oracle of the Hymba hybrid-head layer, prefill and decode.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
CPU-baseline leg of the benchmark may import this module.  The CUDA library
never calls it and shares no code with it.

Source: "Hymba: A Hybrid-head Architecture for Small Language Models"
(arXiv 2411.13676), §2.1 Eq. (1)-(3), §2.2, §2.3 Eq. (4), Appendix E Table 11;
and the authors' OpenReview replies (page "Hymba: A Hybrid-head Architecture
for Small Language Models" on paperhub.cn): the A-shape mask and KV-sharing
groups (reply Q1, "Cache Optimization" / "Meta Tokens") and the 1/sqrt(d)
score scale (reply Q2, "Scaling factor in Equation 1").

Everything is computed per sequence, straight from the definitions, in fp64:
dense masked softmax attention per head, a time-step loop for the selective
scan, explicit tap sums for the convolution.  numpy's matmul is the only
library primitive.  No tiling, online softmax or chunked scan.

Readings taken where the pages are silent (each is listed with its reason in
the design notes of this repository):
  * value head width d_v = d_inner / n_heads, Q/K head width as configured;
  * mask: key j visible from query i iff j <= i and (global or j < m or i - j < W);
  * score scale 1/sqrt(d_qk);
  * GQA: query head h reads KV head floor(h / (H / Hkv));
  * SSM branch = Mamba-1: causal depthwise conv (kernel K, bias, zero history)
    and SiLU, then [delta_r, B, C] = u W_x^T, delta = softplus(delta_r W_dt^T + b_dt),
    A = -exp(A_log), y = C.h + D u, gated by SiLU(z);
  * norm = RMS over all d_inner channels with no weight, eps as configured;
  * Eq. (3)'s two branches are averaged (divided by 2) as the text says;
  * no biases in the in/x/out projections;
  * rotary position embedding of Q and K (§2.5 changes "the ROPE base" for the 8k
    extension; base not given): off unless a base is configured; when on, the rotation
    of the original rotary-embedding definition, each consecutive pair (2i, 2i+1) of a
    head turned by the angle p * base^(-2i/d_qk) at X~ position p (meta rows included).
The pages print no value that checks the readings of the conv, the low-rank
delta, the SiLU gate, the RMS form of "norm" and D; the functions themselves are
pinned by the tests through special cases with closed forms or library routines
(the conv against numpy.convolve; D and the gate with the C rows at zero; delta
with W_dt = 0 and with a full-rank identity; the norm against its closed form).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Spec:
    """Layer shape and attention layout."""
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim_qk: int
    head_dim_v: int
    d_inner: int
    d_state: int
    d_conv: int
    dt_rank: int
    n_meta: int
    window: int          # ignored when is_global
    is_global: bool
    eps: float = 1e-6
    scale: float = 0.0   # 0 -> 1/sqrt(head_dim_qk)
    rope_base: float = 0.0  # 0 -> no rotary position embedding

    @property
    def score_scale(self) -> float:
        return self.scale if self.scale > 0 else 1.0 / np.sqrt(self.head_dim_qk)


# ---------------------------------------------------------------------------
# Mask (OpenReview reply Q1 "A-shape" pattern; Hymba §2.4 Fig. 6; §2.2 global
# attention in the first, middle and last layers)
# ---------------------------------------------------------------------------

def allowed(i: int, j: int, n_meta: int, window: int, is_global: bool) -> bool:
    """Key position j is visible from query position i (positions index X~)."""
    if j > i:
        return False
    if is_global:
        return True
    return j < n_meta or (i - j) < window


def mask_matrix(L: int, n_meta: int, window: int, is_global: bool) -> np.ndarray:
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    causal = j <= i
    if is_global:
        return causal
    return causal & ((j < n_meta) | ((i - j) < window))


def mask_bitmap(L: int, n_meta: int, window: int, is_global: bool) -> np.ndarray:
    """Row-major bitmap [L, ceil(L/32)] uint32; bit (j % 32) of word j // 32 is allowed(i, j)."""
    m = mask_matrix(L, n_meta, window, is_global)
    words = (L + 31) // 32
    pad = np.zeros((L, words * 32), dtype=bool)
    pad[:, :L] = m
    bits = pad.reshape(L, words, 32).astype(np.uint64)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (bits * weights).sum(axis=2).astype(np.uint32)


# ---------------------------------------------------------------------------
# Elementwise functions
# ---------------------------------------------------------------------------

def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


def rms_normalise(x: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis (the 'norm' of Eq. 3)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


# ---------------------------------------------------------------------------
# Input projection (Hymba §2.1: W_in_proj = [W^Q, W^K, W^V, W^SSM, W^G])
# ---------------------------------------------------------------------------

def in_proj(xt: np.ndarray, w_in: np.ndarray, s: Spec, consumer: bool):
    """Returns q [L, H*dqk], k [L, Hkv*dqk] or None, v [L, Hkv*dv] or None, x_ssm, z [L, E]."""
    p = xt @ w_in.T
    nq = s.n_heads * s.head_dim_qk
    nk = s.n_kv_heads * s.head_dim_qk
    nv = s.n_kv_heads * s.head_dim_v
    E = s.d_inner
    q = p[:, :nq]
    c = nq
    if consumer:
        k = v = None
    else:
        k = p[:, c:c + nk]
        v = p[:, c + nk:c + nk + nv]
        c += nk + nv
    xs = p[:, c:c + E]
    z = p[:, c + E:c + 2 * E]
    assert p.shape[1] == c + 2 * E
    return q, k, v, xs, z


# ---------------------------------------------------------------------------
# Rotary position embedding of Q and K (Hymba §2.5 / §3: a RoPE base changed for the
# 8k-context extension)
# ---------------------------------------------------------------------------

def rope(x: np.ndarray, positions: np.ndarray, head_dim: int, base: float) -> np.ndarray:
    """x [rows, n_heads*head_dim] at X~ positions [rows]: in every head, pair (2i, 2i+1)
    rotated by the angle pos * base^(-2i/head_dim)."""
    rows = x.shape[0]
    xh = x.reshape(rows, -1, head_dim // 2, 2)
    i = np.arange(head_dim // 2)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * base ** (-2.0 * i / head_dim)[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    out = np.empty_like(xh)
    out[..., 0] = xh[..., 0] * c - xh[..., 1] * s
    out[..., 1] = xh[..., 0] * s + xh[..., 1] * c
    return out.reshape(rows, -1)


# ---------------------------------------------------------------------------
# Attention heads (Hymba §2.1 Eq. 1 with the 1/sqrt(d) scale of reply Q2)
# ---------------------------------------------------------------------------

def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, s: Spec, row0: int = 0) -> np.ndarray:
    """softmax(Q K^T * scale + mask) V per query head; q rows are positions row0.. of X~,
    k/v rows are positions 0.. .  Returns [rows, H * dv]."""
    Lq = q.shape[0]
    Lk = k.shape[0]
    H, G = s.n_heads, s.n_kv_heads
    dq, dv = s.head_dim_qk, s.head_dim_v
    i = np.arange(row0, row0 + Lq)[:, None]
    j = np.arange(Lk)[None, :]
    causal = j <= i
    mask = causal if s.is_global else causal & ((j < s.n_meta) | ((i - j) < s.window))
    out = np.empty((Lq, H * dv))
    for h in range(H):
        g = h // (H // G)
        qh = q[:, h * dq:(h + 1) * dq]
        kg = k[:, g * dq:(g + 1) * dq]
        vg = v[:, g * dv:(g + 1) * dv]
        sc = (qh @ kg.T) * s.score_scale
        sc = np.where(mask, sc, -np.inf)
        sc = sc - sc.max(axis=1, keepdims=True)
        p = np.exp(sc)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h * dv:(h + 1) * dv] = p @ vg
    return out


# ---------------------------------------------------------------------------
# SSM heads (Hymba §2.1 Eq. 2, "we adopt Mamba"; Mamba-1 selective scan)
# ---------------------------------------------------------------------------

def causal_conv_silu(xs: np.ndarray, conv_w: np.ndarray, conv_b: np.ndarray,
                     history: np.ndarray | None = None) -> np.ndarray:
    """u[t, c] = SiLU(b[c] + sum_k w[c, k] * x[t - (K-1) + k, c]); x before the first row is
    `history` ([K-1, E], oldest first) or zero."""
    T, E = xs.shape
    K = conv_w.shape[1]
    hist = np.zeros((K - 1, E)) if history is None else history
    xx = np.concatenate([hist, xs], axis=0)  # row r of xx is x[r - (K-1)]
    acc = np.broadcast_to(conv_b, (T, E)).copy()
    for k in range(K):
        acc += conv_w[:, k][None, :] * xx[k:k + T]
    return silu(acc)


def ssm_inputs(u: np.ndarray, w_x: np.ndarray, w_dt: np.ndarray, b_dt: np.ndarray, s: Spec):
    """[delta_r, B, C] = u W_x^T; delta = softplus(delta_r W_dt^T + b_dt)."""
    R, N = s.dt_rank, s.d_state
    xdbl = u @ w_x.T
    dr = xdbl[:, :R]
    Bm = xdbl[:, R:R + N]
    Cm = xdbl[:, R + N:R + 2 * N]
    delta = softplus(dr @ w_dt.T + b_dt[None, :])
    return delta, Bm, Cm


def selective_scan(u, delta, A, Bm, Cm, D, h0=None):
    """h_t = exp(delta_t A) * h_{t-1} + delta_t B_t u_t (h_{-1} = h0 or 0);
    y_t = C_t . h_t + D u_t.  Shapes: u, delta [T, E]; A [E, N]; B, C [T, N]; D [E].
    Returns y [T, E] and the final state [E, N]."""
    T, E = u.shape
    h = np.zeros_like(A) if h0 is None else h0.copy()
    y = np.empty((T, E))
    for t in range(T):
        h = np.exp(delta[t][:, None] * A) * h + (delta[t] * u[t])[:, None] * Bm[t][None, :]
        y[t] = h @ Cm[t] + D * u[t]
    return y, h


# ---------------------------------------------------------------------------
# Fusion (Hymba §2.1 Eq. 3: norm, per-channel beta, mean, W_out_proj)
# ---------------------------------------------------------------------------

def fuse(o_attn, y_ssm, beta_attn, beta_ssm, eps):
    return (beta_attn * rms_normalise(o_attn, eps) + beta_ssm * rms_normalise(y_ssm, eps)) / 2.0


# ---------------------------------------------------------------------------
# Decode cache slots (§2.2 local attention; §2.3 meta tokens as cache prefix)
# ---------------------------------------------------------------------------

def kv_slot(pos: int, s: Spec) -> int:
    """Slot of position pos in a layer's decode K/V store: meta rows keep their position,
    real rows of a sliding-window layer cycle through W ring slots after the meta rows,
    a global layer keeps every position."""
    if s.is_global or pos < s.n_meta:
        return pos
    return s.n_meta + (pos - s.n_meta) % s.window


def kv_capacity(s: Spec, max_rows: int) -> int:
    return max_rows if s.is_global else s.n_meta + s.window


def decode_slot_bitmap(pos: int, s: Spec, capacity: int) -> np.ndarray:
    """Slots of the decode K/V store that a query at position pos attends to: the slot of
    every position visible from pos.  [ceil(capacity/32)] uint32; bit (k % 32) of word
    k // 32 is slot k."""
    words = np.zeros((capacity + 31) // 32, dtype=np.uint32)
    for j in range(pos + 1):
        if allowed(pos, j, s.n_meta, s.window, s.is_global):
            k = kv_slot(j, s)
            words[k // 32] |= np.uint32(1 << (k % 32))
    return words


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------

def _f64(a):
    return np.asarray(a, dtype=np.float64)


def layer_prefill(xt, w: dict, s: Spec, kv_from: dict | None = None, capacity: int | None = None):
    """One sequence X~ [L, d] through the hybrid-head layer.

    w: weights (w_in, conv_w, conv_b, w_x, w_dt, b_dt, a_log, d_skip, beta_attn, beta_ssm, w_out).
    kv_from: for a KV-sharing consumer, the producer's result dict (its 'k' and 'v' are used).
    capacity: slots of the decode K/V store to emit (default m+W, or L for a global layer).
    Returns a dict with every stage's value, the final SSM and conv state and the cache."""
    xt = _f64(xt)
    L = xt.shape[0]
    consumer = kv_from is not None
    q, k, v, xs, z = in_proj(xt, _f64(w["w_in"]), s, consumer)
    if s.rope_base > 0:
        q = rope(q, np.arange(L), s.head_dim_qk, s.rope_base)
        if not consumer:
            k = rope(k, np.arange(L), s.head_dim_qk, s.rope_base)
    if consumer:
        k, v = kv_from["k"], kv_from["v"]
    o = attention(q, k, v, s)
    u = causal_conv_silu(xs, _f64(w["conv_w"]), _f64(w["conv_b"]))
    delta, Bm, Cm = ssm_inputs(u, _f64(w["w_x"]), _f64(w["w_dt"]), _f64(w["b_dt"]), s)
    A = -np.exp(_f64(w["a_log"]))
    y, hL = selective_scan(u, delta, A, Bm, Cm, _f64(w["d_skip"]))
    y_ssm = y * silu(z)
    f = fuse(o, y_ssm, _f64(w["beta_attn"]), _f64(w["beta_ssm"]), s.eps)
    Y = f @ _f64(w["w_out"]).T
    K1 = s.d_conv - 1
    conv_state = np.zeros((K1, s.d_inner))
    take = min(K1, L)
    if take:
        conv_state[K1 - take:] = xs[L - take:]
    res = dict(q=q, k=k, v=v, x_ssm=xs, z=z, o=o, u=u, delta=delta, B=Bm, C=Cm, y=y,
               y_ssm=y_ssm, f=f, Y=Y, h=hL, conv=conv_state)
    if not consumer:
        cap = capacity if capacity is not None else kv_capacity(s, L)
        kc = np.zeros((s.n_kv_heads, cap, s.head_dim_qk))
        vc = np.zeros((s.n_kv_heads, cap, s.head_dim_v))
        for j in range(L):
            if not s.is_global and j >= s.n_meta and (L - 1 - j) >= s.window:
                continue  # fell out of the window of every later query
            sl = kv_slot(j, s)
            kc[:, sl] = k[j].reshape(s.n_kv_heads, s.head_dim_qk)
            vc[:, sl] = v[j].reshape(s.n_kv_heads, s.head_dim_v)
        res["k_cache"], res["v_cache"] = kc, vc
    return res


def layer_decode(x_t, pos: int, w: dict, s: Spec, cache: dict, kv_cache: dict | None = None):
    """One new token at X~ position `pos` for one sequence.

    cache: this layer's {'ssm': [E, N], 'conv': [K-1, E]} and, for a layer that owns its K/V,
    {'k': [Hkv, cap, dqk], 'v': [Hkv, cap, dv]} holding positions < pos at kv_slot().
    kv_cache: for a KV-sharing consumer, the producer's store after the producer's own
    decode of this position.  Returns (y_t [d], new cache dict)."""
    x_t = _f64(x_t)[None, :]
    consumer = kv_cache is not None
    q, k, v, xs, z = in_proj(x_t, _f64(w["w_in"]), s, consumer)
    if s.rope_base > 0:
        q = rope(q, np.array([pos]), s.head_dim_qk, s.rope_base)
        if not consumer:
            k = rope(k, np.array([pos]), s.head_dim_qk, s.rope_base)
    new = {key: _f64(val).copy() for key, val in cache.items()}
    if consumer:
        kc, vc = _f64(kv_cache["k"]), _f64(kv_cache["v"])
    else:
        sl = kv_slot(pos, s)
        new["k"][:, sl] = k[0].reshape(s.n_kv_heads, s.head_dim_qk)
        new["v"][:, sl] = v[0].reshape(s.n_kv_heads, s.head_dim_v)
        kc, vc = new["k"], new["v"]
    # Gather the visible positions from their slots, in position order.
    vis = [j for j in range(pos + 1) if allowed(pos, j, s.n_meta, s.window, s.is_global)]
    slots = [kv_slot(j, s) for j in vis]
    kk = np.concatenate([kc[g][slots] for g in range(s.n_kv_heads)], axis=1)  # [nvis, Hkv*dqk]
    vv = np.concatenate([vc[g][slots] for g in range(s.n_kv_heads)], axis=1)
    # attention() masks by position; give it the gathered rows at their own positions.
    H, G, dq, dv = s.n_heads, s.n_kv_heads, s.head_dim_qk, s.head_dim_v
    o = np.empty((1, H * dv))
    for h in range(H):
        g = h // (H // G)
        sc = (kk[:, g * dq:(g + 1) * dq] @ q[0, h * dq:(h + 1) * dq]) * s.score_scale
        sc = sc - sc.max()
        p = np.exp(sc)
        p = p / p.sum()
        o[0, h * dv:(h + 1) * dv] = p @ vv[:, g * dv:(g + 1) * dv]
    hist = new["conv"]
    u = causal_conv_silu(xs, _f64(w["conv_w"]), _f64(w["conv_b"]), history=hist)
    new["conv"] = np.concatenate([hist[1:], xs], axis=0)
    delta, Bm, Cm = ssm_inputs(u, _f64(w["w_x"]), _f64(w["w_dt"]), _f64(w["b_dt"]), s)
    A = -np.exp(_f64(w["a_log"]))
    y, h1 = selective_scan(u, delta, A, Bm, Cm, _f64(w["d_skip"]), h0=new["ssm"])
    new["ssm"] = h1
    y_ssm = y * silu(z)
    f = fuse(o, y_ssm, _f64(w["beta_attn"]), _f64(w["beta_ssm"]), s.eps)
    Y = f @ _f64(w["w_out"]).T
    return Y[0], new


# ---------------------------------------------------------------------------
# The Hymba block and a stack of blocks (Hymba Fig. 4 (b) and Appendix E Table 11:
# the hybrid-head module and an MLP, each behind a norm and inside a residual)
# ---------------------------------------------------------------------------
# Readings (the pages give Fig. 4's caption and the MLP width only): pre-norm, an RMS norm
# with a learnable weight before the mixer and before the MLP; a residual around each; the
# MLP gated by SiLU, down(SiLU(x W_gate^T) * (x W_up^T)), the form whose parameter count,
# with the module of this layer and a tied embedding of a 32K vocabulary, gives the
# printed 1.52B of Table 11 (an ungated MLP gives 1.2B).

def rms_norm(x: np.ndarray, weight: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * weight over the last axis."""
    return rms_normalise(x, eps) * weight


def mlp(x: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    return (silu(x @ w_gate.T) * (x @ w_up.T)) @ w_down.T


def block_prefill(xt, w: dict, s: Spec, kv_from: dict | None = None, capacity: int | None = None):
    """One block over one sequence X~ [L, d] (the residual stream): h = x + M(norm1(x)),
    out = h + MLP(norm2(h)).  w: the layer's weights plus norm1, norm2 [d], w_gate, w_up
    [F, d], w_down [d, F].  Returns (out, the mixer's result dict)."""
    xt = _f64(xt)
    mix = layer_prefill(rms_norm(xt, _f64(w["norm1"]), s.eps), w, s, kv_from=kv_from, capacity=capacity)
    h = xt + mix["Y"]
    out = h + mlp(rms_norm(h, _f64(w["norm2"]), s.eps), _f64(w["w_gate"]), _f64(w["w_up"]), _f64(w["w_down"]))
    return out, mix


def block_decode(x_t, pos: int, w: dict, s: Spec, cache: dict, kv_cache: dict | None = None):
    """The block for one new row: (out [d], the mixer's new cache)."""
    x_t = _f64(x_t)
    y, new = layer_decode(rms_norm(x_t, _f64(w["norm1"]), s.eps), pos, w, s, cache, kv_cache=kv_cache)
    h = x_t + y
    out = h + mlp(rms_norm(h[None, :], _f64(w["norm2"]), s.eps), _f64(w["w_gate"]), _f64(w["w_up"]),
                  _f64(w["w_down"]))[0]
    return out, new


def stack_prefill(xt, weights: list, specs: list, producers: list):
    """A stack of blocks over one sequence X~ [L, d]: block l reads block l-1's output;
    producers[l] is None for a block that owns its K/V, else the index of the block whose
    K/V it shares.  Returns the last output and every block's mixer result."""
    x = _f64(xt)
    mixes = []
    for w, s, p in zip(weights, specs, producers):
        x, mix = block_prefill(x, w, s, kv_from=None if p is None else mixes[p])
        mixes.append(mix)
    return x, mixes
