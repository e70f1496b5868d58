"""The layer with the GPU path's bf16 roundings put back in: the oracle's steps, with
every intermediate that the CUDA path stores in bf16 rounded to bf16 at the same place
(Q, K, V, x_ssm, z from the input projection; the attention probabilities P before
P V and the attention output; u after conv + SiLU; delta; the gated SSM output; the
fused branch average; the layer output).  [delta_r, B, C] stay unrounded (the CUDA
path keeps them in fp32).

Test evidence only: it shows that the CUDA path's distance from the fp64 oracle is the
rounding that the bf16 storage format implies, and it gives the size of that rounding
for a chain of layers.  It is never the reference of a parity check."""
from __future__ import annotations

import numpy as np
import torch

from oracle import hymba_oracle as O


def bf16(a) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even), returned as fp64."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def _attention_p_rounded(q, k, v, s: O.Spec) -> np.ndarray:
    """Eq. 1 per head with P rounded to bf16 before P V; the normaliser is the sum of the
    unrounded P (as the tensor-core kernel accumulates it in fp32)."""
    L = q.shape[0]
    H, G, dq, dv = s.n_heads, s.n_kv_heads, s.head_dim_qk, s.head_dim_v
    allowed = O.mask_matrix(L, s.n_meta, s.window, s.is_global)
    out = np.empty((L, H * dv))
    for h in range(H):
        g = h // (H // G)
        sc = (q[:, h * dq:(h + 1) * dq] @ k[:, g * dq:(g + 1) * dq].T) * s.score_scale
        sc = np.where(allowed, sc, -np.inf)
        p = np.exp(sc - sc.max(axis=1, keepdims=True))
        out[:, h * dv:(h + 1) * dv] = (bf16(p) @ v[:, g * dv:(g + 1) * dv]) / p.sum(axis=1, keepdims=True)
    return out


def layer_prefill(xt, w: dict, s: O.Spec, kv_from: dict | None = None) -> dict:
    """One sequence through the layer with the bf16 roundings of the CUDA path."""
    xt = np.asarray(xt, dtype=np.float64)
    consumer = kv_from is not None
    q, k, v, xs, z = O.in_proj(xt, np.asarray(w["w_in"], np.float64), s, consumer)
    q, xs, gate = bf16(q), bf16(xs), bf16(O.silu(z))
    if consumer:
        k, v = kv_from["k"], kv_from["v"]
    else:
        k, v = bf16(k), bf16(v)
    o = bf16(_attention_p_rounded(q, k, v, s))
    u = bf16(O.causal_conv_silu(xs, w["conv_w"], w["conv_b"]))
    delta, Bm, Cm = O.ssm_inputs(u, w["w_x"], w["w_dt"], w["b_dt"], s)
    delta = bf16(delta)
    y, h = O.selective_scan(u, delta, -np.exp(w["a_log"]), Bm, Cm, w["d_skip"])
    y_ssm = bf16(y * gate)
    f = bf16(O.fuse(o, y_ssm, w["beta_attn"], w["beta_ssm"], s.eps))
    Y = bf16(f @ np.asarray(w["w_out"], np.float64).T)
    return dict(q=q, k=k, v=v, x_ssm=xs, gate=gate, o=o, u=u, delta=delta, y_ssm=y_ssm, f=f, Y=Y, h=h)


def block_prefill(xt, w: dict, s: O.Spec, kv_from: dict | None = None):
    """The block (norm1, mixer, residual, norm2, gated MLP, residual) with the bf16 roundings
    of the CUDA path: the normed rows, the residual stream after each half and the MLP's
    hidden rows are stored in bf16.  Returns (out, the mixer's result dict)."""
    xt = np.asarray(xt, dtype=np.float64)
    xn = bf16(O.rms_norm(xt, np.asarray(w["norm1"], np.float64), s.eps))
    mix = layer_prefill(xn, w, s, kv_from=kv_from)
    h = bf16(xt + mix["f"] @ np.asarray(w["w_out"], np.float64).T)
    hn = bf16(O.rms_norm(h, np.asarray(w["norm2"], np.float64), s.eps))
    hid = bf16(O.silu(hn @ np.asarray(w["w_gate"], np.float64).T) * (hn @ np.asarray(w["w_up"], np.float64).T))
    out = bf16(h + hid @ np.asarray(w["w_down"], np.float64).T)
    return out, mix


def stack_prefill(xt, weights: list, specs: list, producers: list):
    x = np.asarray(xt, dtype=np.float64)
    mixes = []
    for w, s, p in zip(weights, specs, producers):
        x, mix = block_prefill(x, w, s, kv_from=None if p is None else mixes[p])
        mixes.append(mix)
    return x, mixes
