"""Shapes of the five workloads and the seeded recipe for every tensor.

Sizes follow the 1.5B column of the architecture table of "Hymba: A Hybrid-head
Architecture for Small Language Models" (Appendix E, Table 11: hidden 1600,
25 attention heads, 5 query groups, SSM state 16, window 1024) and the meta-token
count of 128 given in the authors' OpenReview reply (question on the number of
meta tokens).  Distributions: real input rows N(0,1); linear, conv and meta
weights N(0, 0.02); A_log ~ U(0, ln 16) so that A = -exp(A_log) lies in
[-16, -1]; dt bias N(0,1) - 4 so that delta ~ softplus(N(0,1) - 4); D = 1;
beta = 1.  "N(0,1)" is the twelve-term Irwin-Hall approximation of
``synth.gen`` (exact on CPU and GPU alike).

No arithmetic of the layer lives here: only shapes, names and distributions.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

from . import gen


@dataclass(frozen=True)
class LayerDims:
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim_qk: int
    d_inner: int
    d_state: int = 16
    d_conv: int = 4
    dt_rank: int = 0  # 0 -> ceil(d_model / 16)

    @property
    def head_dim_v(self) -> int:
        return self.d_inner // self.n_heads

    @property
    def rank(self) -> int:
        return self.dt_rank if self.dt_rank > 0 else math.ceil(self.d_model / 16)

    def in_width(self, consumer: bool = False) -> int:
        kv = 0 if consumer else self.n_kv_heads * (self.head_dim_qk + self.head_dim_v)
        return self.n_heads * self.head_dim_qk + kv + 2 * self.d_inner

    @property
    def xproj_width(self) -> int:
        return self.rank + 2 * self.d_state


@dataclass(frozen=True)
class Workload:
    name: str
    dims: LayerDims
    dtype: str          # "f32" | "bf16"
    batch: int
    n_meta: int
    n_tokens: int       # real tokens n; rows per sequence L = n_meta + n_tokens
    window: int         # <= 0 means global
    n_layers: int = 1
    kv_shared_pair: bool = False
    decode: bool = False
    seed: int = 0
    rope_base: float = 0.0  # rotary position embedding of Q and K: 0 = none

    @property
    def seq_rows(self) -> int:
        return self.n_meta + self.n_tokens


DIMS_SMALL = LayerDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim_qk=64, d_inner=512)
DIMS_1P5B = LayerDims(d_model=1600, n_heads=25, n_kv_heads=5, head_dim_qk=64, d_inner=3200)

CFG0 = Workload("cfg0_f32_b1_n256_m16_w64", DIMS_SMALL, "f32", 1, 16, 256, 64)
CFG1 = Workload("cfg1_bf16_b8_n4096_m128_w1024", DIMS_1P5B, "bf16", 8, 128, 4096, 1024)
CFG2 = Workload("cfg2_bf16_b4_n8192_m128_global", DIMS_1P5B, "bf16", 4, 128, 8192, 0)
CFG3 = Workload("cfg3_bf16_b128_n8192_m128_w1024_kvpair", DIMS_1P5B, "bf16", 128, 128, 8192,
                1024, n_layers=2, kv_shared_pair=True)
CFG4 = Workload("cfg4_bf16_decode_b128_ctx8192_m128_32layers", DIMS_1P5B, "bf16", 128, 128, 8192,
                1024, n_layers=32, decode=True)
CONFIGS = [CFG0, CFG1, CFG2, CFG3, CFG4]

# Stack layout for the 32-layer decode workload: global attention in the first,
# middle and last layers; the remaining sliding-window layers form consecutive
# KV-sharing pairs inside each run of local layers.
GLOBAL_LAYERS_32 = (0, 15, 31)


def stack_layout(n_layers: int = 32, global_layers=GLOBAL_LAYERS_32):
    """Per layer: (is_global, producer_index or None).  producer None -> owns its K/V."""
    out = []
    run_start = None
    for l in range(n_layers):
        if l in global_layers:
            out.append((True, None))
            run_start = None
            continue
        if run_start is None or (l - run_start) % 2 == 0:
            out.append((False, None))
            if run_start is None:
                run_start = l
        else:
            out.append((False, l - 1))
    return out


def torch_dtype(dt: str):
    return torch.float32 if dt == "f32" else torch.bfloat16


@dataclass(frozen=True)
class WeightStd:
    """Standard deviations of the seeded weights (the default is the workloads' recipe)."""
    w_in: float = 0.02
    conv_w: float = 0.02
    conv_b: float = 0.02
    w_x_dt: float = 0.02   # rows of W_x producing the low-rank delta input
    w_x_bc: float = 0.02   # rows of W_x producing B and C
    w_x_bc_unit_gain: bool = False  # True: B/C rows use std 1/sqrt(d_inner) instead
    w_dt: float = 0.02
    w_out: float = 0.02
    meta: float = 0.02
    d_skip: float = 1.0    # D is constant: this value
    beta_attn: float = 1.0
    beta_ssm: float = 1.0


DEFAULT_STD = WeightStd()
# "Scan-stress" set: u, B and C of order one and D = 0, so that the recurrence
# term dominates the SSM output instead of the D*u skip.
STRESS_STD = replace(DEFAULT_STD, conv_w=0.5, conv_b=0.5, w_x_bc_unit_gain=True, d_skip=0.0)
# The same with a dt projection of std 0.2, so that delta varies by a factor of several
# along the sequence (with the default weights it is nearly constant: softplus(b_dt) plus
# a ~5e-3 input term), which makes the decay's use of delta visible.
STRESS_DELTA_STD = replace(STRESS_STD, w_dt=0.2)


def layer_weights(w: Workload, layer: int, consumer: bool = False, device="cpu",
                  std: WeightStd = DEFAULT_STD, tag: str = "") -> dict:
    """Seeded weights of one layer.  Matrices are in the workload's storage dtype;
    per-channel parameters and W_dt are fp32."""
    d = w.dims
    dt = torch_dtype(w.dtype)
    s = w.seed
    pre = f"{w.name}/L{layer}{tag}/"
    E, N, R, K = d.d_inner, d.d_state, d.rank, d.d_conv
    nq = d.n_heads * d.head_dim_qk
    nkv = d.n_kv_heads * (d.head_dim_qk + d.head_dim_v)
    rows_q = gen.normal_tensor((nq, d.d_model), s, pre + "w_q", std.w_in, device=device)
    rows_kv = gen.normal_tensor((nkv, d.d_model), s, pre + "w_kv", std.w_in, device=device)
    rows_sz = gen.normal_tensor((2 * E, d.d_model), s, pre + "w_ssm_g", std.w_in, device=device)
    if consumer:
        w_in = torch.cat([rows_q, rows_sz], 0)
    else:
        w_in = torch.cat([rows_q, rows_kv, rows_sz], 0)
    bc_std = 1.0 / math.sqrt(E) if std.w_x_bc_unit_gain else std.w_x_bc
    w_x = torch.cat([
        gen.normal_tensor((R, E), s, pre + "w_x_dt", std.w_x_dt, device=device),
        gen.normal_tensor((2 * N, E), s, pre + "w_x_bc", bc_std, device=device)], 0)
    out = dict(
        w_in=w_in.to(dt),
        conv_w=gen.normal_tensor((E, K), s, pre + "conv_w", std.conv_w, device=device),
        conv_b=gen.normal_tensor((E,), s, pre + "conv_b", std.conv_b, device=device),
        w_x=w_x.to(dt),
        w_dt=gen.normal_tensor((E, R), s, pre + "w_dt", std.w_dt, device=device),
        b_dt=gen.normal_tensor((E,), s, pre + "b_dt", 1.0, -4.0, device=device),
        a_log=gen.uniform_tensor((E, N), s, pre + "a_log", 0.0, math.log(16.0), device=device),
        d_skip=torch.full((E,), std.d_skip, dtype=torch.float32, device=device),
        beta_attn=torch.full((E,), std.beta_attn, dtype=torch.float32, device=device),
        beta_ssm=torch.full((E,), std.beta_ssm, dtype=torch.float32, device=device),
        w_out=gen.normal_tensor((d.d_model, E), s, pre + "w_out", std.w_out, device=device).to(dt),
    )
    return out


def block_weights(w: Workload, layer: int, mlp_hidden: int, device="cpu", std: float = 0.02) -> dict:
    """Seeded weights of a block's norms and MLP (the mixer's come from layer_weights):
    norm1, norm2 [d] fp32 ~ U(0.5, 1.5); w_gate, w_up [F, d] and w_down [d, F] N(0, std) in
    the storage dtype; and w_gate_up [2F, d], the gate and up rows interleaved (row 2i =
    w_gate row i, row 2i+1 = w_up row i), the layout the library takes."""
    d = w.dims.d_model
    dt = torch_dtype(w.dtype)
    pre = f"{w.name}/L{layer}/block/"
    s = w.seed
    wg = gen.normal_tensor((mlp_hidden, d), s, pre + "w_gate", std, device=device).to(dt)
    wu = gen.normal_tensor((mlp_hidden, d), s, pre + "w_up", std, device=device).to(dt)
    return dict(
        norm1=gen.uniform_tensor((d,), s, pre + "norm1", 0.5, 1.5, device=device),
        norm2=gen.uniform_tensor((d,), s, pre + "norm2", 0.5, 1.5, device=device),
        w_gate=wg, w_up=wu,
        w_gate_up=torch.stack([wg, wu], dim=1).reshape(2 * mlp_hidden, d).contiguous(),
        w_down=gen.normal_tensor((d, mlp_hidden), s, pre + "w_down", std, device=device).to(dt))


def meta_tokens(w: Workload, device="cpu", std: float = DEFAULT_STD.meta) -> torch.Tensor:
    """The m learnable meta rows R (seeded), [m, d_model], storage dtype."""
    return gen.normal_tensor((w.n_meta, w.dims.d_model), w.seed, f"{w.name}/meta", std,
                             device=device).to(torch_dtype(w.dtype))


def real_rows(w: Workload, batch_index: int | None = None, device="cpu",
              tag: str = "x") -> torch.Tensor:
    """Real input rows X, N(0,1): [batch, n, d] or, for one batch row, [n, d]."""
    n, d = w.n_tokens, w.dims.d_model
    name = f"{w.name}/{tag}"
    if batch_index is None:
        return gen.normal_tensor((w.batch, n, d), w.seed, name, device=device).to(torch_dtype(w.dtype))
    return gen.normal_tensor((n, d), w.seed, name, device=device,
                             offset=batch_index * n * d).to(torch_dtype(w.dtype))


def x_tilde(w: Workload, batch_index: int | None = None, device="cpu") -> torch.Tensor:
    """X~ = [R; X] per sequence (the concatenation is input assembly, not layer maths)."""
    meta = meta_tokens(w, device=device)
    x = real_rows(w, batch_index, device=device)
    if batch_index is None:
        return torch.cat([meta.unsqueeze(0).expand(w.batch, -1, -1), x], 1).contiguous()
    return torch.cat([meta, x], 0).contiguous()


def decode_caches(w: Workload, layer: int, capacity: int, consumer: bool, batch_index=None,
                  device="cpu") -> dict:
    """N(0,1) seeded decode caches of one layer.  K/V only for layers that own them.
    Layouts: k [B, Hkv, cap, dqk], v [B, Hkv, cap, dv], ssm [B, E, N] fp32,
    conv [B, d_conv-1, E]."""
    d = w.dims
    dt = torch_dtype(w.dtype)
    pre = f"{w.name}/L{layer}/cache/"

    def part(shape, name):
        per_b = 1
        for s in shape:
            per_b *= s
        if batch_index is None:
            return gen.normal_tensor((w.batch,) + tuple(shape), w.seed, pre + name, device=device)
        return gen.normal_tensor(tuple(shape), w.seed, pre + name, device=device,
                                 offset=batch_index * per_b)

    out = dict(
        ssm=part((d.d_inner, d.d_state), "ssm"),
        conv=part((d.d_conv - 1, d.d_inner), "conv").to(dt),
    )
    if not consumer:
        out["k"] = part((d.n_kv_heads, capacity, d.head_dim_qk), "k").to(dt)
        out["v"] = part((d.n_kv_heads, capacity, d.head_dim_v), "v").to(dt)
    return out


def decode_tokens(w: Workload, device="cpu") -> torch.Tensor:
    """The new token's hidden state per sequence, [B, d], N(0,1)."""
    return gen.normal_tensor((w.batch, w.dims.d_model), w.seed, f"{w.name}/x_t",
                             device=device).to(torch_dtype(w.dtype))
