"""Tiny seeded layers for the oracle's self-checks (numpy RNG, CPU only)."""
from __future__ import annotations

import numpy as np

from oracle.hymba_oracle import Spec


def spec(d=24, H=4, G=2, dq=8, E=32, N=4, K=4, R=3, m=3, W=5, is_global=False, eps=1e-6):
    return Spec(d_model=d, n_heads=H, n_kv_heads=G, head_dim_qk=dq, head_dim_v=E // H,
                d_inner=E, d_state=N, d_conv=K, dt_rank=R, n_meta=m, window=W,
                is_global=is_global, eps=eps)


def in_width(s: Spec, consumer=False):
    kv = 0 if consumer else s.n_kv_heads * (s.head_dim_qk + s.head_dim_v)
    return s.n_heads * s.head_dim_qk + kv + 2 * s.d_inner


def weights(s: Spec, seed=0, consumer=False, scale_in=0.3, scan_stress=True):
    """Weights with O(1) branch outputs so that every term of the layer is visible."""
    r = np.random.default_rng(seed)
    E, N, R, K = s.d_inner, s.d_state, s.dt_rank, s.d_conv
    return dict(
        w_in=r.normal(0, scale_in, (in_width(s, consumer), s.d_model)),
        conv_w=r.normal(0, 0.5, (E, K)),
        conv_b=r.normal(0, 0.5, (E,)),
        w_x=r.normal(0, 1.0 / np.sqrt(E), (R + 2 * N, E)) * (1.0 if scan_stress else 0.1),
        w_dt=r.normal(0, 0.5, (E, R)),
        b_dt=r.normal(-1.0, 1.0, (E,)),
        a_log=r.uniform(0, np.log(16.0), (E, N)),
        d_skip=r.normal(0, 1.0, (E,)),
        beta_attn=r.uniform(0.5, 1.5, (E,)),
        beta_ssm=r.uniform(0.5, 1.5, (E,)),
        w_out=r.normal(0, 1.0 / np.sqrt(E), (s.d_model, E)),
    )


def x_tilde(s: Spec, L, seed=1):
    r = np.random.default_rng(seed)
    return r.normal(0, 1.0, (L, s.d_model))
