"""The bf16 rounding model behind the GPU tests' tolerances (CPU only).

tests/_bf16_emulation.py runs the oracle with every intermediate that the bf16 CUDA path
stores rounded to bf16 at the same place.  On the seeded workloads of the GPU tests this
checks three things:
  1. rounding alone uses at most half of every elementwise stage bound the GPU tests
     apply (the stated 2e-2 + 2e-2|o| on the projections; on the stages whose terms
     cancel, 2e-2 x the stage's error magnitude) and at most 0.6 of their relative L2
     tolerance of 1e-2 (tests/_bounds.py), so those bounds leave room for the kernels' own fp32 (and, for
     dt_proj, tf32) arithmetic and nothing more; the layer output, held to the stated
     bound as it is, uses 0.63 of it (0.93 on the scan-stress set);
  2. the bound of two chained layers: the chain's error spread over one layer's is the
     factor applied to the single-layer bound (1.5), and the chain's rounding uses at
     most 3/4 of that bound;
  3. the checks are not vacuous: plausible mistakes planted in the scan (a step lag in B
     or in delta, B and C swapped, the states reordered, the exp2 scaling applied to exp,
     delta dropped from the input term, the D skip dropped) all fail them (the relative L2
     check by a factor of 26 or more)."""
from __future__ import annotations

import numpy as np
import pytest

import synth
from oracle import hymba_oracle as O
from synth.configs import STRESS_DELTA_STD, STRESS_STD, LayerDims, Workload
from tests import _bf16_emulation as E
from tests import _bounds as BD
from tests import _harness as H

pytestmark = pytest.mark.slow

MAG_KEYS = ("u", "B", "C", "delta", "h", "y_ssm", "o", "f")


def _case(w, b, std=synth.configs.DEFAULT_STD):
    s = H.spec_of(w)
    wt = {k: H.to64(v) for k, v in synth.configs.layer_weights(w, 0, std=std).items()}
    x = H.to64(synth.configs.x_tilde(w)[b])
    ref = O.layer_prefill(x, wt, s)
    emu = E.layer_prefill(x, wt, s)
    R, N = s.dt_rank, s.d_state
    xd = emu["u"] @ wt["w_x"].T
    emu["B"], emu["C"] = xd[:, R:R + N], xd[:, R + N:]
    return s, wt, x, ref, emu, BD.prefill_magnitudes(x, wt, s, ref)


def _stated(g, o):
    return float((np.abs(g - o) / (2e-2 + 2e-2 * np.abs(o))).max())


EDGE_DIMS = LayerDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim_qk=64, d_inner=512)


@pytest.mark.parametrize("which", ["default", "stress", "stress_delta", "edge_one_row", "edge_ragged"])
def test_rounding_uses_at_most_half_of_each_bound(which):
    std = synth.configs.DEFAULT_STD
    if which == "default":
        w, b = H.small_workload("t_bf16_pair_b2_n300", window=256), 0
    elif which == "stress":
        w, b, std = H.small_workload("t_bf16_stress_b2_n200", n_tokens=200, n_meta=16, window=64), 1, STRESS_STD
    elif which == "stress_delta":
        w, b, std = (H.small_workload("t_bf16_stress_delta_b2_n200", n_tokens=200, n_meta=16, window=64), 1,
                     STRESS_DELTA_STD)
    elif which == "edge_one_row":  # one row, no meta: the state is a single term delta B u
        w, b = Workload("edge_bf16_1_0_1_4", EDGE_DIMS, "bf16", 1, 0, 1, 4), 0
    else:
        w, b = Workload("edge_bf16_3_130_127_129", EDGE_DIMS, "bf16", 3, 130, 127, 129), 0
    s, wt, x, ref, emu, mag = _case(w, b, std)
    ref["gate"] = O.silu(ref["z"])
    for key in ("q", "k", "v", "x_ssm", "gate"):
        assert _stated(emu[key], ref[key]) <= 0.5, key
    # the layer output is held to the stated bound as it is: rounding alone stays inside it
    # (it takes 0.63 of it with the default weights, 0.93 on the scan-stress set); on the
    # varying-delta set it does not (1.24), so that set is compared stage by stage only
    if which != "stress_delta":
        assert _stated(emu["Y"], ref["Y"]) <= (0.95 if which == "stress" else 0.7)
    for key in MAG_KEYS:
        r = float((np.abs(emu[key] - ref[key]) / BD.bound_of(ref[key], mag[key])).max())
        assert r <= 0.5, (key, r)
        rel = np.linalg.norm(emu[key] - ref[key]) / np.linalg.norm(ref[key])
        assert rel <= 0.6e-2, (key, rel)


def test_chained_pair_bound_from_the_rounding_model():
    w = H.small_workload("t_bf16_pair_b2_n300", window=256)
    s = H.spec_of(w)
    wp = {k: H.to64(v) for k, v in synth.configs.layer_weights(w, 0).items()}
    wc = {k: H.to64(v) for k, v in synth.configs.layer_weights(w, 1, consumer=True).items()}
    x = H.to64(synth.configs.x_tilde(w)[0])
    r1, e1 = O.layer_prefill(x, wp, s), E.layer_prefill(x, wp, s)
    r2 = O.layer_prefill(r1["Y"], wc, s, kv_from=r1)
    e2 = E.layer_prefill(e1["Y"], wc, s, kv_from=e1)
    spread = np.std(e2["Y"] - r2["Y"]) / np.std(e1["Y"] - r1["Y"])
    assert 1.0 < spread <= H.CHAIN2_ATOL / 2e-2, spread
    chain = float((np.abs(e2["Y"] - r2["Y"]) / (H.CHAIN2_ATOL + H.CHAIN2_RTOL * np.abs(r2["Y"]))).max())
    assert chain <= 0.75, chain


def _scan_variant(u, d, A, B, C, D, lag_delta=False, drop_delta=False):
    T, E_ = u.shape
    h = np.zeros_like(A)
    y = np.empty((T, E_))
    dprev = np.zeros(E_)
    for t in range(T):
        dec = np.exp((dprev if lag_delta else d[t])[:, None] * A)
        inp = (u[t] if drop_delta else d[t] * u[t])[:, None] * B[t][None, :]
        h = dec * h + inp
        y[t] = h @ C[t] + D * u[t]
        dprev = d[t]
    return y, h


def _fails(g, o, mag, rel_tol=1e-2):
    over = (np.abs(g - o) > BD.bound_of(o, mag)).any()
    rel = np.linalg.norm(g - o) / np.linalg.norm(o)
    return bool(over or rel > rel_tol)


def test_planted_scan_mistakes_fail_the_bounds():
    w = H.small_workload("t_bf16_stress_delta_b2_n200", n_tokens=200, n_meta=16, window=64)
    s, wt, x, ref, emu, mag = _case(w, 1, STRESS_DELTA_STD)
    A = -np.exp(wt["a_log"])
    u, d, B, C, D = ref["u"], ref["delta"], ref["B"], ref["C"], wt["d_skip"]
    mistakes = {
        "B one step late": O.selective_scan(u, d, A, np.roll(B, 1, 0), C, D),
        "delta one step late in the decay": _scan_variant(u, d, A, B, C, D, lag_delta=True),
        "delta missing from the input term": _scan_variant(u, d, A, B, C, D, drop_delta=True),
        "exp2 scaling applied to exp": O.selective_scan(u, d * 1.4426950408889634, A, B, C, D),
        "B and C swapped": O.selective_scan(u, d, A, C, B, D),
        "states reordered": O.selective_scan(u, d, A, B[:, ::-1], C, D),
    }
    for name, (y, h) in mistakes.items():
        assert _fails(h, ref["h"], mag["h"]), name
        assert _fails(y * O.silu(ref["z"]), ref["y_ssm"], mag["y_ssm"]), name
    # the D skip dominates the SSM output with the default weights: dropping it must show
    w2 = H.small_workload("t_bf16_pair_b2_n300", window=256)
    s2, wt2, x2, ref2, emu2, mag2 = _case(w2, 0)
    y, _ = O.selective_scan(ref2["u"], ref2["delta"], -np.exp(wt2["a_log"]), ref2["B"], ref2["C"],
                            0 * wt2["d_skip"])
    assert _fails(y * O.silu(ref2["z"]), ref2["y_ssm"], mag2["y_ssm"])


def test_block_stack_rounding_within_the_chained_bound():
    """Four blocks (global, sliding-window producer, consumer, global) with the bf16
    roundings of the CUDA path: the stack's output error stays within 0.6 of the
    two-chained-layer bound that the GPU test applies to it."""
    D = LayerDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim_qk=64, d_inner=512)
    w = Workload("block_stack", D, "bf16", 2, 16, 200, 64)
    layout = [(True, None), (False, None), (False, 1), (True, None)]
    ws, specs, prods = [], [], []
    for l, (g, p) in enumerate(layout):
        lw = {k: H.to64(v) for k, v in synth.configs.layer_weights(w, l, consumer=p is not None).items()}
        lw.update({k: H.to64(v) for k, v in synth.configs.block_weights(w, l, 512).items()})
        ws.append(lw)
        specs.append(H.spec_of(w, g))
        prods.append(p)
    for b in range(2):
        x = H.to64(synth.configs.x_tilde(w)[b])
        r, _ = O.stack_prefill(x, ws, specs, prods)
        e, _ = E.stack_prefill(x, ws, specs, prods)
        ratio = float((np.abs(e - r) / (H.CHAIN2_ATOL + H.CHAIN2_RTOL * np.abs(r))).max())
        assert ratio <= 0.6, ratio
