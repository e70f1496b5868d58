"""bf16 path at the 1.5B layer widths on short sequences (several 128-row tiles
and a ragged tail), stage by stage and end to end against the fp64 oracle;
KV sharing; decode after prefill; scan-stress weights."""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import hybrid_attention_ssm_head_b200 as hy
import synth
from oracle import hymba_oracle as O
from synth.configs import STRESS_DELTA_STD, STRESS_STD
from tests import _bf16_emulation as EMU
from tests import _bounds as BD
from tests import _harness as H

pytestmark = pytest.mark.gpu

# Stages compared elementwise.  Outputs of the input projection (the gate as SiLU(z))
# against the stated bf16 bound; stages that are sums whose terms cancel (and delta, which
# follows its low-rank sum) elementwise against 2e-2 x their first-order error magnitude
# (tests/_bounds.py) and as a whole against a relative L2 error of 1e-2.
GEMM_STAGES = [("q", "q"), ("x_ssm", "x_ssm"), ("gate", "gate")]
MAG_STAGES = [("u", "u"), ("y_ssm", "y_ssm"), ("o_attn", "o"), ("fused", "f")]


def _check_prefill(w, lay, x, y, ws, k, v, h=None, conv=None, rows=(0,), stages=True, kv_from=None,
                   diag=None):
    B, L = x.shape[0], x.shape[1]
    for b in rows:
        chk = H.Checks()
        ow = H.oracle_weights(lay.cpu)
        ref = O.layer_prefill(H.to64(x[b]), ow, lay.spec, kv_from=kv_from[b] if kv_from is not None else None)
        ref["gate"] = O.silu(ref["z"])  # the input projection stores the gate SiLU(z)
        mag = BD.prefill_magnitudes(H.to64(x[b]), ow, lay.spec, ref,
                                    kv_from=kv_from[b] if kv_from is not None else None)
        got = {}
        if stages:
            for name, key in GEMM_STAGES:
                got[key] = H.to64(H.stage(lay, ws, B, L, name)[b])
                chk(H.close_bf16, got[key], ref[key], f"{name}[b={b}]")
            for name, key in MAG_STAGES + [("delta", "delta")]:
                got[key] = H.to64(H.stage(lay, ws, B, L, name)[b])
            xd = H.to64(H.stage(lay, ws, B, L, "xdbl")[b])
            R = lay.spec.dt_rank
            got["B"], got["C"] = xd[:, R:R + 16], xd[:, R + 16:]
            for key in ("u", "delta", "B", "C", "y_ssm", "o", "f"):
                chk(BD.close_mag, got[key], ref[key], mag[key], f"{key}[b={b}]")
                chk(H.close_rel_l2, got[key], ref[key], 1e-2, f"{key}[b={b}]")
            if kv_from is None:
                chk(H.close_bf16, H.to64(k[b]), ref["k"], "k")
                chk(H.close_bf16, H.to64(v[b]), ref["v"], "v")
        got["Y"] = H.to64(y[b])
        chk(H.close_bf16, got["Y"], ref["Y"], f"Y[b={b}]")
        if h is not None:
            got["h"], got["conv"] = H.to64(h[b]), H.to64(conv[b])
            chk(BD.close_mag, got["h"], ref["h"], mag["h"], "h_final")
            chk(H.close_rel_l2, got["h"], ref["h"], 1e-2, "h_final")
            chk(H.close_bf16, got["conv"], ref["conv"], "conv_state")
            if stages:
                # the conv state is a copy of this call's last x_ssm rows: bit for bit
                want = H.conv_state_from_stage(H.stage(lay, ws, B, L, "x_ssm")[b], lay.spec.d_conv)
                chk(H.assert_bits_equal, conv[b], want, "conv_state copy")
        if diag and chk.errors:
            H.diag_dump(f"{diag}_b{b}", got)
        chk.done()
        yield b, ref


@pytest.mark.parametrize("glob", [False, True])
def test_bf16_prefill_stage_parity(glob):
    w = H.small_workload("t_bf16_b2_n300_m128_w256", window=0 if glob else 256)
    lay = H.GpuLayer(w, 0)
    B, L = w.batch, w.seq_rows
    x = synth.configs.x_tilde(w).cuda()
    k, v, kv = H.alloc_kv_seq(w, B, L)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y, ws = H.run_prefill(lay, x, kv, None, ssm)
    assert kv.owner != 0 and kv.rows == L and kv.batch == B
    for _ in _check_prefill(w, lay, x, y, ws, k, v, h, conv, rows=(0, 1),
                            diag="prefill_global" if glob else "prefill_swa"):
        pass
    lay.close()


def test_bf16_scan_stress_parity():
    """u, B, C of order one and D = 0: the recurrence term carries the SSM output."""
    w = H.small_workload("t_bf16_stress_b2_n200", n_tokens=200, n_meta=16, window=64)
    lay = H.GpuLayer(w, 0, std=STRESS_STD)
    B, L = w.batch, w.seq_rows
    x = synth.configs.x_tilde(w).cuda()
    k, v, kv = H.alloc_kv_seq(w, B, L)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y, ws = H.run_prefill(lay, x, kv, None, ssm)
    for b, ref in _check_prefill(w, lay, x, y, ws, k, v, h, conv, rows=(0, 1), diag="stress"):
        # the recurrence is visible: y_ssm far from zero and not the D*u skip (D = 0)
        assert np.abs(ref["y"]).mean() > 1e-2
    lay.close()


def test_bf16_scan_stress_varying_delta_stages():
    """The scan-stress set with a delta that varies along the sequence, so that a slip in how
    the decay uses delta shows: the SSM stages and the final state, stage by stage."""
    w = H.small_workload("t_bf16_stress_delta_b2_n200", n_tokens=200, n_meta=16, window=64)
    lay = H.GpuLayer(w, 0, std=STRESS_DELTA_STD)
    B, L = w.batch, w.seq_rows
    x = synth.configs.x_tilde(w).cuda()
    k, v, kv = H.alloc_kv_seq(w, B, L)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y, ws = H.run_prefill(lay, x, kv, None, ssm)
    ow = H.oracle_weights(lay.cpu)
    R = lay.spec.dt_rank
    for b in range(B):
        chk = H.Checks()
        ref = O.layer_prefill(H.to64(x[b]), ow, lay.spec)
        mag = BD.ssm_magnitudes(ow, lay.spec, ref)
        xd = H.to64(H.stage(lay, ws, B, L, "xdbl")[b])
        got = dict(u=H.to64(H.stage(lay, ws, B, L, "u")[b]), delta=H.to64(H.stage(lay, ws, B, L, "delta")[b]),
                   y_ssm=H.to64(H.stage(lay, ws, B, L, "y_ssm")[b]), B=xd[:, R:R + 16], C=xd[:, R + 16:],
                   h=H.to64(h[b]))
        for key in got:
            chk(BD.close_mag, got[key], ref[key], mag[key], f"{key}[b={b}]")
        chk(H.close_rel_l2, got["h"], ref["h"], 1e-2, "h")
        chk(H.close_rel_l2, got["y_ssm"], ref["y_ssm"], 1e-2, "y_ssm")
        assert float(ref["delta"].max() / ref["delta"].min()) > 3.0  # delta does vary
        chk.done()
    lay.close()


def test_bf16_kv_shared_pair():
    """Layer 2 attends over layer 1's K/V and projects none of its own.  Strict parity with
    an independent seeded input for each layer; the chained case (layer 2 fed layer 1's
    bf16 output) against the two-layer bound."""
    w = H.small_workload("t_bf16_pair_b2_n300", window=256)
    prod = H.GpuLayer(w, 0)
    cons = H.GpuLayer(w, 1, consumer=True)
    hy.hymba_kv_share_bind(cons.handle, prod.handle)
    B, L = w.batch, w.seq_rows
    x = synth.configs.x_tilde(w).cuda()
    x2 = synth.gen.normal_tensor((B, L, w.dims.d_model), 0, "t_bf16_pair/x2", device="cuda").to(torch.bfloat16)
    k, v, kv = H.alloc_kv_seq(w, B, L)
    y1, ws = H.run_prefill(prod, x, kv)
    y2, ws = H.run_prefill(cons, x2, kv, ws=ws)
    y2c, ws = H.run_prefill(cons, y1, kv, ws=ws)
    for b in range(B):
        wp, wc = H.oracle_weights(prod.cpu), H.oracle_weights(cons.cpu)
        ref1 = O.layer_prefill(H.to64(x[b]), wp, prod.spec)
        H.close_bf16(H.to64(y1[b]), ref1["Y"], "producer Y")
        ref2 = O.layer_prefill(H.to64(x2[b]), wc, cons.spec, kv_from=ref1)
        H.close_bf16(H.to64(y2[b]), ref2["Y"], "consumer Y")
        # chained: the oracle chains its own fp64 output
        ref2c = O.layer_prefill(ref1["Y"], wc, cons.spec, kv_from=ref1)
        H.close_chain2(H.to64(y2c[b]), ref2c["Y"], "chained consumer Y")
        # the chain's error is the bf16 rounding the storage format implies: its spread
        # matches the rounding model's (the model run on the same seeded inputs)
        e1 = EMU.layer_prefill(H.to64(x[b]), wp, prod.spec)
        e2 = EMU.layer_prefill(e1["Y"], wc, cons.spec, kv_from=e1)
        sd_gpu = float(np.std(H.to64(y2c[b]) - ref2c["Y"]))
        sd_model = float(np.std(e2["Y"] - ref2c["Y"]))
        assert 0.75 * sd_model <= sd_gpu <= 1.25 * sd_model, (sd_gpu, sd_model)
    # the consumer refuses a K/V store its producer did not stamp
    kv2 = hy.hymba_kv_seq(kv.k, kv.v, B, L, 12345)
    with pytest.raises(hy.HymbaError):
        H.run_prefill(cons, y1, kv2, ws=ws)
    prod.close()
    cons.close()


@pytest.mark.parametrize("kind", ["swa", "global", "consumer"])
def test_bf16_decode_after_prefill(kind):
    w = H.small_workload("t_bf16_dec_b3_n400", batch=3, n_tokens=400, window=0 if kind == "global" else 256)
    prod = H.GpuLayer(w, 0)
    B, L = w.batch, w.seq_rows
    cap = L + 8 if kind == "global" else w.n_meta + w.window
    xs = synth.configs.x_tilde(w).cuda()
    x_new = synth.gen.normal_tensor((B, w.dims.d_model), 0, "t_bf16_dec/xnew", device="cuda").to(torch.bfloat16)
    k, v, kv = H.alloc_kv_seq(w, B, L)
    kc, vc, kvc = H.alloc_kv_cache(w, B, cap)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y, ws = H.run_prefill(prod, xs, kv, kvc, ssm)
    layer = prod
    if kind == "consumer":
        cons = H.GpuLayer(w, 1, consumer=True)
        hy.hymba_kv_share_bind(cons.handle, prod.handle)
        h2, conv2, ssm2 = H.alloc_ssm_cache(w, B)
        xs2 = synth.gen.normal_tensor((B, L, w.dims.d_model), 0, "t_bf16_dec/x2",
                                      device="cuda").to(torch.bfloat16)
        y2, ws = H.run_prefill(cons, xs2, kv, None, ssm2, ws=ws)
    dws = H.workspace(hy.hymba_layer_decode_workspace(prod.handle, B, L))
    yt = torch.empty_like(x_new)
    conv_before = conv.clone()
    hy.hymba_layer_decode_step(prod.handle, B, L, x_new, yt, kvc, ssm, dws, dws.numel(),
                               torch.cuda.current_stream())
    hy.hymba_stream_status(torch.cuda.current_stream())
    if kind == "consumer":
        x_new2 = synth.gen.normal_tensor((B, w.dims.d_model), 0, "t_bf16_dec/xnew2",
                                         device="cuda").to(torch.bfloat16)
        yt2 = torch.empty_like(x_new)
        hy.hymba_layer_decode_step(cons.handle, B, L, x_new2, yt2, kvc, ssm2, dws, dws.numel(),
                                   torch.cuda.current_stream())
        hy.hymba_stream_status(torch.cuda.current_stream())
    for b in range(B):
        refp = O.layer_prefill(H.to64(xs[b]), H.oracle_weights(prod.cpu), prod.spec, capacity=cap)
        cache = dict(k=refp["k_cache"], v=refp["v_cache"], ssm=refp["h"], conv=refp["conv"])
        yo, newc = O.layer_decode(H.to64(x_new[b]), L, H.oracle_weights(prod.cpu), prod.spec, cache)
        H.close_bf16(H.to64(yt[b]), yo, f"decode y[b={b}]")
        h0m = BD.ssm_magnitudes(H.oracle_weights(prod.cpu), prod.spec, refp)["h"]  # the prefill's state
        hm = BD.decode_state_magnitude(H.to64(x_new[b]), L, H.oracle_weights(prod.cpu), prod.spec, cache,
                                       h0_mag=h0m)
        BD.close_mag(H.to64(h[b]), newc["ssm"], hm, "decode h")
        H.close_rel_l2(H.to64(h[b]), newc["ssm"], 1e-2, "decode h")
        # the window moves by one row: the older rows are the prefill's, bit for bit
        H.assert_bits_equal(conv[b][:-1], conv_before[b][1:], "decode conv, shifted rows")
        H.close_bf16(H.to64(conv[b][-1]), newc["conv"][-1], "decode conv, new row")
        # the appended K/V row sits at its slot
        sl = O.kv_slot(L, prod.spec)
        H.close_bf16(H.to64(kc[b][:, sl]), newc["k"][:, sl], "appended k")
        H.close_bf16(H.to64(vc[b][:, sl]), newc["v"][:, sl], "appended v")
        if kind == "consumer":
            refc = O.layer_prefill(H.to64(xs2[b]), H.oracle_weights(cons.cpu), cons.spec, kv_from=refp)
            yc, _ = O.layer_decode(H.to64(x_new2[b]), L, H.oracle_weights(cons.cpu), cons.spec,
                                   dict(ssm=refc["h"], conv=refc["conv"]), kv_cache=newc)
            H.close_bf16(H.to64(yt2[b]), yc, f"consumer decode y[b={b}]")
    prod.close()
    if kind == "consumer":
        cons.close()
