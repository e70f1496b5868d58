"""Edge cases through the C ABI against the oracle: only meta rows (n = 0), a
single row, ragged lengths around the 128-row tiles, no meta tokens, window 1,
window >= L, meta count not a multiple of the tile, one sequence; both dtypes."""
from __future__ import annotations

import pytest
import torch

import hybrid_attention_ssm_head_b200 as hy
import synth
from oracle import hymba_oracle as O
from synth.configs import LayerDims
from tests import _bounds as BD
from tests import _harness as H

pytestmark = pytest.mark.gpu

# bf16 kernels need d_qk 64 and d_v 128: 4 heads over d_inner 512
DIMS_BF16_SMALL = LayerDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim_qk=64, d_inner=512)

CASES = [
    # (dtype, batch, n_meta, n_tokens, window)
    ("bf16", 1, 16, 0, 64),       # only meta rows
    ("bf16", 1, 0, 1, 4),         # one row, no meta
    ("bf16", 2, 0, 300, 1),       # window 1: each query sees itself only
    ("bf16", 2, 7, 250, 5000),    # window covers the sequence
    ("bf16", 3, 130, 127, 129),   # meta count past one tile, ragged tail
    ("bf16", 1, 128, 129, 0),     # global, one row past two tiles
    ("bf16", 2, 1, 383, 64),
    ("f32", 1, 0, 1, 4),
    ("f32", 2, 0, 100, 1),
    ("f32", 1, 5, 60, 0),
    ("f32", 2, 16, 200, 3000),
]


@pytest.mark.parametrize("dtype,B,m,n,W", CASES)
def test_edge_prefill(dtype, B, m, n, W):
    dims = DIMS_BF16_SMALL if dtype == "bf16" else synth.configs.DIMS_SMALL
    w = synth.configs.Workload(f"edge_{dtype}_{B}_{m}_{n}_{W}", dims, dtype, B, m, n, W)
    lay = H.GpuLayer(w, 0)
    L = w.seq_rows
    x = synth.configs.x_tilde(w).cuda() if n > 0 else \
        synth.configs.meta_tokens(w).unsqueeze(0).expand(B, -1, -1).contiguous().cuda()
    k, v, kv = H.alloc_kv_seq(w, B, L)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y, ws = H.run_prefill(lay, x, kv, None, ssm)
    for b in range(B):
        ref = O.layer_prefill(H.to64(x[b]), H.oracle_weights(lay.cpu), lay.spec)
        H.close(w, H.to64(y[b]), ref["Y"], f"Y[b={b}]")
        if dtype == "f32":
            H.close_f32(H.to64(h[b]), ref["h"], "h_final")
        else:
            mag = BD.ssm_magnitudes(H.oracle_weights(lay.cpu), lay.spec, ref)
            BD.close_mag(H.to64(h[b]), ref["h"], mag["h"], "h_final")
            H.close_rel_l2(H.to64(h[b]), ref["h"], 1e-2, "h_final")
            H.close_bf16(H.to64(conv[b]), ref["conv"], "conv_state")
    lay.close()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_edge_decode_short_context(dtype):
    """Decode right after the meta rows and with a context shorter than the window."""
    dims = DIMS_BF16_SMALL if dtype == "bf16" else synth.configs.DIMS_SMALL
    for n in (0, 3):
        w = synth.configs.Workload(f"edge_dec_{dtype}_{n}", dims, dtype, 2, 16, n, 64)
        lay = H.GpuLayer(w, 0)
        B, L = w.batch, w.seq_rows
        x = synth.configs.x_tilde(w).cuda() if n > 0 else \
            synth.configs.meta_tokens(w).unsqueeze(0).expand(B, -1, -1).contiguous().cuda()
        cap = w.n_meta + w.window
        k, v, kv = H.alloc_kv_seq(w, B, L)
        kc, vc, kvc = H.alloc_kv_cache(w, B, cap)
        h, conv, ssm = H.alloc_ssm_cache(w, B)
        H.run_prefill(lay, x, kv, kvc, ssm)
        xt = synth.gen.normal_tensor((B, dims.d_model), 0, f"edge_dec/{n}", device="cuda").to(
            synth.configs.torch_dtype(dtype))
        dws = H.workspace(hy.hymba_layer_decode_workspace(lay.handle, B, L))
        yt = torch.empty_like(xt)
        hy.hymba_layer_decode_step(lay.handle, B, L, xt, yt, kvc, ssm, dws, dws.numel(),
                                   torch.cuda.current_stream())
        hy.hymba_stream_status(torch.cuda.current_stream())
        for b in range(B):
            refp = O.layer_prefill(H.to64(x[b]), H.oracle_weights(lay.cpu), lay.spec, capacity=cap)
            yo, _ = O.layer_decode(H.to64(xt[b]), L, H.oracle_weights(lay.cpu), lay.spec,
                                   dict(k=refp["k_cache"], v=refp["v_cache"], ssm=refp["h"],
                                        conv=refp["conv"]))
            H.close(w, H.to64(yt[b]), yo, f"decode y n={n} b={b}")
        lay.close()


def test_nan_inputs_propagate_without_fault():
    """A NaN in one input row reaches that row's output and every later row (through the
    scan), no device error is raised, and the other sequence still matches the oracle."""
    w = synth.configs.Workload("edge_nan", DIMS_BF16_SMALL, "bf16", 2, 16, 100, 32)
    lay = H.GpuLayer(w, 0)
    B, L = w.batch, w.seq_rows
    x = synth.configs.x_tilde(w).cuda()
    x[0, 50, 3] = float("nan")
    k, v, kv = H.alloc_kv_seq(w, B, L)
    y, ws = H.run_prefill(lay, x, kv)
    assert torch.isnan(y[0, 50:]).any(dim=-1).all()
    ref = O.layer_prefill(H.to64(x[1]), H.oracle_weights(lay.cpu), lay.spec)
    H.close_bf16(H.to64(y[1]), ref["Y"], "clean sequence")
    lay.close()


def test_decode_nan_row_stays_in_its_row():
    """A NaN in one sequence's new row reaches that sequence's decode output and SSM state
    (the x_proj shares are summed as fixed-point integers, which hold no NaN: the row is
    flagged and its delta_r, B, C become NaN), and the other sequences match the oracle."""
    w = synth.configs.Workload("edge_dec_nan", DIMS_BF16_SMALL, "bf16", 3, 16, 60, 32)
    lay = H.GpuLayer(w, 0)
    pos = w.n_meta + w.n_tokens
    cap = w.n_meta + w.window
    c = {k: t.contiguous() for k, t in synth.configs.decode_caches(w, 0, cap, False, device="cuda").items()}
    kvc = hy.hymba_kv_cache(c["k"].data_ptr(), c["v"].data_ptr(), w.batch, cap, 0)
    ssm = hy.hymba_ssm_cache(c["ssm"].data_ptr(), c["conv"].data_ptr())
    dws = H.workspace(hy.hymba_layer_decode_workspace(lay.handle, w.batch, pos))
    xt = synth.gen.normal_tensor((w.batch, w.dims.d_model), 0, "edge_dec_nan/x", device="cuda").to(torch.bfloat16)
    xt[1, 7] = float("nan")
    yt = torch.empty_like(xt)
    hy.hymba_layer_decode_step(lay.handle, w.batch, pos, xt, yt, kvc, ssm, dws, dws.numel(),
                               torch.cuda.current_stream())
    hy.hymba_stream_status(torch.cuda.current_stream())
    assert torch.isnan(yt[1]).all()
    assert torch.isnan(c["ssm"][1]).any()
    for b in (0, 2):
        cache = {k: H.to64(t) for k, t in synth.configs.decode_caches(w, 0, cap, False, batch_index=b).items()}
        yo, _ = O.layer_decode(H.to64(xt[b]), pos, H.oracle_weights(lay.cpu), lay.spec, cache)
        H.close_bf16(H.to64(yt[b]), yo, f"decode y, clean sequence {b}")
    lay.close()


def test_decode_global_more_runs_than_a_warp():
    """Batch 1 on a long global layer: few (sequence, kv head, chunk) items, so every chunk
    of the store becomes its own run of the persistent decode attention (35 runs per head),
    more than one warp merges in one round."""
    w = synth.configs.Workload("edge_dec_runs", DIMS_BF16_SMALL, "bf16", 1, 128, 4300, 0)
    lay = H.GpuLayer(w, 0, is_global=True)
    pos = w.n_meta + w.n_tokens
    cap = pos + 1
    c = {k: t.contiguous() for k, t in synth.configs.decode_caches(w, 0, cap, False, device="cuda").items()}
    kvc = hy.hymba_kv_cache(c["k"].data_ptr(), c["v"].data_ptr(), 1, cap, 0)
    ssm = hy.hymba_ssm_cache(c["ssm"].data_ptr(), c["conv"].data_ptr())
    dws = H.workspace(hy.hymba_layer_decode_workspace(lay.handle, 1, pos))
    xt = synth.gen.normal_tensor((1, w.dims.d_model), 0, "edge_dec_runs/x", device="cuda").to(torch.bfloat16)
    yt = torch.empty_like(xt)
    hy.hymba_layer_decode_step(lay.handle, 1, pos, xt, yt, kvc, ssm, dws, dws.numel(),
                               torch.cuda.current_stream())
    hy.hymba_stream_status(torch.cuda.current_stream())
    cache = {k: H.to64(t) for k, t in synth.configs.decode_caches(w, 0, cap, False, batch_index=0).items()}
    yo, _ = O.layer_decode(H.to64(xt[0]), pos, H.oracle_weights(lay.cpu), lay.spec, cache)
    H.close_bf16(H.to64(yt[0]), yo, "decode y, 35 runs")
    lay.close()


@pytest.mark.parametrize("batch", [129, 200, 300])
def test_decode_batch_over_128_rows(batch):
    """More than 128 sequences: the decode projections take 256-row activation tiles."""
    w = synth.configs.Workload(f"edge_dec_b{batch}", DIMS_BF16_SMALL, "bf16", batch, 16, 40, 32)
    lay = H.GpuLayer(w, 0)
    pos = w.n_meta + w.n_tokens
    cap = w.n_meta + w.window
    c = {k: t.contiguous() for k, t in synth.configs.decode_caches(w, 0, cap, False, device="cuda").items()}
    kvc = hy.hymba_kv_cache(c["k"].data_ptr(), c["v"].data_ptr(), batch, cap, 0)
    ssm = hy.hymba_ssm_cache(c["ssm"].data_ptr(), c["conv"].data_ptr())
    dws = H.workspace(hy.hymba_layer_decode_workspace(lay.handle, batch, pos))
    xt = synth.gen.normal_tensor((batch, w.dims.d_model), 0, f"edge_dec_b{batch}/x", device="cuda").to(torch.bfloat16)
    yt = torch.empty_like(xt)
    hy.hymba_layer_decode_step(lay.handle, batch, pos, xt, yt, kvc, ssm, dws, dws.numel(),
                               torch.cuda.current_stream())
    hy.hymba_stream_status(torch.cuda.current_stream())
    for b in (0, 127, 128, batch - 1):
        cache = {k: H.to64(t) for k, t in synth.configs.decode_caches(w, 0, cap, False, batch_index=b).items()}
        yo, _ = O.layer_decode(H.to64(xt[b]), pos, H.oracle_weights(lay.cpu), lay.spec, cache)
        H.close_bf16(H.to64(yt[b]), yo, f"decode y b={b}")
    lay.close()
