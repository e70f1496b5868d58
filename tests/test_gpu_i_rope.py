"""Rotary position embedding of Q and K, fused into the input projection's epilogue
(Hymba §2.5 changes the RoPE base for the 8k extension; the five workloads have no RoPE):
prefill, a K/V-sharing consumer, the meta-cached prefill and a decode step after the
prefill, against the fp64 oracle with the same base, for both storage dtypes."""
from __future__ import annotations

from dataclasses import replace

import pytest
import torch

import hybrid_attention_ssm_head_b200 as hy
import synth
from oracle import hymba_oracle as O
from synth.configs import LayerDims, Workload
from tests import _harness as H

pytestmark = pytest.mark.gpu

DIMS_BF16 = LayerDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim_qk=64, d_inner=512)


@pytest.mark.parametrize("dtype,glob", [("bf16", False), ("bf16", True), ("f32", False)])
def test_rope_prefill_consumer_and_decode(dtype, glob):
    dims = DIMS_BF16 if dtype == "bf16" else synth.configs.DIMS_SMALL
    w = Workload(f"rope_{dtype}_{glob}", dims, dtype, 2, 16, 300, 0 if glob else 128, rope_base=10000.0)
    prod = H.GpuLayer(w, 0, is_global=glob)
    cons = H.GpuLayer(w, 1, consumer=True, is_global=glob)
    hy.hymba_kv_share_bind(cons.handle, prod.handle)
    B, L = w.batch, w.seq_rows
    cap = L + 4 if glob else w.n_meta + w.window
    x = synth.configs.x_tilde(w).cuda()
    x2 = synth.gen.normal_tensor(tuple(x.shape), 0, f"{w.name}/x2", device="cuda").to(H.torch_dt(w))
    k, v, kv = H.alloc_kv_seq(w, B, L)
    kc, vc, kvc = H.alloc_kv_cache(w, B, cap)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y1, ws = H.run_prefill(prod, x, kv, kvc, ssm)
    y2, ws = H.run_prefill(cons, x2, kv, ws=ws)
    xn = synth.gen.normal_tensor((B, dims.d_model), 0, f"{w.name}/xn", device="cuda").to(H.torch_dt(w))
    dws = H.workspace(hy.hymba_layer_decode_workspace(prod.handle, B, L))
    yt = torch.empty_like(xn)
    hy.hymba_layer_decode_step(prod.handle, B, L, xn, yt, kvc, ssm, dws, dws.numel(), torch.cuda.current_stream())
    hy.hymba_stream_status(torch.cuda.current_stream())
    wp, wc = H.oracle_weights(prod.cpu), H.oracle_weights(cons.cpu)
    for b in range(B):
        r1 = O.layer_prefill(H.to64(x[b]), wp, prod.spec, capacity=cap)
        H.close(w, H.to64(y1[b]), r1["Y"], f"producer Y b={b}")
        H.close(w, H.to64(k[b]), r1["k"], f"rotated K b={b}")
        r2 = O.layer_prefill(H.to64(x2[b]), wc, cons.spec, kv_from=r1)
        H.close(w, H.to64(y2[b]), r2["Y"], f"consumer Y b={b}")
        yo, newc = O.layer_decode(H.to64(xn[b]), L, wp, prod.spec,
                                  dict(k=r1["k_cache"], v=r1["v_cache"], ssm=r1["h"], conv=r1["conv"]))
        H.close(w, H.to64(yt[b]), yo, f"decode y b={b}")
        sl = O.kv_slot(L, prod.spec)
        H.close(w, H.to64(kc[b][:, sl]), newc["k"][:, sl], f"decode rotated K slot b={b}")
    # without the rotation the outputs differ: the embedding is really applied
    r_plain = O.layer_prefill(H.to64(x[0]), wp, replace(prod.spec, rope_base=0.0))
    assert float(abs(H.to64(y1[0]) - r_plain["Y"]).max()) > 0.05
    prod.close()
    cons.close()


def test_rope_with_meta_cache():
    w = Workload("rope_meta_bf16", DIMS_BF16, "bf16", 2, 128, 200, 128, rope_base=500.0)
    lay = H.GpuLayer(w, 0)
    B, L, m = w.batch, w.seq_rows, w.n_meta
    xt = synth.configs.x_tilde(w).cuda()
    d = w.dims
    bufs = dict(k=torch.zeros(m, d.n_kv_heads * 64, dtype=torch.bfloat16, device="cuda"),
                v=torch.zeros(m, d.n_kv_heads * 128, dtype=torch.bfloat16, device="cuda"),
                h=torch.zeros(d.d_inner, 16, dtype=torch.float32, device="cuda"),
                conv=torch.zeros(3, d.d_inner, dtype=torch.bfloat16, device="cuda"),
                y=torch.zeros(m, d.d_model, dtype=torch.bfloat16, device="cuda"))
    mc = hy.hymba_meta_cache(*[bufs[n].data_ptr() for n in ("k", "v", "h", "conv", "y")], 0)
    mws = H.workspace(hy.hymba_layer_meta_workspace(lay.handle))
    s = torch.cuda.current_stream()
    hy.hymba_layer_meta_precompute(lay.handle, xt[0, :m].contiguous(), mc, None, mws, mws.numel(), s)
    k, v, kv = H.alloc_kv_seq(w, B, L)
    xr = xt[:, m:].contiguous()
    y = torch.empty_like(xr)
    ws = H.workspace(hy.hymba_layer_prefill_cached_workspace(lay.handle, B, w.n_tokens))
    hy.hymba_layer_prefill_cached(lay.handle, B, w.n_tokens, xr, y, mc, kv, None, None, ws, ws.numel(), s)
    hy.hymba_stream_status(s)
    for b in range(B):
        r = O.layer_prefill(H.to64(xt[b]), H.oracle_weights(lay.cpu), lay.spec)
        H.close_bf16(H.to64(y[b]), r["Y"][m:], f"cached prefill with RoPE b={b}")
        H.close_bf16(H.to64(k[b]), r["k"], f"rotated K b={b}")
    lay.close()
