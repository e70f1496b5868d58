"""Prefill from a precomputed meta-token cache (Hymba §2.3: the meta rows are the same
for every input, so their K/V, SSM state and conv history are computed once, at batch 1,
and every prefill starts from them).  Against the fp64 oracle's prefill of the whole
X~ = [R; X]: the cached prefill's outputs for the real rows, the meta rows' outputs in the
cache, the states it returns, and a decode step after it; for a K/V owner, a consumer
bound to it, and a global layer; meta counts on and off the 128-row tile grid."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hybrid_attention_ssm_head_b200 as hy
import synth
from oracle import hymba_oracle as O
from synth.configs import LayerDims, Workload
from tests import _bounds as BD
from tests import _harness as H

pytestmark = pytest.mark.gpu

DIMS_SMALL_BF16 = LayerDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim_qk=64, d_inner=512)


def _meta_cache(lay, w, x_meta, producer_meta=None):
    d, m = w.dims, w.n_meta
    dt = H.torch_dt(w)
    bufs = dict(
        k=torch.zeros(m, d.n_kv_heads * d.head_dim_qk, dtype=dt, device="cuda"),
        v=torch.zeros(m, d.n_kv_heads * d.head_dim_v, dtype=dt, device="cuda"),
        h=torch.zeros(d.d_inner, d.d_state, dtype=torch.float32, device="cuda"),
        conv=torch.zeros(d.d_conv - 1, d.d_inner, dtype=dt, device="cuda"),
        y=torch.zeros(m, d.d_model, dtype=dt, device="cuda"))
    consumer = producer_meta is not None
    mc = hy.hymba_meta_cache(None if consumer else bufs["k"].data_ptr(),
                             None if consumer else bufs["v"].data_ptr(),
                             bufs["h"].data_ptr(), bufs["conv"].data_ptr(), bufs["y"].data_ptr(), 0)
    ws = H.workspace(hy.hymba_layer_meta_workspace(lay.handle))
    hy.hymba_layer_meta_precompute(lay.handle, x_meta, mc, producer_meta, ws, ws.numel(),
                                   torch.cuda.current_stream())
    return mc, bufs


def _cached_prefill(lay, w, x_real, mc, kv, kv_cache=None, ssm=None):
    B, n = x_real.shape[0], x_real.shape[1]
    y = torch.empty_like(x_real)
    ws = H.workspace(hy.hymba_layer_prefill_cached_workspace(lay.handle, B, n))
    hy.hymba_layer_prefill_cached(lay.handle, B, n, x_real, y, mc, kv, kv_cache, ssm, ws, ws.numel(),
                                  torch.cuda.current_stream())
    hy.hymba_stream_status(torch.cuda.current_stream())
    return y


@pytest.mark.parametrize("dtype,m,n,W,glob", [
    ("bf16", 128, 300, 256, False), ("bf16", 16, 250, 64, False), ("bf16", 130, 129, 129, False),
    ("bf16", 128, 200, 0, True), ("f32", 16, 100, 32, False)])
def test_cached_prefill_equals_full_prefill(dtype, m, n, W, glob):
    dims = DIMS_SMALL_BF16 if dtype == "bf16" else synth.configs.DIMS_SMALL
    w = Workload(f"meta_{dtype}_m{m}_n{n}_w{W}", dims, dtype, 3, m, n, W)
    prod = H.GpuLayer(w, 0, is_global=glob)
    cons = H.GpuLayer(w, 1, consumer=True, is_global=glob)
    hy.hymba_kv_share_bind(cons.handle, prod.handle)
    B, L = w.batch, w.seq_rows
    xt = synth.configs.x_tilde(w).cuda()
    x_meta = xt[0, :m].contiguous()
    x_real = xt[:, m:].contiguous()
    mp, bp = _meta_cache(prod, w, x_meta)
    mc, bc = _meta_cache(cons, w, bp["y"], producer_meta=mp)
    cap = L + 4 if glob else m + w.window
    k, v, kv = H.alloc_kv_seq(w, B, L)
    kc, vc, kvc = H.alloc_kv_cache(w, B, cap)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y1 = _cached_prefill(prod, w, x_real, mp, kv, kvc, ssm)
    h2, conv2, ssm2 = H.alloc_ssm_cache(w, B)
    y2 = _cached_prefill(cons, w, y1, mc, kv, None, ssm2)
    # a decode step of the producer after the cached prefill
    x_new = synth.gen.normal_tensor((B, dims.d_model), 0, f"{w.name}/xnew", device="cuda").to(H.torch_dt(w))
    dws = H.workspace(hy.hymba_layer_decode_workspace(prod.handle, B, L))
    yt = torch.empty_like(x_new)
    hy.hymba_layer_decode_step(prod.handle, B, L, x_new, yt, kvc, ssm, dws, dws.numel(),
                               torch.cuda.current_stream())
    hy.hymba_stream_status(torch.cuda.current_stream())
    wp, wc = H.oracle_weights(prod.cpu), H.oracle_weights(cons.cpu)
    for b in range(B):
        ref1 = O.layer_prefill(H.to64(xt[b]), wp, prod.spec, capacity=cap)
        H.close(w, H.to64(y1[b]), ref1["Y"][m:], f"producer real rows b={b}")
        # the consumer chains the producer's outputs: its oracle input is the oracle's own
        x2 = np.concatenate([ref1["Y"][:m], ref1["Y"][m:]], 0)
        ref2 = O.layer_prefill(x2, wc, cons.spec, kv_from=ref1)
        if dtype == "f32":
            H.close_f32(H.to64(y2[b]), ref2["Y"][m:], f"consumer real rows b={b}")
        else:
            H.close_chain2(H.to64(y2[b]), ref2["Y"][m:], f"consumer real rows b={b}")
        # K/V rows of the sequence: the meta rows copied from the cache, the real rows written
        H.close(w, H.to64(k[b]), ref1["k"], f"K b={b}")
        H.close(w, H.to64(v[b]), ref1["v"], f"V b={b}")
        if b == 0:
            H.close(w, H.to64(bp["y"]), ref1["Y"][:m], "producer meta outputs")
            H.close(w, H.to64(bp["k"]), ref1["k"][:m], "meta K")
            if dtype == "f32":
                H.close_f32(H.to64(bc["y"]), ref2["Y"][:m], "consumer meta outputs")
            else:
                H.close_chain2(H.to64(bc["y"]), ref2["Y"][:m], "consumer meta outputs")
        cache = dict(k=ref1["k_cache"], v=ref1["v_cache"], ssm=ref1["h"], conv=ref1["conv"])
        if dtype == "f32":
            continue
        mag = BD.ssm_magnitudes(wp, prod.spec, ref1)
        yo, newc = O.layer_decode(H.to64(x_new[b]), L, wp, prod.spec, cache)
        H.close_bf16(H.to64(yt[b]), yo, f"decode after cached prefill b={b}")
    # the returned state before the decode step moved it: checked through the decode output;
    # the meta cache's own state against the oracle's state after the meta rows
    refm = O.layer_prefill(H.to64(xt[0, :m]), wp, prod.spec)
    if dtype == "bf16":
        magm = BD.ssm_magnitudes(wp, prod.spec, refm)
        BD.close_mag(H.to64(bp["h"]), refm["h"], magm["h"], "meta cache h")
        H.close_bf16(H.to64(bp["conv"]), refm["conv"], "meta cache conv")
    else:
        H.close_f32(H.to64(bp["h"]), refm["h"], "meta cache h")
    prod.close()
    cons.close()


def test_cached_prefill_rejects_a_foreign_meta_cache():
    w = Workload("meta_reject", DIMS_SMALL_BF16, "bf16", 2, 16, 50, 32)
    a, b = H.GpuLayer(w, 0), H.GpuLayer(w, 1)
    xt = synth.configs.x_tilde(w).cuda()
    ma, _ = _meta_cache(a, w, xt[0, :16].contiguous())
    k, v, kv = H.alloc_kv_seq(w, 2, w.seq_rows)
    with pytest.raises(hy.HymbaError) as e:
        _cached_prefill(b, w, xt[:, 16:].contiguous(), ma, kv)
    assert e.value.status == hy.HYMBA_ERR_NOT_BOUND
    a.close()
    b.close()
