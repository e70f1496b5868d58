"""The two branches side by side (Hymba Fig. 1 and §2.1: the attention and SSM heads read
the same input in parallel; the OpenReview reply on speed proposes two CUDA streams).
With branch_chunks >= 2 the prefill splits the batch into chunks and runs each chunk's
selective scan on the handle's side stream beside the next chunk's projections and
attention.  Every kernel computes each sequence the same way in either schedule, so the
concurrent prefill must reproduce the serial one bit for bit: outputs, K/V, the decode
stores and the SSM state, for even and ragged chunkings, a K/V-sharing consumer, the
meta-cache prefill and the block; and the result must not depend on how the side stream
and the caller's stream happen to interleave (repeated calls)."""
from __future__ import annotations

import pytest
import torch

import hybrid_attention_ssm_head_b200 as hy
import synth
from synth.configs import LayerDims, Workload
from tests import _harness as H

pytestmark = pytest.mark.gpu

DIMS_SMALL_BF16 = LayerDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim_qk=64, d_inner=512)


def _prefill(lay, w, x, glob):
    B, L = x.shape[0], x.shape[1]
    k, v, kv = H.alloc_kv_seq(w, B, L)
    cap = L + 2 if glob else w.n_meta + w.window
    kc, vc, kvc = H.alloc_kv_cache(w, B, cap)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y, _ = H.run_prefill(lay, x, kv, kvc, ssm)
    return dict(y=y, k=k, v=v, kc=kc, vc=vc, h=h, conv=conv), kv


def _equal(a, b, what):
    for key in a:
        assert torch.equal(a[key], b[key]), f"{what}: {key} differs"


@pytest.mark.parametrize("dtype,batch,chunks,glob", [
    ("bf16", 5, 2, False), ("bf16", 5, 4, False), ("bf16", 5, 8, False), ("bf16", 4, 4, True),
    ("bf16", 3, 2, False), ("f32", 5, 3, False)])
def test_concurrent_prefill_equals_serial_bitwise(dtype, batch, chunks, glob):
    dims = DIMS_SMALL_BF16 if dtype == "bf16" else synth.configs.DIMS_SMALL
    w = Workload(f"branch_{dtype}_{batch}_{chunks}_{glob}", dims, dtype, batch, 128, 333,
                 0 if glob else 128)
    x = synth.configs.x_tilde(w).cuda()
    ser_p = H.GpuLayer(w, 0, is_global=glob, branch_chunks=0)
    ser_c = H.GpuLayer(w, 1, consumer=True, is_global=glob, branch_chunks=0)
    con_p = H.GpuLayer(w, 0, is_global=glob, branch_chunks=chunks)
    con_c = H.GpuLayer(w, 1, consumer=True, is_global=glob, branch_chunks=chunks)
    hy.hymba_kv_share_bind(ser_c.handle, ser_p.handle)
    hy.hymba_kv_share_bind(con_c.handle, con_p.handle)
    a, kva = _prefill(ser_p, w, x, glob)
    b, kvb = _prefill(con_p, w, x, glob)
    _equal(a, b, "producer")
    # the consumer reads its producer's K/V in place
    B, L = x.shape[0], x.shape[1]
    ya, _ = H.run_prefill(ser_c, a["y"], kva)
    yb, _ = H.run_prefill(con_c, b["y"], kvb)
    assert torch.equal(ya, yb), "consumer output differs"
    for lay in (ser_p, ser_c, con_p, con_c):
        lay.close()


def test_concurrent_prefill_repeatable():
    w = H.small_workload("branch_repeat", batch=8, n_meta=128, n_tokens=500, window=256)
    x = synth.configs.x_tilde(w).cuda()
    lay = H.GpuLayer(w, 0, branch_chunks=4)
    first, _ = _prefill(lay, w, x, False)
    for _ in range(3):
        again, _ = _prefill(lay, w, x, False)
        _equal(first, again, "repeat")
    ser = H.GpuLayer(w, 0, branch_chunks=1)
    s, _ = _prefill(ser, w, x, False)
    _equal(s, first, "serial vs concurrent")
    lay.close()
    ser.close()


def test_concurrent_cached_prefill_equals_serial():
    w = Workload("branch_meta", DIMS_SMALL_BF16, "bf16", 6, 128, 300, 128)
    xt = synth.configs.x_tilde(w).cuda()
    m = w.n_meta
    x_meta, x_real = xt[0, :m].contiguous(), xt[:, m:].contiguous()
    outs = []
    for chunks in (0, 3):
        lay = H.GpuLayer(w, 0, branch_chunks=chunks)
        d = w.dims
        dt = H.torch_dt(w)
        bufs = dict(k=torch.zeros(m, d.n_kv_heads * d.head_dim_qk, dtype=dt, device="cuda"),
                    v=torch.zeros(m, d.n_kv_heads * d.head_dim_v, dtype=dt, device="cuda"),
                    h=torch.zeros(d.d_inner, d.d_state, dtype=torch.float32, device="cuda"),
                    conv=torch.zeros(d.d_conv - 1, d.d_inner, dtype=dt, device="cuda"),
                    y=torch.zeros(m, d.d_model, dtype=dt, device="cuda"))
        mc = hy.hymba_meta_cache(bufs["k"].data_ptr(), bufs["v"].data_ptr(), bufs["h"].data_ptr(),
                                 bufs["conv"].data_ptr(), bufs["y"].data_ptr(), 0)
        ws = H.workspace(hy.hymba_layer_meta_workspace(lay.handle))
        hy.hymba_layer_meta_precompute(lay.handle, x_meta, mc, None, ws, ws.numel(), torch.cuda.current_stream())
        B, n = x_real.shape[0], x_real.shape[1]
        k, v, kv = H.alloc_kv_seq(w, B, w.seq_rows)
        h, conv, ssm = H.alloc_ssm_cache(w, B)
        y = torch.empty_like(x_real)
        ws = H.workspace(hy.hymba_layer_prefill_cached_workspace(lay.handle, B, n))
        hy.hymba_layer_prefill_cached(lay.handle, B, n, x_real, y, mc, kv, None, ssm, ws, ws.numel(),
                                      torch.cuda.current_stream())
        hy.hymba_stream_status(torch.cuda.current_stream())
        outs.append(dict(y=y, k=k, v=v, h=h, conv=conv))
        lay.close()
    _equal(outs[0], outs[1], "cached prefill")


def test_concurrent_prefill_captured_in_a_graph():
    """The fork to the side stream and the joins are recorded by stream capture: replaying
    the graph gives the eager result."""
    w = H.small_workload("branch_graph", batch=4, n_meta=128, n_tokens=300, window=128)
    x = synth.configs.x_tilde(w).cuda()
    lay = H.GpuLayer(w, 0, branch_chunks=4)
    eager, _ = _prefill(lay, w, x, False)
    B, L = x.shape[0], x.shape[1]
    k, v, kv = H.alloc_kv_seq(w, B, L)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y = torch.empty_like(x)
    ws = H.workspace(hy.hymba_layer_prefill_workspace(lay.handle, B, L - w.n_meta))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        hy.hymba_layer_prefill(lay.handle, B, L - w.n_meta, x, y, kv, None, ssm, ws, ws.numel(), s)
    g.replay()
    torch.cuda.synchronize()
    hy.hymba_stream_status(torch.cuda.current_stream())
    assert torch.equal(y, eager["y"])
    assert torch.equal(k, eager["k"]) and torch.equal(v, eager["v"])
    assert torch.equal(h, eager["h"]) and torch.equal(conv, eager["conv"])
    del g
    lay.close()


@pytest.mark.parametrize("glob", [False, True])
def test_decode_side_by_side_equals_serial_bitwise(glob):
    """With a side stream the decode step runs its SSM branch there, beside the attention:
    the same kernels on the same inputs, so the same bits as the serial order."""
    w = Workload(f"branch_dec_{glob}", DIMS_SMALL_BF16, "bf16", 6, 128, 200, 0 if glob else 64)
    d = w.dims
    pos = w.seq_rows
    cap = pos + 4 if glob else w.n_meta + w.window
    x_new = synth.gen.normal_tensor((w.batch, d.d_model), 0, f"{w.name}/xnew", device="cuda").to(torch.bfloat16)
    outs = []
    for chunks in (0, 4):
        lay = H.GpuLayer(w, 0, is_global=glob, branch_chunks=chunks)
        c = {k: v.cuda().contiguous() for k, v in synth.configs.decode_caches(w, 0, cap, False).items()}
        kvc = hy.hymba_kv_cache(c["k"].data_ptr(), c["v"].data_ptr(), w.batch, cap, 0)
        ssm = hy.hymba_ssm_cache(c["ssm"].data_ptr(), c["conv"].data_ptr())
        ws = H.workspace(hy.hymba_layer_decode_workspace(lay.handle, w.batch, pos))
        ys = []
        for step in range(3):  # three tokens: the caches carry each step into the next
            y = torch.empty_like(x_new)
            hy.hymba_layer_decode_step(lay.handle, w.batch, pos + step, x_new, y, kvc, ssm, ws, ws.numel(),
                                       torch.cuda.current_stream())
            ys.append(y)
        hy.hymba_stream_status(torch.cuda.current_stream())
        outs.append(dict(y=torch.stack(ys), k=c["k"], v=c["v"], h=c["ssm"], conv=c["conv"]))
        lay.close()
    _equal(outs[0], outs[1], "decode")
