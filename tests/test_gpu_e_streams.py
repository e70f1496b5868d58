"""The decode step on an explicitly created stream, directly after a kernel on that stream
that writes its input, and the same step captured in a CUDA graph and replayed (the
launch mode of the benchmark, where the library's kernels start while their predecessor
finishes and wait for its results on the device).  Both are checked against the oracle."""
from __future__ import annotations

import pytest
import torch

import hybrid_attention_ssm_head_b200 as hy
import synth
from oracle import hymba_oracle as O
from tests import _harness as H

pytestmark = pytest.mark.gpu


def _setup(kind):
    w = H.small_workload("t_stream_dec_b3_n300", batch=3, n_tokens=300, window=0 if kind == "global" else 128)
    lay = H.GpuLayer(w, 0, is_global=kind == "global")
    B, L = w.batch, w.seq_rows
    cap = L + 8 if kind == "global" else w.n_meta + w.window
    xs = synth.configs.x_tilde(w).cuda()
    k, v, kv = H.alloc_kv_seq(w, B, L)
    kc, vc, kvc = H.alloc_kv_cache(w, B, cap)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    H.run_prefill(lay, xs, kv, kvc, ssm)
    return w, lay, xs, (kc, vc, kvc), (h, conv, ssm), cap


def _oracle_decode(w, lay, xs, x_new, cap, b):
    L = w.seq_rows
    refp = O.layer_prefill(H.to64(xs[b]), H.oracle_weights(lay.cpu), lay.spec, capacity=cap)
    cache = dict(k=refp["k_cache"], v=refp["v_cache"], ssm=refp["h"], conv=refp["conv"])
    yo, _ = O.layer_decode(H.to64(x_new[b]), L, H.oracle_weights(lay.cpu), lay.spec, cache)
    return yo


@pytest.mark.parametrize("kind", ["swa", "global"])
def test_decode_on_explicit_stream_after_producer_kernel(kind):
    w, lay, xs, (kc, vc, kvc), (h, conv, ssm), cap = _setup(kind)
    B, L = w.batch, w.seq_rows
    dws = H.workspace(hy.hymba_layer_decode_workspace(lay.handle, B, L))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        base = synth.gen.normal_tensor((B, w.dims.d_model), 0, "t_stream/x", device="cuda")
        x_new = base.to(torch.bfloat16)  # the kernel right before the step writes its input
        yt = torch.empty_like(x_new)
        hy.hymba_layer_decode_step(lay.handle, B, L, x_new, yt, kvc, ssm, dws, dws.numel(), s)
    hy.hymba_stream_status(s)
    for b in range(B):
        H.close_bf16(H.to64(yt[b]), _oracle_decode(w, lay, xs, x_new, cap, b), f"{kind} decode y[b={b}]")
    lay.close()


def test_decode_graph_replay():
    w, lay, xs, (kc, vc, kvc), (h, conv, ssm), cap = _setup("swa")
    B, L = w.batch, w.seq_rows
    dws = H.workspace(hy.hymba_layer_decode_workspace(lay.handle, B, L))
    x_new = synth.gen.normal_tensor((B, w.dims.d_model), 0, "t_graph/x", device="cuda").to(torch.bfloat16)
    x_in = torch.zeros_like(x_new)
    yt = torch.empty_like(x_new)
    # the captured step advances the caches: keep a copy to restore before the replay
    saved = {n: t.clone() for n, t in (("kc", kc), ("vc", vc), ("h", h), ("conv", conv))}
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            x_in.copy_(x_new)
            hy.hymba_layer_decode_step(lay.handle, B, L, x_in, yt, kvc, ssm, dws, dws.numel(), s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for n, t in (("kc", kc), ("vc", vc), ("h", h), ("conv", conv)):
        t.copy_(saved[n])
    yt.zero_()
    g.replay()
    torch.cuda.synchronize()
    hy.hymba_stream_status(torch.cuda.current_stream())
    for b in range(B):
        H.close_bf16(H.to64(yt[b]), _oracle_decode(w, lay, xs, x_new, cap, b), f"graph decode y[b={b}]")
    del g
    lay.close()
