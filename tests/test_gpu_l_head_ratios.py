"""GQA group sizes other than the benchmark's 5 (Hymba Appendix E Table 11 groups query
heads over shared K/V heads; §2.1 Eq. 1 per head): the tensor-core prefill attention
and the decode attention, whose accumulator columns are the query heads of one group
(up to 8), against the oracle for groups of 1, 3, 7 and 8 heads.  Prefill, then one
decode step from the emitted caches, with the context past the window (ring wrapped)."""
from __future__ import annotations

import pytest
import torch

import hybrid_attention_ssm_head_b200 as hy
import synth
from oracle import hymba_oracle as O
from synth.configs import LayerDims
from tests import _harness as H

pytestmark = pytest.mark.gpu

# bf16 tensor-core kernels take d_qk 64 and d_v 128, so d_inner = 128 * n_heads
RATIOS = [(2, 2), (6, 2), (7, 1), (8, 1)]


@pytest.mark.parametrize("n_heads,n_kv_heads", RATIOS)
def test_head_groups_prefill_and_decode(n_heads, n_kv_heads):
    dims = LayerDims(d_model=256, n_heads=n_heads, n_kv_heads=n_kv_heads, head_dim_qk=64,
                     d_inner=128 * n_heads)
    B, m, n, W = 2, 16, 150, 64
    w = synth.configs.Workload(f"groups_{n_heads}_{n_kv_heads}", dims, "bf16", B, m, n, W)
    lay = H.GpuLayer(w, 0)
    L = w.seq_rows
    cap = m + W
    x = synth.configs.x_tilde(w).cuda()
    k, v, kv = H.alloc_kv_seq(w, B, L)
    kc, vc, kvc = H.alloc_kv_cache(w, B, cap)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y, _ = H.run_prefill(lay, x, kv, kvc, ssm)
    xt = synth.gen.normal_tensor((B, dims.d_model), 0, f"groups/{n_heads}/{n_kv_heads}", device="cuda").to(
        torch.bfloat16)
    dws = H.workspace(hy.hymba_layer_decode_workspace(lay.handle, B, L))
    yt = torch.empty_like(xt)
    hy.hymba_layer_decode_step(lay.handle, B, L, xt, yt, kvc, ssm, dws, dws.numel(),
                               torch.cuda.current_stream())
    hy.hymba_stream_status(torch.cuda.current_stream())
    for b in range(B):
        refp = O.layer_prefill(H.to64(x[b]), H.oracle_weights(lay.cpu), lay.spec, capacity=cap)
        H.close(w, H.to64(y[b]), refp["Y"], f"Y[b={b}] groups {n_heads}/{n_kv_heads}")
        yo, _ = O.layer_decode(H.to64(xt[b]), L, H.oracle_weights(lay.cpu), lay.spec,
                               dict(k=refp["k_cache"], v=refp["v_cache"], ssm=refp["h"],
                                    conv=refp["conv"]))
        H.close(w, H.to64(yt[b]), yo, f"decode y[b={b}] groups {n_heads}/{n_kv_heads}")
    lay.close()
