"""The bounded-wait path on the GPU, without a fault or an unbounded wait: with a short
wait limit, a prefill whose output projection's MMA warp waits for an arrival that never
comes (hymba_debug_stall_next_prefill) ends on its own, hymba_stream_status reports
HYMBA_ERR_TIMEOUT, and the next normal call on the same context is correct."""
from __future__ import annotations

import pytest
import torch

import hybrid_attention_ssm_head_b200 as hy
import synth
from oracle import hymba_oracle as O
from synth.configs import LayerDims, Workload
from tests import _harness as H

pytestmark = pytest.mark.gpu

DIMS = LayerDims(d_model=256, n_heads=4, n_kv_heads=2, head_dim_qk=64, d_inner=512)


def test_stalled_wait_times_out_and_the_next_call_is_correct():
    w = Workload("timeout_bf16_b1_m16_n100_w32", DIMS, "bf16", 1, 16, 100, 32)
    lay = H.GpuLayer(w, 0)
    x = synth.configs.x_tilde(w).cuda()
    k, v, kv = H.alloc_kv_seq(w, w.batch, w.seq_rows)
    stream = torch.cuda.current_stream()
    hy.hymba_stream_status(stream)
    try:
        assert hy.hymba_set_wait_limit(2_000_000) == 2_000_000  # ~1 ms
        hy.hymba_debug_stall_next_prefill(1)
        y = torch.empty_like(x)
        ws = H.workspace(hy.hymba_layer_prefill_workspace(lay.handle, w.batch, w.n_tokens))
        hy.hymba_layer_prefill(lay.handle, w.batch, w.n_tokens, x, y, kv, None, None, ws, ws.numel(), stream)
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_stream_status(stream)
        assert e.value.status == hy.HYMBA_ERR_TIMEOUT, e.value
    finally:
        hy.hymba_debug_stall_next_prefill(0)
        hy.hymba_set_wait_limit(0)
    hy.hymba_stream_status(stream)  # the error word was cleared by the report
    y2, _ = H.run_prefill(lay, x, kv)
    ref = O.layer_prefill(H.to64(x[0]), H.oracle_weights(lay.cpu), lay.spec)
    H.close_bf16(H.to64(y2[0]), ref["Y"], "Y after the timed-out call")
    lay.close()
