"""The decode step that allocates nothing (hymba_layer_decode_step_static).

Some callers cannot call cudaMalloc: their device memory is all handed out in
advance by another owner, or they run in a loop that cannot afford cudaMalloc's
device synchronisation.  For them the library keeps the decode step's scratch in
a static device buffer.  This checks, through the C ABI, that two calls in a row
of that entry point give what the workspace entry point gives on identical
caches, and that a request larger than the buffer is refused before launch.
Collected last: a failure here leaves every other test already run."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hybrid_attention_ssm_head_b200 as hy
import synth
from tests import _harness as H

pytestmark = pytest.mark.gpu


def _layer_and_caches(w, consumer_of=None):
    lay = H.GpuLayer(w, 0)
    cap = w.n_meta + w.window
    pos = w.n_meta + w.n_tokens
    c = {k: t.contiguous() for k, t in synth.configs.decode_caches(w, 0, cap, False, device="cuda").items()}
    return lay, c, cap, pos


def _structs(c, B, cap):
    return (hy.hymba_kv_cache(c["k"].data_ptr(), c["v"].data_ptr(), B, cap, 0),
            hy.hymba_ssm_cache(c["ssm"].data_ptr(), c["conv"].data_ptr()))


def test_static_scratch_decode_matches_workspace_decode():
    # the headline decode shape on a sliding-window layer: batch 128, 8k context
    w = synth.configs.CFG4
    B = w.batch
    lay, base, cap, pos = _layer_and_caches(w)
    ref = {k: v.clone() for k, v in base.items()}
    got = {k: v.clone() for k, v in base.items()}
    kv_r, ssm_r = _structs(ref, B, cap)
    kv_g, ssm_g = _structs(got, B, cap)
    stream = torch.cuda.current_stream()
    ws = H.workspace(hy.hymba_layer_decode_workspace(lay.handle, B, pos + 1))
    for step in range(2):  # two calls in a row: the buffer keeps the previous call's contents
        x = synth.gen.normal_tensor((B, w.dims.d_model), 0, f"noalloc/x{step}", device="cuda").to(torch.bfloat16)
        y_ref = torch.empty_like(x)
        y_got = torch.empty_like(x)
        hy.hymba_layer_decode_step(lay.handle, B, pos + step, x, y_ref, kv_r, ssm_r, ws, ws.numel(), stream)
        hy.hymba_layer_decode_step_static(lay.handle, B, pos + step, x, y_got, kv_g, ssm_g, stream)
        hy.hymba_stream_status(stream)
        H.close_bf16(H.to64(y_got), H.to64(y_ref), f"y_t, call {step}")
        for k in ("ssm", "conv", "k", "v"):
            H.close_bf16(H.to64(got[k]), H.to64(ref[k]), f"{k} after call {step}")
    lay.close()


def test_static_scratch_refuses_requests_beyond_its_size():
    # a global layer at batch 128 and 8k context needs far more scratch than the buffer
    w = synth.configs.CFG4
    lay = H.GpuLayer(w, 0, is_global=True)
    pos = w.n_meta + w.n_tokens
    need = hy.hymba_layer_decode_workspace(lay.handle, w.batch, pos)
    assert need > hy.HYMBA_DECODE_STATIC_SCRATCH_BYTES
    kv = hy.hymba_kv_cache(1 << 40, 1 << 40, w.batch, pos + 1, 0)
    ssm = hy.hymba_ssm_cache(1 << 40, 1 << 40)
    with pytest.raises(hy.HymbaError) as e:
        hy.hymba_layer_decode_step_static(lay.handle, w.batch, pos, 1 << 40, 1 << 40, kv, ssm)
    assert e.value.status == hy.HYMBA_ERR_WORKSPACE
    lay.close()
