"""Invariances of the GPU path that hold bit for bit:
  * the meta rows are the same input for every sequence, so their outputs (and their
    K/V) are identical across the batch (Hymba §2.3: meta tokens do not depend on the
    input);
  * sequences are independent, so permuting the batch permutes every output, although
    the persistent kernels then hand each sequence's work to different CTAs in a
    different order;
  * the prefill is deterministic: the same call repeated, or two calls issued in the
    opposite order, give identical bits."""
from __future__ import annotations

import pytest
import torch

import synth
from tests import _harness as H

pytestmark = pytest.mark.gpu


def _prefill_all(lay, w, x):
    B, L = x.shape[0], x.shape[1]
    k, v, kv = H.alloc_kv_seq(w, B, L)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y, _ = H.run_prefill(lay, x, kv, None, ssm)
    return dict(y=y, k=k, v=v, h=h, conv=conv)


@pytest.mark.parametrize("dtype,glob", [("bf16", False), ("bf16", True), ("f32", False)])
def test_meta_rows_identical_across_the_batch(dtype, glob):
    w = H.small_workload(f"inv_meta_{dtype}_{glob}", dtype=dtype, batch=4, n_meta=128, n_tokens=200,
                         window=0 if glob else 64)
    lay = H.GpuLayer(w, 0, is_global=glob)
    out = _prefill_all(lay, w, synth.configs.x_tilde(w).cuda())
    m = w.n_meta
    for key in ("y", "k", "v"):
        t = out[key][:, :m]
        for b in range(1, w.batch):
            assert torch.equal(t[b], t[0]), (key, b)
    lay.close()


@pytest.mark.parametrize("glob", [False, True])
def test_batch_permutation_permutes_outputs_bitwise(glob):
    w = H.small_workload(f"inv_perm_{glob}", batch=5, n_meta=128, n_tokens=333, window=0 if glob else 256)
    lay = H.GpuLayer(w, 0, is_global=glob)
    x = synth.configs.x_tilde(w).cuda()
    perm = torch.tensor([3, 0, 4, 2, 1], device="cuda")
    a = _prefill_all(lay, w, x)
    b = _prefill_all(lay, w, x[perm].contiguous())
    for key in a:
        assert torch.equal(b[key], a[key][perm]), key
    lay.close()


def test_prefill_deterministic_across_launch_orders():
    w = H.small_workload("inv_order", batch=3, n_meta=128, n_tokens=300, window=256)
    lay = H.GpuLayer(w, 0)
    x1 = synth.configs.x_tilde(w).cuda()
    x2 = synth.gen.normal_tensor(tuple(x1.shape), 0, "inv_order/x2", device="cuda").to(torch.bfloat16)
    first = [_prefill_all(lay, w, x1), _prefill_all(lay, w, x2)]
    second = [_prefill_all(lay, w, x2), _prefill_all(lay, w, x1)]
    for key in first[0]:
        assert torch.equal(first[0][key], second[1][key]), key
        assert torch.equal(first[1][key], second[0][key]), key
    lay.close()
