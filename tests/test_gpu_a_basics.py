"""First GPU checks: the generator agrees CPU/GPU bit for bit, the mask bitmap
the attention kernel evaluates equals the oracle's bit for bit, and the fp32
layer (the 256 + 16 meta-token workload) matches the oracle stage by stage."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import hybrid_attention_ssm_head_b200 as hy
import synth
from oracle import hymba_oracle as O
from tests import _harness as H

pytestmark = pytest.mark.gpu


def test_generator_bit_identical_on_gpu():
    for name in ("a", "cfg/x"):
        c = synth.gen.normal(100003, 7, name, offset=12345)
        g = synth.gen.normal(100003, 7, name, offset=12345, device="cuda").cpu()
        assert torch.equal(c, g)
        cu = synth.gen.uniform(5001, 3, name)
        gu = synth.gen.uniform(5001, 3, name, device="cuda").cpu()
        assert torch.equal(cu, gu)
    w = synth.configs.CFG1
    a = synth.configs.layer_weights(w, 0)
    b = synth.configs.layer_weights(w, 0, device="cuda")
    for k in a:
        assert torch.equal(a[k], b[k].cpu()), k


@pytest.mark.parametrize("L,m,W,g", [
    (272, 16, 64, False), (8320, 128, 1024, False), (8320, 128, 0, True), (300, 0, 1, False),
    (257, 1, 63, False), (129, 128, 65, False), (1000, 16, 1000, False), (64, 0, 64, True),
    (385, 200, 128, False)])
def test_mask_bitmap_bit_exact(L, m, W, g):
    words = (L + 31) // 32
    nt = (L + 127) // 128
    bits = torch.zeros(L, words, dtype=torch.int32, device="cuda")
    cls = torch.zeros(nt, nt, dtype=torch.uint8, device="cuda")
    hy.hymba_debug_mask_bitmap(L, m, W, g, bits, cls, torch.cuda.current_stream())
    hy.hymba_stream_status(torch.cuda.current_stream())
    got = bits.cpu().numpy().view(np.uint32)
    want = O.mask_bitmap(L, m, max(W, 1), g)
    np.testing.assert_array_equal(got, want)
    # tile classes: a skipped tile holds no visible pair, a full tile no masked pair
    mm = O.mask_matrix(L, m, max(W, 1), g)
    cl = cls.cpu().numpy()
    for qt in range(nt):
        for kt in range(nt):
            blk = mm[qt * 128:(qt + 1) * 128, kt * 128:(kt + 1) * 128]
            if cl[qt, kt] == 0:
                assert not blk.any(), (qt, kt)
            elif cl[qt, kt] == 1:
                assert blk.all() and (kt + 1) * 128 <= L, (qt, kt)
            else:
                assert cl[qt, kt] == 2


def test_fp32_layer_matches_oracle_stage_by_stage():
    w = synth.configs.CFG0
    lay = H.GpuLayer(w, 0)
    B, L = w.batch, w.seq_rows
    x = synth.configs.x_tilde(w).cuda()
    k, v, kv = H.alloc_kv_seq(w, B, L)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y, ws = H.run_prefill(lay, x, kv, None, ssm)
    ref = O.layer_prefill(H.to64(x[0]), H.oracle_weights(lay.cpu), lay.spec)
    for name, key in [("q", "q"), ("x_ssm", "x_ssm"), ("z", "z"), ("u", "u"), ("delta", "delta"),
                      ("y_ssm", "y_ssm"), ("o_attn", "o"), ("fused", "f")]:
        H.close_f32(H.to64(H.stage(lay, ws, B, L, name)[0]), ref[key], name)
    H.close_f32(H.to64(k[0]), ref["k"], "k")
    H.close_f32(H.to64(v[0]), ref["v"], "v")
    xd = H.to64(H.stage(lay, ws, B, L, "xdbl")[0])
    R = lay.spec.dt_rank
    H.close_f32(xd[:, R:R + 16], ref["B"], "B")
    H.close_f32(xd[:, R + 16:], ref["C"], "C")
    H.close_f32(H.to64(y[0]), ref["Y"], "Y")
    H.close_f32(H.to64(h[0]), ref["h"], "h_final")
    np.testing.assert_allclose(H.to64(conv[0]), ref["conv"], rtol=1e-5, atol=1e-6)
    lay.close()
