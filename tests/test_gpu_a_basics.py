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


MASK_SHAPES = [
    (272, 16, 64, False), (8320, 128, 1024, False), (8320, 128, 0, True), (300, 0, 1, False),
    (257, 1, 63, False), (129, 128, 65, False), (1000, 16, 1000, False), (64, 0, 64, True),
    (385, 200, 128, False), (4224, 128, 1024, False), (700, 0, 129, False), (513, 3, 255, False)]


@pytest.mark.parametrize("path", [0, 1])
@pytest.mark.parametrize("L,m,W,g", MASK_SHAPES)
def test_mask_bitmap_bit_exact(L, m, W, g, path):
    """path 0: the tensor-core kernel's own tile enumeration, tile classes and column
    keep-masks; path 1: the fp32 kernel's per-pair predicate.  Both equal the definition."""
    words = (L + 31) // 32
    nt = (L + 127) // 128
    bits = torch.zeros(L, words, dtype=torch.int32, device="cuda")
    cls = torch.zeros(nt, nt, dtype=torch.uint8, device="cuda")
    hy.hymba_debug_mask_bitmap(L, m, W, g, bits, cls, torch.cuda.current_stream(), path=path)
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


@pytest.mark.parametrize("m,W,g", [(128, 1024, False), (16, 64, False), (0, 1, False), (3, 5, False),
                                   (128, 0, True), (1, 0, True)])
def test_decode_slot_mask_bit_exact(m, W, g):
    """The decode kernels' slot predicate against the oracle's gather of visible positions,
    for queries before the ring wraps, at the wrap and long after it."""
    Wr = max(W, 1)
    for pos in sorted({m, m + 1, m + Wr - 1, m + Wr, m + Wr + 1, m + 2 * Wr + 3, m + 8192}):
        cap = pos + 1 if g else m + Wr
        bits = torch.zeros((cap + 31) // 32, dtype=torch.int32, device="cuda")
        hy.hymba_debug_decode_mask(pos, m, Wr, g, cap, bits, torch.cuda.current_stream())
        hy.hymba_stream_status(torch.cuda.current_stream())
        s = O.Spec(d_model=1, n_heads=1, n_kv_heads=1, head_dim_qk=1, head_dim_v=1, d_inner=1,
                   d_state=1, d_conv=1, dt_rank=1, n_meta=m, window=Wr, is_global=g)
        np.testing.assert_array_equal(bits.cpu().numpy().view(np.uint32), O.decode_slot_bitmap(pos, s, cap),
                                      err_msg=f"pos {pos}")


@pytest.mark.parametrize("degree,bound", [(3, 7.5e-5), (5, 2.4e-7)])
def test_exp2_polynomial_within_its_stated_bound(degree, bound):
    """The FMA-pipe 2^x of the attention softmax against exact 2^x over the range the
    softmax feeds it ([-125, 0]: scores minus the running maximum), plus the clamp below
    -125.  Relative error <= the stated bound plus one fp32 rounding."""
    grid = np.concatenate([np.linspace(-125.0, 0.0, 1_000_003), -np.arange(0, 125.5, 0.5),
                           np.random.default_rng(0).uniform(-125, 0, 200_000), [0.0, -1e-30, -0.5, 0.5]])
    x = torch.tensor(grid.astype(np.float32), device="cuda")
    y = torch.empty_like(x)
    hy.hymba_debug_exp2_poly(degree, x, y, x.numel(), torch.cuda.current_stream())
    hy.hymba_stream_status(torch.cuda.current_stream())
    xs = x.cpu().numpy().astype(np.float64)
    want = np.exp2(xs)
    rel = np.abs(y.cpu().numpy().astype(np.float64) - want) / want
    assert rel.max() <= bound + 2 ** -23, (degree, rel.max(), xs[rel.argmax()])
    low = torch.tensor([-126.0, -200.0, -1e4], device="cuda")
    ylow = torch.empty_like(low)
    hy.hymba_debug_exp2_poly(degree, low, ylow, 3, torch.cuda.current_stream())
    np.testing.assert_allclose(ylow.cpu().numpy(), 2.0 ** -125, rtol=bound + 2 ** -23)


def test_fp32_layer_matches_oracle_stage_by_stage():
    w = synth.configs.CFG0
    lay = H.GpuLayer(w, 0)
    B, L = w.batch, w.seq_rows
    x = synth.configs.x_tilde(w).cuda()
    k, v, kv = H.alloc_kv_seq(w, B, L)
    h, conv, ssm = H.alloc_ssm_cache(w, B)
    y, ws = H.run_prefill(lay, x, kv, None, ssm)
    ref = O.layer_prefill(H.to64(x[0]), H.oracle_weights(lay.cpu), lay.spec)
    ref["gate"] = O.silu(ref["z"])
    for name, key in [("q", "q"), ("x_ssm", "x_ssm"), ("gate", "gate"), ("u", "u"), ("delta", "delta"),
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
