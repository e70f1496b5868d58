"""The seeded generator: determinism, slice independence, moments, and the stack layout."""
import numpy as np
import torch

import synth
from synth import gen


def test_deterministic_and_sliceable():
    a = gen.normal(1000, 0, "s")
    b = gen.normal(1000, 0, "s")
    assert torch.equal(a, b)
    part = gen.normal(300, 0, "s", offset=500)
    assert torch.equal(part, a[500:800])
    assert not torch.equal(gen.normal(1000, 1, "s"), a)
    assert not torch.equal(gen.normal(1000, 0, "t"), a)
    u = gen.uniform(1000, 3, "u")
    assert torch.equal(gen.uniform(10, 3, "u", offset=990), u[990:])
    # chunking does not change values
    assert torch.equal(gen.normal(1000, 0, "s", chunk=77), a)


def test_moments():
    v = gen.normal(1 << 20, 0, "m").double()
    assert abs(v.mean().item()) < 5e-3 and abs(v.std().item() - 1.0) < 5e-3
    assert v.abs().max().item() <= 6.0
    u = gen.uniform(1 << 20, 0, "m").double()
    assert 0.0 <= u.min().item() and u.max().item() < 1.0 and abs(u.mean().item() - 0.5) < 2e-3
    # every value is an exact multiple of 2^-16 (normal) / 2^-24 (uniform)
    assert torch.equal(torch.round(v * 65536) / 65536, v)


def test_batch_row_slice_matches_full_tensor():
    w = synth.configs.CFG0
    full = synth.configs.real_rows(w)
    assert torch.equal(synth.configs.real_rows(w, 0), full[0])
    xt = synth.configs.x_tilde(w)
    assert xt.shape == (w.batch, w.seq_rows, w.dims.d_model)
    assert torch.equal(xt[0, : w.n_meta], synth.configs.meta_tokens(w))


def test_stack_layout_of_the_32_layer_stack():
    lay = synth.configs.stack_layout()
    assert [i for i, (g, _) in enumerate(lay) if g] == [0, 15, 31]
    producers = [i for i, (g, p) in enumerate(lay) if not g and p is None]
    consumers = {i: p for i, (g, p) in enumerate(lay) if p is not None}
    assert len(producers) == 15
    assert all(p == i - 1 and p in producers for i, p in consumers.items())
    assert 30 in producers and 30 not in consumers.values()
