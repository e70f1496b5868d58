"""The C-ABI library: it loads, exports every function include/hymba.h declares,
and rejects bad arguments on the host before touching a device (CPU only)."""
from __future__ import annotations

import ctypes as C
import os
import re

import pytest

import hybrid_attention_ssm_head_b200 as hy

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "hymba.h")).read()
    return sorted(set(re.findall(r"HYMBA_API\s+[\w\s\*]*?\b(hymba_\w+)\s*\(", src)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = hy.lib()
    declared = _declared_functions()
    assert len(declared) >= 14
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(hy.EXPORTED) == declared
    assert "sm_100a" in hy.hymba_version()


def _cfg(**kw):
    base = dict(d_model=1600, n_heads=25, n_kv_heads=5, head_dim_qk=64, d_inner=3200, d_state=16,
                d_conv=4, dt_rank=100, n_meta=128, window=1024, is_global=False, dtype="bf16")
    base.update(kw)
    return hy.make_config(**base)


def _fake_weights(addr=1 << 40):
    # aligned, non-null fake device addresses: creation never dereferences them
    return hy.hymba_layer_weights(*[addr + 4096 * i for i in range(11)])


def test_create_validates_configuration():
    h = hy.hymba_layer_create(_cfg(), _fake_weights())
    assert h and not hy.hymba_layer_is_consumer(h)
    hy.hymba_layer_destroy(h)
    bad = [
        (dict(n_kv_heads=4), hy.HYMBA_ERR_INVALID_ARG),        # 25 % 4 != 0
        (dict(d_state=8), hy.HYMBA_ERR_UNSUPPORTED),
        (dict(dt_rank=101), hy.HYMBA_ERR_UNSUPPORTED),
        (dict(window=0), hy.HYMBA_ERR_INVALID_ARG),
        (dict(head_dim_qk=32), hy.HYMBA_ERR_UNSUPPORTED),     # bf16 attention kernel shape
        (dict(d_conv=5), hy.HYMBA_ERR_UNSUPPORTED),
        (dict(branch_chunks=-1), hy.HYMBA_ERR_INVALID_ARG),
        (dict(branch_chunks=9), hy.HYMBA_ERR_INVALID_ARG),
    ]
    for kw, want in bad:
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_create(_cfg(**kw), _fake_weights())
        assert e.value.status == want, (kw, e.value)
    cfg = _cfg()
    cfg.head_dim_v = 64  # branch widths differ: Eq. 3 cannot add them
    with pytest.raises(hy.HymbaError) as e:
        hy.hymba_layer_create(cfg, _fake_weights())
    assert e.value.status == hy.HYMBA_ERR_INVALID_ARG
    w = _fake_weights()
    w.w_out = None
    with pytest.raises(hy.HymbaError):
        hy.hymba_layer_create(_cfg(), w)
    w = _fake_weights()
    w.w_x = (1 << 40) + 8  # misaligned
    with pytest.raises(hy.HymbaError):
        hy.hymba_layer_create(_cfg(), w)


def test_kv_share_bind_checks_compatibility():
    p = hy.hymba_layer_create(_cfg(), _fake_weights())
    c = hy.hymba_layer_create(_cfg(), _fake_weights(1 << 41))
    other = hy.hymba_layer_create(_cfg(window=512), _fake_weights(1 << 42))
    glob = hy.hymba_layer_create(_cfg(is_global=True), _fake_weights(1 << 43))
    try:
        for prod in (other, glob, c):
            with pytest.raises(hy.HymbaError) as e:
                hy.hymba_kv_share_bind(c, prod)
            assert e.value.status == hy.HYMBA_ERR_NOT_BOUND
        hy.hymba_kv_share_bind(c, p)
        assert hy.hymba_layer_is_consumer(c)
        with pytest.raises(hy.HymbaError) as e:  # a consumer cannot produce
            hy.hymba_kv_share_bind(other, c)
        assert e.value.status == hy.HYMBA_ERR_NOT_BOUND
    finally:
        for h in (p, c, other, glob):
            hy.hymba_layer_destroy(h)


def test_prefill_rejects_bad_arguments_before_launch():
    p = hy.hymba_layer_create(_cfg(), _fake_weights())
    c = hy.hymba_layer_create(_cfg(), _fake_weights(1 << 41))
    hy.hymba_kv_share_bind(c, p)
    A = 1 << 44
    B, n = 2, 300
    ws = hy.hymba_layer_prefill_workspace(p, B, n)
    lay = hy.hymba_layer_prefill_layout(p, B, n)
    assert lay.total == ws and lay.q == 0
    offs = [lay.q, lay.x_ssm, lay.gate, lay.u, lay.xdbl, lay.delta, lay.y_ssm, lay.o_attn, lay.fused]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    M = B * (128 + n)
    assert lay.x_ssm - lay.q >= M * 1600 * 2 and lay.delta - lay.xdbl >= M * 132 * 4
    kv = hy.hymba_kv_seq(A, A + (1 << 30), 0, 0, 0)
    try:
        # workspace too small
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_prefill(p, B, n, A, A, kv, None, None, A, ws - 256)
        assert e.value.status == hy.HYMBA_ERR_WORKSPACE
        # consumer before its producer wrote the K/V
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_prefill(c, B, n, A, A, kv, None, None, A, ws)
        assert e.value.status == hy.HYMBA_ERR_NOT_BOUND
        # a stamp from another layer is refused too
        kv.owner, kv.batch, kv.rows = 987654, B, 128 + n
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_prefill(c, B, n, A, A, kv, None, None, A, ws)
        assert e.value.status == hy.HYMBA_ERR_NOT_BOUND
        # misaligned input, null kv, bad batch, small decode store
        for args in [(p, B, n, A + 2, A, kv, None, None, A, ws),
                     (p, 0, n, A, A, kv, None, None, A, ws)]:
            with pytest.raises(hy.HymbaError) as e:
                hy.hymba_layer_prefill(*args)
            assert e.value.status == hy.HYMBA_ERR_INVALID_ARG
        small = hy.hymba_kv_cache(A, A, B, 128 + 1023, 0)
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_prefill(p, B, n, A, A, kv, small, None, A, ws)
        assert e.value.status == hy.HYMBA_ERR_INVALID_ARG
    finally:
        hy.hymba_layer_destroy(p)
        hy.hymba_layer_destroy(c)


def test_decode_rejects_bad_arguments_before_launch():
    p = hy.hymba_layer_create(_cfg(), _fake_weights())
    c = hy.hymba_layer_create(_cfg(), _fake_weights(1 << 41))
    hy.hymba_kv_share_bind(c, p)
    A = 1 << 44
    ws = hy.hymba_layer_decode_workspace(p, 4, 2000)
    kvc = hy.hymba_kv_cache(A, A, 4, 128 + 1024, 0)
    ssm = hy.hymba_ssm_cache(A, A)
    try:
        with pytest.raises(hy.HymbaError) as e:  # meta position
            hy.hymba_layer_decode_step(p, 4, 5, A, A, kvc, ssm, A, ws)
        assert e.value.status == hy.HYMBA_ERR_INVALID_ARG
        with pytest.raises(hy.HymbaError) as e:  # consumer with an unstamped store
            hy.hymba_layer_decode_step(c, 4, 2000, A, A, kvc, ssm, A, ws)
        assert e.value.status == hy.HYMBA_ERR_NOT_BOUND
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_decode_step(p, 4, 2000, A, A, kvc, ssm, A, 64)
        assert e.value.status == hy.HYMBA_ERR_WORKSPACE
        kvc.capacity = 100
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_decode_step(p, 4, 2000, A, A, kvc, ssm, A, ws)
        assert e.value.status == hy.HYMBA_ERR_INVALID_ARG
    finally:
        hy.hymba_layer_destroy(p)
        hy.hymba_layer_destroy(c)


def test_mask_bitmap_rejects_bad_shape():
    with pytest.raises(hy.HymbaError):
        hy.hymba_debug_mask_bitmap(0, 0, 4, False, 1 << 44)
    with pytest.raises(hy.HymbaError):
        hy.hymba_debug_mask_bitmap(10, 0, 0, False, 1 << 44)


def _c_kind(decl: str) -> str:
    decl = decl.strip()
    if "*" in decl or decl.startswith("hymba_stream_t"):
        return "ptr"
    if decl.startswith("int64_t"):
        return "i64"
    if decl.startswith("size_t"):
        return "size"
    if decl.startswith("int") or decl.startswith("hymba_status"):
        return "int"
    raise AssertionError(f"unclassified parameter {decl!r}")


def _ctypes_kind(t) -> str:
    import ctypes as C
    if t in (C.c_void_p, C.c_char_p) or (isinstance(t, type) and issubclass(t, C._Pointer)):
        return "ptr"
    if t is C.c_int64:
        return "i64"
    if t is C.c_size_t:
        return "size"
    if t is C.c_int:
        return "int"
    raise AssertionError(f"unclassified ctypes type {t!r}")


def test_binding_signatures_match_the_header():
    """Every declaration's parameter list (count and kind: pointer, int, int64, size_t) and
    return kind agree with the argument types the binding gives ctypes."""
    import ctypes as C
    from hybrid_attention_ssm_head_b200 import _abi
    src = open(os.path.join(ROOT, "include", "hymba.h")).read()
    decls = re.findall(r"HYMBA_API\s+([\w\s\*]+?)\b(hymba_\w+)\s*\(([^)]*)\)\s*;", src)
    assert len(decls) == len(_abi._SIGS)
    for ret, name, params in decls:
        res, args = _abi._SIGS[name]
        plist = [p for p in params.split(",") if p.strip() and p.strip() != "void"]
        assert [_c_kind(p) for p in plist] == [_ctypes_kind(a) for a in args], name
        ret = ret.strip()
        want = {"hymba_status": C.c_int, "int": C.c_int, "void": None, "const char *": C.c_char_p}[ret]
        assert res is want, name


@pytest.mark.parametrize("kw", [
    dict(),
    dict(dtype="f32"),
    dict(is_global=True),
    dict(d_model=256, n_heads=4, n_kv_heads=2, d_inner=512, dt_rank=16, n_meta=16, window=64),
    dict(d_model=256, n_heads=4, n_kv_heads=2, d_inner=512, dt_rank=16, n_meta=0, window=64, dtype="f32"),
])
def test_prefill_workspace_holds_every_documented_intermediate(kw):
    """The workspace layout gives each intermediate the [M, width] extent the header documents,
    256-byte aligned and in order without overlap, for producers and consumers of either dtype;
    an empty sequence is refused."""
    cfg = _cfg(**kw)
    es = 4 if kw.get("dtype") == "f32" else 2
    E, N, R = cfg.d_inner, cfg.d_state, cfg.dt_rank
    for consumer in (False, True):
        h = hy.hymba_layer_create(cfg, _fake_weights())
        prod = hy.hymba_layer_create(cfg, _fake_weights(1 << 41)) if consumer else None
        if consumer:
            hy.hymba_kv_share_bind(h, prod)
        for B, n in [(1, 1), (3, 127), (2, 300), (128, 8192)]:
            if cfg.n_meta + n < 1:
                continue
            M = B * (cfg.n_meta + n)
            lay = hy.hymba_layer_prefill_layout(h, B, n)
            assert lay.total == hy.hymba_layer_prefill_workspace(h, B, n)
            regions = [(lay.q, M * cfg.n_heads * cfg.head_dim_qk * es), (lay.x_ssm, M * E * es),
                       (lay.gate, M * E * es), (lay.u, M * E * es), (lay.xdbl, M * (R + 2 * N) * 4),
                       (lay.delta, M * E * es), (lay.y_ssm, M * E * es), (lay.o_attn, M * E * es),
                       (lay.fused, M * E * es)]
            for (o, size), (o_next, _) in zip(regions, regions[1:] + [(lay.total, 0)]):
                assert o % 256 == 0 and o + size <= o_next, (kw, consumer, B, n)
        if cfg.n_meta == 0:
            with pytest.raises(hy.HymbaError) as e:
                hy.hymba_layer_prefill_layout(h, 1, 0)
            assert e.value.status == hy.HYMBA_ERR_INVALID_ARG
        hy.hymba_layer_destroy(h)
        if prod:
            hy.hymba_layer_destroy(prod)


@pytest.mark.parametrize("glob", [False, True])
def test_decode_workspace_never_shrinks_as_the_position_grows(glob):
    """A workspace sized for max_pos serves every earlier step: the size is non-decreasing in
    the position, and constant for a sliding-window layer once the window is full."""
    h = hy.hymba_layer_create(_cfg(is_global=glob), _fake_weights())
    sizes = [hy.hymba_layer_decode_workspace(h, 128, p) for p in range(128, 128 + 20000, 97)]
    assert all(a <= b for a, b in zip(sizes, sizes[1:]))
    if glob:
        assert sizes[-1] > sizes[0]
    else:
        tail = [hy.hymba_layer_decode_workspace(h, 128, p) for p in range(128 + 1024, 128 + 9000, 331)]
        assert len(set(tail)) == 1
    with pytest.raises(hy.HymbaError) as e:
        hy.hymba_layer_decode_workspace(h, 128, 127)   # a meta position
    assert e.value.status == hy.HYMBA_ERR_INVALID_ARG
    hy.hymba_layer_destroy(h)


def test_wait_limit_is_clamped_and_restorable():
    assert hy.hymba_set_wait_limit(10) == 100000
    assert hy.hymba_set_wait_limit(5_000_000) == 5_000_000
    default = hy.hymba_set_wait_limit(0)
    assert default >= 100000
    with pytest.raises(hy.HymbaError):
        hy.hymba_set_wait_limit(-1)
    hy.hymba_debug_stall_next_prefill(0)
    with pytest.raises(hy.HymbaError):
        hy.hymba_debug_stall_next_prefill(-1)


def test_meta_cache_calls_check_their_stamps_before_launch():
    p = hy.hymba_layer_create(_cfg(), _fake_weights())
    c = hy.hymba_layer_create(_cfg(), _fake_weights(1 << 41))
    hy.hymba_kv_share_bind(c, p)
    A = 1 << 44
    try:
        assert hy.hymba_layer_meta_workspace(p) == hy.hymba_layer_prefill_workspace(p, 1, 0)
        assert hy.hymba_layer_prefill_cached_workspace(p, 4, 300) < hy.hymba_layer_prefill_workspace(p, 4, 300)
        meta = hy.hymba_meta_cache(A, A, A, A, A, 0)
        # a consumer needs its producer's meta cache, stamped by the producer
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_meta_precompute(c, A, meta, None, A, 1 << 30)
        assert e.value.status == hy.HYMBA_ERR_NOT_BOUND
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_meta_precompute(c, A, meta, hy.hymba_meta_cache(A, A, A, A, A, 42), A, 1 << 30)
        assert e.value.status == hy.HYMBA_ERR_NOT_BOUND
        # a prefill from a meta cache this layer did not compute
        kv = hy.hymba_kv_seq(A, A, 0, 0, 0)
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_prefill_cached(p, 2, 100, A, A, meta, kv, None, None, A, 1 << 34)
        assert e.value.status == hy.HYMBA_ERR_NOT_BOUND
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_layer_prefill_cached(p, 2, 0, A, A, meta, kv, None, None, A, 1 << 34)
        assert e.value.status == hy.HYMBA_ERR_INVALID_ARG
        # no meta tokens, no meta cache
        nom = hy.hymba_layer_create(_cfg(n_meta=0), _fake_weights(1 << 42))
        with pytest.raises(hy.HymbaError):
            hy.hymba_layer_meta_workspace(nom)
        hy.hymba_layer_destroy(nom)
    finally:
        hy.hymba_layer_destroy(p)
        hy.hymba_layer_destroy(c)


def test_rope_configuration_is_validated():
    h = hy.hymba_layer_create(_cfg(rope_base=10000.0), _fake_weights())
    plain = hy.hymba_layer_create(_cfg(), _fake_weights(1 << 41))
    try:
        for bad, want in ((-1.0, hy.HYMBA_ERR_INVALID_ARG), (0.5, hy.HYMBA_ERR_UNSUPPORTED)):
            with pytest.raises(hy.HymbaError) as e:
                hy.hymba_layer_create(_cfg(rope_base=bad), _fake_weights(1 << 42))
            assert e.value.status == want
        # K/V sharing needs the same rotation on both sides
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_kv_share_bind(plain, h)
        assert e.value.status == hy.HYMBA_ERR_NOT_BOUND
        # the rotary table lives in the workspace
        assert hy.hymba_layer_prefill_workspace(h, 2, 100) > hy.hymba_layer_prefill_workspace(plain, 2, 100)
    finally:
        hy.hymba_layer_destroy(h)
        hy.hymba_layer_destroy(plain)


def test_block_calls_validate_before_launch():
    p = hy.hymba_layer_create(_cfg(), _fake_weights())
    A = 1 << 44
    try:
        bw = hy.hymba_block_weights(A, A, A, A, 5504)
        ws = hy.hymba_block_prefill_workspace(p, 5504, 2, 100)
        assert ws > hy.hymba_layer_prefill_workspace(p, 2, 100)
        kv = hy.hymba_kv_seq(A, A, 0, 0, 0)
        for bad in (hy.hymba_block_weights(A, A, A, A, 5500),      # not a multiple of 8
                    hy.hymba_block_weights(A, None, A, A, 5504),   # missing norm
                    hy.hymba_block_weights(A, A, A + 4, A, 5504)):  # misaligned
            with pytest.raises(hy.HymbaError):
                hy.hymba_block_prefill(p, bad, 2, 100, A, A + (1 << 32), kv, None, None, A, ws)
        with pytest.raises(hy.HymbaError) as e:   # the output may not alias the input
            hy.hymba_block_prefill(p, bw, 2, 100, A, A, kv, None, None, A, ws)
        assert e.value.status == hy.HYMBA_ERR_INVALID_ARG
        with pytest.raises(hy.HymbaError) as e:
            hy.hymba_block_prefill(p, bw, 2, 100, A, A + (1 << 32), kv, None, None, A, ws - 256)
        assert e.value.status == hy.HYMBA_ERR_WORKSPACE
        assert hy.hymba_block_decode_workspace(p, 5504, 128, 8320) > hy.hymba_layer_decode_workspace(p, 128, 8320)
    finally:
        hy.hymba_layer_destroy(p)


def test_branch_chunks_workspace():
    """The concurrent prefill's chunks share one scan chunk-state region sized for the
    largest chunk; every chunking of a batch gets a workspace (no device needed)."""
    sizes = {}
    for chunks in (0, 1, 2, 3, 8):
        h = hy.hymba_layer_create(_cfg(branch_chunks=chunks), _fake_weights())
        try:
            for batch in (1, 2, 5, 128):
                sizes[(chunks, batch)] = hy.hymba_layer_prefill_workspace(h, batch, 1000)
        finally:
            hy.hymba_layer_destroy(h)
    for batch in (1, 2, 5, 128):
        assert sizes[(0, batch)] == sizes[(1, batch)]
        for chunks in (2, 3, 8):
            assert sizes[(chunks, batch)] > 0
    # batch 1 never splits
    assert len({sizes[(c, 1)] for c in (0, 1, 2, 3, 8)}) == 1
