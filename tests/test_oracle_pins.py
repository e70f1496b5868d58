"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
brute force on tiny inputs, closed forms, library routines, invariants the pages
state, and the cache sizes the pages print.  CPU only."""
from __future__ import annotations

import json
import math
import os

from dataclasses import replace

import numpy as np
import pytest

from oracle import hymba_oracle as O
from tests import _small

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --- P1: attention equals a brute-force per-query loop (Eq. 1 with scale and mask) ----------

def _attention_loop(q, k, v, s):
    """Pure-Python scalar loops with math.exp, one query and one key at a time."""
    L = q.shape[0]
    H, G, dq, dv = s.n_heads, s.n_kv_heads, s.head_dim_qk, s.head_dim_v
    out = np.zeros((L, H * dv))
    for h in range(H):
        g = h // (H // G)
        for i in range(L):
            scores = []
            for j in range(L):
                ok = j <= i and (s.is_global or j < s.n_meta or i - j < s.window)
                if ok:
                    dot = sum(q[i, h * dq + t] * k[j, g * dq + t] for t in range(dq))
                    scores.append((j, dot / math.sqrt(dq)))
            mx = max(sc for _, sc in scores)
            ws = [(j, math.exp(sc - mx)) for j, sc in scores]
            tot = sum(w for _, w in ws)
            for t in range(dv):
                out[i, h * dv + t] = sum(w * v[j, g * dv + t] for j, w in ws) / tot
    return out


@pytest.mark.parametrize("m,W,glob", [(3, 5, False), (0, 4, False), (2, 100, False), (3, 5, True)])
def test_p1_attention_bruteforce(m, W, glob):
    s = _small.spec(m=m, W=W, is_global=glob, H=4, G=2, dq=4, E=16)
    r = np.random.default_rng(7)
    L = 13
    q = r.normal(size=(L, s.n_heads * s.head_dim_qk))
    k = r.normal(size=(L, s.n_kv_heads * s.head_dim_qk))
    v = r.normal(size=(L, s.n_kv_heads * s.head_dim_v))
    np.testing.assert_allclose(O.attention(q, k, v, s), _attention_loop(q, k, v, s),
                               rtol=0, atol=1e-12)


# --- P2: mask special cases -------------------------------------------------------------------

def test_p2_window_covering_sequence_is_global():
    L = 37
    for m in (0, 1, 5):
        for W in (L, L + 1, 1000):
            np.testing.assert_array_equal(O.mask_matrix(L, m, W, False), O.mask_matrix(L, m, 0, True))
    s_loc = _small.spec(m=2, W=40)
    s_glob = _small.spec(m=2, W=1, is_global=True)
    w = _small.weights(s_loc, seed=3)
    x = _small.x_tilde(s_loc, 20)
    np.testing.assert_allclose(O.layer_prefill(x, w, s_loc)["Y"], O.layer_prefill(x, w, s_glob)["Y"],
                               rtol=0, atol=1e-13)


def test_p2_zero_meta_is_plain_sliding_window():
    L = 29
    for W in (1, 2, 7, 28, 29):
        want = np.array([[j <= i and i - j < W for j in range(L)] for i in range(L)])
        np.testing.assert_array_equal(O.mask_matrix(L, 0, W, False), want)


def test_mask_predicate_and_bitmap_match_explicit_loops():
    for (L, m, W, g) in [(70, 16, 8, False), (33, 0, 1, False), (64, 64, 3, False), (65, 1, 64, False),
                         (40, 5, 0, True)]:
        mat = O.mask_matrix(L, m, W, g)
        for i in range(L):
            for j in range(L):
                assert mat[i, j] == O.allowed(i, j, m, W, g)
        bm = O.mask_bitmap(L, m, W, g)
        for i in range(L):
            for j in range(L):
                assert bool((int(bm[i, j // 32]) >> (j % 32)) & 1) == mat[i, j]
            # bits past L are zero
            for j in range(L, bm.shape[1] * 32):
                assert ((int(bm[i, j // 32]) >> (j % 32)) & 1) == 0


# --- P3: beta = 0 isolates one branch (Eq. 3; head-importance analysis of §2.1) ----------------

def test_p3_beta_isolates_branches():
    s = _small.spec()
    w = _small.weights(s, seed=5)
    x = _small.x_tilde(s, 17)
    base = O.layer_prefill(x, w, s)
    # beta_ssm = 0: output is W_out(beta_attn * norm(attn) / 2) and does not depend on SSM weights.
    w_a = dict(w, beta_ssm=np.zeros(s.d_inner))
    ya = O.layer_prefill(x, w_a, s)["Y"]
    na = base["o"] / np.sqrt((base["o"] ** 2).mean(1, keepdims=True) + s.eps)
    np.testing.assert_allclose(ya, (w["beta_attn"] * na / 2) @ w["w_out"].T, atol=1e-12)
    w_a2 = dict(w_a, conv_w=w["conv_w"] * 3.0, a_log=w["a_log"] * 0.5, w_x=-w["w_x"])
    np.testing.assert_allclose(O.layer_prefill(x, w_a2, s)["Y"], ya, atol=1e-12)
    # beta_attn = 0: output does not depend on the Q/K/V rows of W_in.
    w_s = dict(w, beta_attn=np.zeros(s.d_inner))
    ys = O.layer_prefill(x, w_s, s)["Y"]
    nqkv = s.n_heads * s.head_dim_qk + s.n_kv_heads * (s.head_dim_qk + s.head_dim_v)
    w_in2 = w["w_in"].copy()
    w_in2[:nqkv] = np.random.default_rng(9).normal(size=(nqkv, s.d_model))
    np.testing.assert_allclose(O.layer_prefill(x, dict(w_s, w_in=w_in2), s)["Y"], ys, atol=1e-12)
    ns = base["y_ssm"] / np.sqrt((base["y_ssm"] ** 2).mean(1, keepdims=True) + s.eps)
    np.testing.assert_allclose(ys, (w["beta_ssm"] * ns / 2) @ w["w_out"].T, atol=1e-12)
    # Both on: the mean of the two normalised branches (factor 1/2, not a sum).
    np.testing.assert_allclose(base["Y"], ya + ys, atol=1e-12)


# --- P4: constant delta, scalar A, constant B and u -> geometric sum --------------------------

def test_p4_scan_geometric_closed_form():
    T, E, N = 50, 3, 2
    dl, a_val, b_val, u_val = 0.3, -1.7, 0.8, 1.3
    u = np.full((T, E), u_val)
    delta = np.full((T, E), dl)
    A = np.full((E, N), a_val)
    Bm = np.full((T, N), b_val)
    Cm = np.ones((T, N))
    y, h = O.selective_scan(u, delta, A, Bm, Cm, np.zeros(E))
    a = math.exp(dl * a_val)
    for t in range(T):
        want = dl * b_val * u_val * (1 - a ** (t + 1)) / (1 - a)
        np.testing.assert_allclose(y[t], N * want, rtol=1e-13)
    np.testing.assert_allclose(h, dl * b_val * u_val * (1 - a ** T) / (1 - a), rtol=1e-13)


def test_scan_with_zero_A_is_cumulative_sum():
    r = np.random.default_rng(2)
    T, E, N = 40, 5, 3
    u, delta = r.normal(size=(T, E)), r.uniform(0.1, 1, (T, E))
    Bm, Cm = r.normal(size=(T, N)), r.normal(size=(T, N))
    y, h = O.selective_scan(u, delta, np.zeros((E, N)), Bm, Cm, np.zeros(E))
    hs = np.cumsum((delta * u)[:, :, None] * Bm[:, None, :], axis=0)
    np.testing.assert_allclose(y, np.einsum("ten,tn->te", hs, Cm), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h, hs[-1], rtol=1e-12)


# --- P5: Eq. 2's materialised operator equals the recurrence ----------------------------------

def test_p5_materialised_eq2_equals_recurrence():
    r = np.random.default_rng(4)
    T, E, N = 24, 6, 4
    u, delta = r.normal(size=(T, E)), r.uniform(0.05, 0.8, (T, E))
    A = -np.exp(r.uniform(0, math.log(16), (E, N)))
    Bm, Cm = r.normal(size=(T, N)), r.normal(size=(T, N))
    Dv = r.normal(size=E)
    z = r.normal(size=(T, E))
    y_rec, _ = O.selective_scan(u, delta, A, Bm, Cm, Dv)
    # alpha^{i,j}[c] = sum_n C_i[n] * prod_{k=j+1..i} exp(A[c,n] delta_k[c]) * B_j[n] * delta_j[c]
    y_mat = np.zeros((T, E))
    for i in range(T):
        for j in range(i + 1):
            decay = np.exp(A * delta[j + 1:i + 1].sum(axis=0)[:, None])  # empty product -> 1
            alpha = (Cm[i][None, :] * decay * Bm[j][None, :]).sum(axis=1) * delta[j]
            y_mat[i] += alpha * u[j]
        y_mat[i] += Dv * u[i]
    np.testing.assert_allclose(y_rec, y_mat, rtol=1e-11, atol=1e-12)
    silu = z / (1 + np.exp(-z))
    np.testing.assert_allclose(y_rec * silu, y_mat * silu, rtol=1e-11, atol=1e-12)


# --- conv: causal depthwise conv equals numpy.convolve; tap order --------------------------------

def test_causal_conv_matches_numpy_convolve():
    r = np.random.default_rng(6)
    T, E, K = 19, 4, 4
    x = r.normal(size=(T, E))
    w = r.normal(size=(E, K))
    b = r.normal(size=E)
    u = O.causal_conv_silu(x, w, b)
    for c in range(E):
        pre = np.convolve(x[:, c], w[c, ::-1])[:T] + b[c]
        np.testing.assert_allclose(u[:, c], pre / (1 + np.exp(-pre)), rtol=1e-13, atol=1e-14)
    # history rows act as the K-1 inputs before row 0
    hist = r.normal(size=(K - 1, E))
    full = O.causal_conv_silu(np.concatenate([hist, x]), w, b)[K - 1:]
    np.testing.assert_allclose(O.causal_conv_silu(x, w, b, history=hist), full, rtol=1e-13)


def test_elementwise_functions_known_values():
    np.testing.assert_allclose(O.softplus(np.array([0.0, -4.0, 30.0, -50.0])),
                               [math.log(2.0), math.log1p(math.exp(-4.0)), 30.0 + math.log1p(math.exp(-30.0)),
                                math.exp(-50.0)], rtol=1e-14)
    np.testing.assert_allclose(O.silu(np.array([0.0, 1.0, -2.0])),
                               [0.0, 1 / (1 + math.exp(-1)), -2 / (1 + math.exp(2))], rtol=1e-14)


# --- the SSM readings (Mamba-1 form) reduced to closed forms by special weights --------------

def _silu_scalar(x):
    return x / (1.0 + math.exp(-x))


def _softplus_scalar(x):
    return math.log1p(math.exp(x)) if x < 30 else x + math.log1p(math.exp(-x))


def test_ssm_with_C_zero_is_the_D_skip_times_the_gate():
    """With the C rows of W_x at zero the recurrence term of y vanishes: y = D * u (D acts on
    the conv output, not on x_ssm) and y_ssm = D * u * SiLU(z), whatever A, delta and B are."""
    s = _small.spec()
    w = _small.weights(s, seed=11)
    R, N = s.dt_rank, s.d_state
    w_x = w["w_x"].copy()
    w_x[R + N:R + 2 * N] = 0.0
    w0 = dict(w, w_x=w_x)
    x = _small.x_tilde(s, 14, seed=3)
    r0 = O.layer_prefill(x, w0, s)
    T, E = r0["u"].shape
    for t in range(T):
        for c in range(E):
            want_y = w["d_skip"][c] * r0["u"][t, c]
            assert abs(r0["y"][t, c] - want_y) <= 1e-13 * (1 + abs(want_y))
            want = want_y * _silu_scalar(r0["z"][t, c])
            assert abs(r0["y_ssm"][t, c] - want) <= 1e-13 * (1 + abs(want))
    # the recurrence inputs no longer matter
    w_x2 = w_x.copy()
    w_x2[:R + N] *= -2.5
    w1 = dict(w0, w_x=w_x2, a_log=w["a_log"][::-1].copy(), b_dt=w["b_dt"] + 1.0, w_dt=-w["w_dt"])
    np.testing.assert_allclose(O.layer_prefill(x, w1, s)["y_ssm"], r0["y_ssm"], rtol=1e-13, atol=1e-14)


def test_delta_with_zero_W_dt_is_softplus_of_the_bias():
    """delta = softplus(delta_r W_dt^T + b_dt): with W_dt = 0 every row is softplus(b_dt)."""
    s = _small.spec()
    w = dict(_small.weights(s, seed=12), w_dt=np.zeros((s.d_inner, s.dt_rank)))
    r = O.layer_prefill(_small.x_tilde(s, 9), w, s)
    for c in range(s.d_inner):
        want = _softplus_scalar(w["b_dt"][c])
        assert np.all(np.abs(r["delta"][:, c] - want) <= 1e-14 * want)


def test_full_rank_delta_of_the_conv_output():
    """R = E with W_x[:R] = I and W_dt = I: delta = softplus(u + b_dt) elementwise, so delta is
    driven by the conv + SiLU output u (not by x_ssm), through W_x first and W_dt second."""
    E = 16
    s = _small.spec(E=E, R=E)
    w = _small.weights(s, seed=13)
    w_x = w["w_x"].copy()
    w_x[:E] = np.eye(E)
    w = dict(w, w_x=w_x, w_dt=np.eye(E))
    r = O.layer_prefill(_small.x_tilde(s, 11), w, s)
    T = r["u"].shape[0]
    for t in range(T):
        for c in range(E):
            want = _softplus_scalar(r["u"][t, c] + w["b_dt"][c])
            assert abs(r["delta"][t, c] - want) <= 1e-14 * (1 + want)


# --- P6: a KV-sharing consumer equals recomputation with the producer's K/V -------------------

def test_p6_kv_shared_consumer_equals_recompute():
    s = _small.spec(m=2, W=4)
    wp = _small.weights(s, seed=11)
    wc = _small.weights(s, seed=12, consumer=True)
    x = _small.x_tilde(s, 15, seed=3)
    prod = O.layer_prefill(x, wp, s)
    cons = O.layer_prefill(x, wc, s, kv_from=prod)
    # A standalone layer with the consumer's Q/SSM/gate rows and the producer's K/V rows, on the
    # same input: its own K/V equal the producer's, so it must match the consumer exactly.
    nq = s.n_heads * s.head_dim_qk
    nkv = s.n_kv_heads * (s.head_dim_qk + s.head_dim_v)
    w_in = np.concatenate([wc["w_in"][:nq], wp["w_in"][nq:nq + nkv], wc["w_in"][nq:]], 0)
    alone = O.layer_prefill(x, dict(wc, w_in=w_in), s)
    np.testing.assert_allclose(cons["Y"], alone["Y"], atol=1e-13)
    # With a different consumer input the K/V still come from the producer's input.
    x2 = _small.x_tilde(s, 15, seed=4)
    cons2 = O.layer_prefill(x2, wc, s, kv_from=prod)
    cons3 = O.layer_prefill(x2, wc, s, kv_from=O.layer_prefill(x2, wp, s))
    assert np.abs(cons2["o"] - cons3["o"]).max() > 1e-3


# --- P7: GQA equals MHA with K/V heads repeated per group --------------------------------------

def test_p7_gqa_equals_mha_with_repeated_kv():
    s = _small.spec(H=4, G=2, dq=4, E=16)
    w = _small.weights(s, seed=13)
    x = _small.x_tilde(s, 14)
    nq = s.n_heads * s.head_dim_qk
    nk = s.n_kv_heads * s.head_dim_qk
    nv = s.n_kv_heads * s.head_dim_v
    Wk = w["w_in"][nq:nq + nk].reshape(s.n_kv_heads, s.head_dim_qk, -1)
    Wv = w["w_in"][nq + nk:nq + nk + nv].reshape(s.n_kv_heads, s.head_dim_v, -1)
    rep = s.n_heads // s.n_kv_heads
    Wk_m = np.repeat(Wk, rep, axis=0).reshape(-1, s.d_model)  # head h <- group h // rep
    Wv_m = np.repeat(Wv, rep, axis=0).reshape(-1, s.d_model)
    s_mha = _small.spec(H=4, G=4, dq=4, E=16)
    w_m = dict(w, w_in=np.concatenate([w["w_in"][:nq], Wk_m, Wv_m, w["w_in"][nq + nk + nv:]], 0))
    np.testing.assert_allclose(O.layer_prefill(x, w, s)["Y"], O.layer_prefill(x, w_m, s_mha)["Y"],
                               atol=1e-13)


# --- P8: causality, window locality, meta rows ------------------------------------------------

def test_p8_causality_window_and_meta():
    s = _small.spec(m=3, W=4)
    w = _small.weights(s, seed=21)
    L = 18
    x = _small.x_tilde(s, L)
    base = O.layer_prefill(x, w, s)
    t = 9
    x2 = x.copy()
    x2[t] += 1.0
    y2 = O.layer_prefill(x2, w, s)
    np.testing.assert_array_equal(y2["Y"][:t], base["Y"][:t])
    assert np.abs(y2["Y"][t:] - base["Y"][t:]).min(axis=1).max() > 0
    # attention branch alone: a real row only reaches rows [j, j + W - 1]
    changed = np.abs(y2["o"] - base["o"]).max(axis=1) > 0
    assert changed.tolist() == [t <= i <= t + s.window - 1 for i in range(L)]
    # a meta row reaches every later row through attention
    x3 = x.copy()
    x3[1] += 1.0
    ch3 = np.abs(O.layer_prefill(x3, w, s)["o"] - base["o"]).max(axis=1) > 0
    assert ch3.tolist() == [i >= 1 for i in range(L)]
    # meta-row outputs do not depend on the real rows
    x4 = x.copy()
    x4[s.n_meta:] = _small.x_tilde(s, L - s.n_meta, seed=99)
    np.testing.assert_array_equal(O.layer_prefill(x4, w, s)["Y"][:s.n_meta], base["Y"][:s.n_meta])


# --- P9: prefill(n) then decode == prefill(n + 1) ------------------------------------------------

@pytest.mark.parametrize("glob,rope_base", [(False, 0.0), (True, 0.0), (False, 100.0), (True, 10000.0)])
def test_p9_decode_after_prefill(glob, rope_base):
    s = _small.spec(m=3, W=4, is_global=glob)
    if rope_base:
        s = replace(s, rope_base=rope_base)
    wp = _small.weights(s, seed=31)
    wc = _small.weights(s, seed=32, consumer=True)
    L = 16
    x = _small.x_tilde(s, L + 1)
    cap = L + 1 if glob else None
    full_p = O.layer_prefill(x, wp, s, capacity=cap)
    full_c = O.layer_prefill(x, wc, s, kv_from=full_p)
    pre_p = O.layer_prefill(x[:L], wp, s, capacity=cap)
    pre_c = O.layer_prefill(x[:L], wc, s, kv_from=pre_p)
    cache_p = dict(k=pre_p["k_cache"], v=pre_p["v_cache"], ssm=pre_p["h"], conv=pre_p["conv"])
    y_p, new_p = O.layer_decode(x[L], L, wp, s, cache_p)
    np.testing.assert_allclose(y_p, full_p["Y"][L], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(new_p["ssm"], full_p["h"], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(new_p["conv"], full_p["conv"], rtol=1e-13, atol=1e-14)
    cache_c = dict(ssm=pre_c["h"], conv=pre_c["conv"])
    y_c, _ = O.layer_decode(x[L], L, wc, s, cache_c, kv_cache=new_p)
    np.testing.assert_allclose(y_c, full_c["Y"][L], rtol=1e-11, atol=1e-12)


# --- rotary position embedding (Hymba §2.5: a RoPE base; off in the five workloads) -------------

def test_rope_closed_forms():
    """Position 0 is the identity; every head keeps its norm; pair i at position p is the
    complex product (x_2i + j x_2i+1) exp(j p base^(-2i/d)), computed here with Python's
    complex numbers."""
    rng = np.random.default_rng(7)
    d, heads, base = 8, 3, 500.0
    x = rng.normal(size=(5, heads * d))
    pos = np.array([0, 1, 7, 1000, 8319])
    r = O.rope(x, pos, d, base)
    np.testing.assert_array_equal(r[0], x[0])
    np.testing.assert_allclose(np.linalg.norm(r.reshape(5, heads, d), axis=2),
                               np.linalg.norm(x.reshape(5, heads, d), axis=2), rtol=1e-13)
    import cmath
    for row, p in enumerate(pos):
        for h in range(heads):
            for i in range(d // 2):
                z = complex(x[row, h * d + 2 * i], x[row, h * d + 2 * i + 1]) * cmath.exp(
                    1j * p * base ** (-2.0 * i / d))
                assert abs(complex(r[row, h * d + 2 * i], r[row, h * d + 2 * i + 1]) - z) <= 1e-9 * (1 + abs(z))


def test_rope_scores_depend_only_on_the_relative_position():
    rng = np.random.default_rng(8)
    d, base = 16, 10000.0
    q, k = rng.normal(size=(1, d)), rng.normal(size=(1, d))
    for i, j, shift in [(5, 2, 100), (300, 0, 7), (8000, 7990, 123)]:
        a = (O.rope(q, [i], d, base) @ O.rope(k, [j], d, base).T).item()
        b = (O.rope(q, [i + shift], d, base) @ O.rope(k, [j + shift], d, base).T).item()
        assert abs(a - b) <= 1e-9 * (1 + abs(a))
    # and they do depend on it
    a = (O.rope(q, [10], d, base) @ O.rope(k, [3], d, base).T).item()
    b = (O.rope(q, [10], d, base) @ O.rope(k, [4], d, base).T).item()
    assert abs(a - b) > 1e-3


def test_ring_slots_hold_the_window():
    """Simulate appending positions one at a time into a ring of W slots after m meta slots;
    after every append the slots hold exactly the meta rows plus the last W positions."""
    for m, W in [(0, 1), (3, 4), (5, 7), (128, 1024)]:
        s = _small.spec(m=m, W=W)
        store = {}
        for p in range(m + 3 * W + 5):
            store[O.kv_slot(p, s)] = p
            held = sorted(store.values())
            want = list(range(min(p + 1, m))) + list(range(max(m, p - W + 1), p + 1))
            assert held == want
            assert max(store) < m + W


def test_decode_slot_bitmap_by_ring_simulation():
    """The decode slot mask against a simulated store: append positions 0..pos one at a
    time (each overwrites its slot), then mark the slots whose held position is visible
    from pos under the mask predicate; before and after the ring wraps, and global."""
    for m, W, glob in [(0, 1, False), (3, 4, False), (5, 7, False), (16, 64, False), (4, 1, True),
                       (7, 0, True)]:
        s = _small.spec(m=m, W=max(W, 1), is_global=glob)
        for pos in range(m, m + 3 * max(W, 1) + 9):
            cap = pos + 1 if glob else m + W
            store = {}
            for p in range(pos + 1):
                store[p if glob or p < m else m + (p - m) % W] = p
            want = np.zeros((cap + 31) // 32, dtype=np.uint32)
            for slot, p in store.items():
                if O.allowed(pos, p, m, max(W, 1), glob):
                    want[slot // 32] |= np.uint32(1 << (slot % 32))
            np.testing.assert_array_equal(O.decode_slot_bitmap(pos, s, cap), want)


# --- P10: the printed cache sizes fix the value head width -------------------------------------

def test_p10_cache_size_reading():
    g = json.load(open(os.path.join(GOLDEN, "cache_sizes.json")))
    tokens, b = g["convention"]["tokens"], g["convention"]["bytes_per_value"]
    ll = g["llama_3_2_3b_public_config"]
    llama = ll["layers"] * ll["kv_heads"] * ll["head_dim"] * 2 * b * tokens / 1e6
    assert abs(llama - g["printed"]["llama_3_2_3b_MB"]) / g["printed"]["llama_3_2_3b_MB"] < 0.005

    def hymba(dv):
        t = g["hymba_1p5b"]
        full = t["global_layers"] * tokens * t["kv_heads"] * (t["head_dim_qk"] + dv) * b
        ring = t["swa_kv_producers"] * t["window"] * t["kv_heads"] * (t["head_dim_qk"] + dv) * b
        ssm = t["layers"] * t["d_inner"] * t["d_state"] * b
        return (full + ring + ssm) / 1e6

    printed = g["printed"]["hymba_1p5b_MB"]
    assert abs(hymba(128) - printed) / printed < 0.005
    assert abs(hymba(64) - printed) / printed > 0.25
    assert abs(g["printed"]["llama_3_2_3b_MB"] / printed - g["printed"]["ratio_vs_llama"]) < 0.05


# --- P11 / P12: softmax rows sum to one; RMS normalisation ------------------------------------

def test_p11_softmax_rows_sum_to_one():
    s = _small.spec(H=4, G=2, dq=4, E=16)
    r = np.random.default_rng(8)
    L = 11
    q = r.normal(size=(L, s.n_heads * s.head_dim_qk)) * 5
    k = r.normal(size=(L, s.n_kv_heads * s.head_dim_qk))
    v = np.ones((L, s.n_kv_heads * s.head_dim_v))
    np.testing.assert_allclose(O.attention(q, k, v, s), 1.0, atol=1e-14)
    # a constant added to every score of a row changes nothing: give every key an extra
    # coordinate equal to 1 and the query a value there
    s2 = _small.spec(H=4, G=2, dq=5, E=16)
    v2 = r.normal(size=(L, s.n_kv_heads * s.head_dim_v))

    def widen(a, heads, extra):
        a = a.reshape(L, heads, 4)
        return np.concatenate([a, np.broadcast_to(extra, (L, heads, 1))], 2).reshape(L, heads * 5)

    o1 = O.attention(widen(q, 4, 0.0), widen(k, 2, 1.0), v2, s2)
    o2 = O.attention(widen(q, 4, 3.7), widen(k, 2, 1.0), v2, s2)
    np.testing.assert_allclose(o1, o2, atol=1e-12)


def test_p12_rms_normalise():
    r = np.random.default_rng(1)
    x = r.normal(size=(7, 300)) * 9.0
    n = O.rms_normalise(x, 0.0)
    np.testing.assert_allclose(np.sqrt((n ** 2).mean(1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(n * np.sqrt((x ** 2).mean(1, keepdims=True)), x, rtol=1e-14)


# --- the block and the stack (Fig. 4 (b); Table 11) ----------------------------------------------

def _block_weights(s, seed, consumer=False, F=12):
    r = np.random.default_rng(seed)
    w = _small.weights(s, seed=seed, consumer=consumer)
    d = s.d_model
    w.update(norm1=r.uniform(0.5, 1.5, d), norm2=r.uniform(0.5, 1.5, d), w_gate=r.normal(0, 0.3, (F, d)),
             w_up=r.normal(0, 0.3, (F, d)), w_down=r.normal(0, 0.3, (d, F)))
    return w


def test_block_with_zero_branches_is_the_identity():
    s = _small.spec()
    w = _block_weights(s, 41)
    w["w_out"] = np.zeros_like(w["w_out"])
    w["w_down"] = np.zeros_like(w["w_down"])
    x = _small.x_tilde(s, 12)
    out, _ = O.block_prefill(x, w, s)
    np.testing.assert_array_equal(out, x)


def test_mlp_and_norm_against_scalar_loops():
    import math
    rng = np.random.default_rng(42)
    d, F = 5, 3
    x = rng.normal(size=(2, d))
    wg, wu, wd = rng.normal(size=(F, d)), rng.normal(size=(F, d)), rng.normal(size=(d, F))
    nw = rng.uniform(0.5, 1.5, d)
    got = O.mlp(x, wg, wu, wd)
    gn = O.rms_norm(x, nw, 1e-6)
    for r in range(2):
        ms = sum(v * v for v in x[r]) / d
        for c in range(d):
            assert abs(gn[r, c] - x[r, c] / math.sqrt(ms + 1e-6) * nw[c]) < 1e-12
        hid = []
        for f in range(F):
            g = sum(x[r, k] * wg[f, k] for k in range(d))
            u = sum(x[r, k] * wu[f, k] for k in range(d))
            hid.append(g / (1.0 + math.exp(-g)) * u)
        for c in range(d):
            assert abs(got[r, c] - sum(hid[f] * wd[c, f] for f in range(F))) < 1e-10


@pytest.mark.parametrize("glob", [False, True])
def test_block_decode_after_prefill(glob):
    s = _small.spec(m=3, W=4, is_global=glob)
    wp, wc = _block_weights(s, 43), _block_weights(s, 44, consumer=True)
    L = 14
    x = _small.x_tilde(s, L + 1)
    cap = L + 1 if glob else None
    full_p, mix_fp = O.block_prefill(x, wp, s, capacity=cap)
    full_c, _ = O.block_prefill(full_p, wc, s, kv_from=mix_fp)
    pre_p, mix_p = O.block_prefill(x[:L], wp, s, capacity=cap)
    pre_c, mix_c = O.block_prefill(pre_p, wc, s, kv_from=mix_p)
    yp, newp = O.block_decode(x[L], L, wp, s, dict(k=mix_p["k_cache"], v=mix_p["v_cache"], ssm=mix_p["h"],
                                                   conv=mix_p["conv"]))
    np.testing.assert_allclose(yp, full_p[L], rtol=1e-11, atol=1e-12)
    yc, _ = O.block_decode(yp, L, wc, s, dict(ssm=mix_c["h"], conv=mix_c["conv"]), kv_cache=newp)
    np.testing.assert_allclose(yc, full_c[L], rtol=1e-11, atol=1e-12)


def test_stack_chains_blocks_and_shares_kv():
    s = _small.spec(m=2, W=3)
    ws = [_block_weights(s, 50), _block_weights(s, 51, consumer=True), _block_weights(s, 52)]
    x = _small.x_tilde(s, 9)
    out, mixes = O.stack_prefill(x, ws, [s, s, s], [None, 0, None])
    a, m0 = O.block_prefill(x, ws[0], s)
    b, _ = O.block_prefill(a, ws[1], s, kv_from=m0)
    c, _ = O.block_prefill(b, ws[2], s)
    np.testing.assert_array_equal(out, c)
    assert mixes[1]["k"] is mixes[0]["k"]  # the consumer attends over its producer's K/V


def test_parameter_count_reading_of_the_mlp():
    """Table 11 prints 1.52B parameters for the 1.5B model.  With this layer's module
    (K/V projections only in the 18 layers that own K/V), a tied embedding of a 32K
    vocabulary and a gated MLP (gate, up, down) the count is 1.52B; an ungated MLP
    (up, down) would give 1.24B."""
    g = json.load(open(os.path.join(GOLDEN, "parameter_count.json")))
    t = g["table11_1p5b"]
    d, H, G, N, F = t["d_model"], t["n_heads"], t["n_kv_heads"], t["d_state"], t["mlp_hidden"]
    E, dq, R, K = 3200, 64, 100, 4
    dv = E // H
    owners = t["global_layers"] + 15
    consumers = t["blocks"] - owners
    def mixer(own):
        P = H * dq + (G * (dq + dv) if own else 0) + 2 * E
        return P * d + E * K + E + (R + 2 * N) * E + E * R + E + E * N + E + 2 * E + d * E + 2 * d
    mixers = owners * mixer(True) + consumers * mixer(False)
    emb = g["assumed_vocab"] * d + 128 * d   # tied embedding + meta tokens
    gated = mixers + t["blocks"] * 3 * d * F + emb
    ungated = mixers + t["blocks"] * 2 * d * F + emb
    assert abs(gated - g["printed"]["parameters_1p5b"]) < 0.01e9, gated
    assert abs(ungated - g["printed"]["parameters_1p5b"]) > 0.25e9, ungated
