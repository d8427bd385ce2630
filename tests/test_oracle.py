"""Pins for the CPU oracle: each check holds it to something other than itself.

Hand-worked examples (tests/golden/), closed forms, special cases that reduce
to textbook or library routines, brute force on tiny inputs, and the
agreement of the three independently written forms of retention.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import read_golden, slice_rel_err

rng = np.random.default_rng(7)


def _rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


# ---------------------------------------------------------------- constants
def test_gammas_match_golden_table():
    g = read_golden("gammas_h16.txt")
    table = {}
    # each data line is "h gamma": keys are the head indices
    for key, val in g.items():
        table[int(key)] = val[0]
    got = oracle.decay_gammas(16)
    for h in range(16):
        assert got[h] == table[h], (h, got[h], table[h])
    # the first four are the 200M-layer heads
    assert list(oracle.decay_gammas(4)) == [0.96875, 0.984375, 0.9921875, 0.99609375]


def test_decay_mask_closed_form():
    D = oracle.decay_mask(8, 0.5)
    for a in range(8):
        for b in range(8):
            want = 2.0 ** (-(a - b)) if a >= b else 0.0
            assert D[a, b] == want
    assert np.array_equal(oracle.decay_mask(5, 0.0), np.eye(5))   # 0^0 = 1 on the diagonal
    assert np.array_equal(oracle.decay_mask(4, 1.0), np.tril(np.ones((4, 4))))


def test_thetas_closed_form():
    # d = 8: theta_j = 10000^(-2j/8) = 10^-j exactly
    assert np.allclose(oracle.rotation_thetas(8), [1.0, 0.1, 0.01, 0.001], rtol=1e-15, atol=0)
    assert oracle.rotation_thetas(2)[0] == 1.0


# ------------------------------------------------------- hand-worked examples
def _scalar_case():
    g = read_golden("scalar_retention_n4.txt")
    q = g["q"].reshape(1, 4, 1, 1)
    k = g["k"].reshape(1, 4, 1, 1)
    v = g["v"].reshape(1, 4, 1, 1)
    return g, q, k, v


@pytest.mark.parametrize("form", ["parallel", "recurrent", "chunk1", "chunk2", "chunk3", "chunk4"])
def test_scalar_golden(form):
    g, q, k, v = _scalar_case()
    gam = [g["gamma"][0]]
    for state_in, o_key, s_key in [(None, "o", "state"),
                                   (g["state_in"].reshape(1, 1, 1, 1), "o_with_state", "state_with_state")]:
        if form == "parallel":
            o, s = oracle.retention_parallel(q, k, v, gam, state_in)
        elif form == "recurrent":
            o, s = oracle.retention_recurrent(q, k, v, gam, state_in)
        else:
            o, s = oracle.retention_chunkwise(q, k, v, gam, int(form[5:]), state_in)
        assert np.allclose(o.ravel(), g[o_key], rtol=0, atol=1e-14), (form, o.ravel())
        assert np.allclose(s.ravel(), g[s_key], rtol=0, atol=1e-14), (form, s.ravel())


@pytest.mark.parametrize("form", ["parallel", "recurrent", "chunk1", "chunk2", "chunk3"])
def test_matrix_golden(form):
    g = read_golden("matrix_retention_n3.txt")
    q = g["q"].reshape(1, 3, 1, 2)
    k = g["k"].reshape(1, 3, 1, 2)
    v = g["v"].reshape(1, 3, 1, 2)
    gam = [g["gamma"][0]]
    if form == "parallel":
        o, s = oracle.retention_parallel(q, k, v, gam)
    elif form == "recurrent":
        o, s = oracle.retention_recurrent(q, k, v, gam)
    else:
        o, s = oracle.retention_chunkwise(q, k, v, gam, int(form[5:]))
    assert np.allclose(o.ravel(), g["o"], rtol=0, atol=1e-14), o.ravel()
    assert np.allclose(s.ravel(), g["state"], rtol=0, atol=1e-14), s.ravel()


# ------------------------------------------------------- forms agree (pages)
@pytest.mark.parametrize("chunk", [1, 2, 4, 5, 13, 16])
@pytest.mark.parametrize("with_state", [False, True])
def test_three_forms_agree(chunk, with_state):
    B, n, H, dk, dv = 2, 13, 3, 4, 6        # dk != dv catches a transposed state
    q, k, v = _rand(B, n, H, dk), _rand(B, n, H, dk), _rand(B, n, H, dv)
    gam = [0.5, 0.96875, 1.0]
    s0 = _rand(B, H, dk, dv) if with_state else None
    o_p, s_p = oracle.retention_parallel(q, k, v, gam, s0)
    o_r, s_r = oracle.retention_recurrent(q, k, v, gam, s0)
    o_c, s_c = oracle.retention_chunkwise(q, k, v, gam, chunk, s0)
    assert np.allclose(o_p, o_r, rtol=0, atol=1e-12)
    assert np.allclose(o_c, o_r, rtol=0, atol=1e-12)
    assert np.allclose(s_p, s_r, rtol=0, atol=1e-12)
    assert np.allclose(s_c, s_r, rtol=0, atol=1e-12)


def test_state_brute_force():
    B, n, H, dk, dv = 1, 9, 2, 3, 5
    q, k, v = _rand(B, n, H, dk), _rand(B, n, H, dk), _rand(B, n, H, dv)
    gam = [0.75, 0.9]
    _, S = oracle.retention_recurrent(q, k, v, gam)
    for h in range(H):
        for a in range(dk):
            for c in range(dv):
                want = 0.0
                for m in range(n):
                    want += gam[h] ** (n - 1 - m) * k[0, m, h, a] * v[0, m, h, c]
                assert abs(S[0, h, a, c] - want) < 1e-12


def test_step_is_one_token_of_the_recurrence():
    B, n, H, d = 2, 7, 2, 4
    q, k, v = _rand(B, n + 1, H, d), _rand(B, n + 1, H, d), _rand(B, n + 1, H, d)
    gam = [0.9, 0.99]
    o_full, s_full = oracle.retention_recurrent(q, k, v, gam)
    _, s_pref = oracle.retention_chunkwise(q[:, :n], k[:, :n], v[:, :n], gam, 4)
    o_step, s_step = oracle.retention_step(q[:, n], k[:, n], v[:, n], gam, s_pref)
    assert np.allclose(o_step, o_full[:, n], atol=1e-12)
    assert np.allclose(s_step, s_full, atol=1e-12)


# --------------------------------------------- special cases (textbook forms)
def test_gamma_one_is_causal_linear_attention():
    B, n, H, dk, dv = 1, 11, 2, 3, 4
    q, k, v = _rand(B, n, H, dk), _rand(B, n, H, dk), _rand(B, n, H, dv)
    o, _ = oracle.retention_chunkwise(q, k, v, [1.0, 1.0], 4)
    outer = k[..., :, None] * v[..., None, :]               # [B, n, H, dk, dv]
    prefix = np.cumsum(outer, axis=1)                        # library prefix sum
    want = np.einsum("bnhk,bnhkv->bnhv", q, prefix)
    assert np.allclose(o, want, atol=1e-12)


def test_gamma_zero_is_diagonal():
    B, n, H, dk, dv = 2, 10, 1, 3, 2
    q, k, v = _rand(B, n, H, dk), _rand(B, n, H, dk), _rand(B, n, H, dv)
    for fn in (lambda: oracle.retention_chunkwise(q, k, v, [0.0], 3),
               lambda: oracle.retention_parallel(q, k, v, [0.0]),
               lambda: oracle.retention_recurrent(q, k, v, [0.0])):
        o, s = fn()
        want = (q * k).sum(-1, keepdims=True) * v
        assert np.allclose(o, want, atol=1e-12)
        assert np.allclose(s[:, 0], k[:, -1, 0, :, None] * v[:, -1, 0, None, :], atol=1e-12)


def test_rotation_d2_is_complex_multiplication():
    n = 6
    x = _rand(1, n, 1, 2)
    for pos0 in (0, 3, 1000):
        y = oracle.xpos_rotate(x, pos0)
        z = (x[..., 0] + 1j * x[..., 1]) * np.exp(1j * (pos0 + np.arange(n)))[None, :, None]
        assert np.allclose(y[..., 0], z.real, atol=1e-12)
        assert np.allclose(y[..., 1], z.imag, atol=1e-12)


def test_rotation_d4_hand_values():
    x = np.array([1.0, 0.0, 0.0, 1.0]).reshape(1, 1, 1, 4)
    for p in (0, 1, 7, 123):
        y = oracle.xpos_rotate(x, p).ravel()
        want = [math.cos(p), math.sin(p), -math.sin(0.01 * p), math.cos(0.01 * p)]
        assert np.allclose(y, want, atol=1e-12)


def test_rotation_d8_complex_pairs_and_norm():
    x = _rand(2, 5, 3, 8)
    y = oracle.xpos_rotate(x, 11)
    theta = np.array([1.0, 0.1, 0.01, 0.001])
    pos = 11 + np.arange(5)
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * pos[None, :, None, None] * theta)
    assert np.allclose(y[..., 0::2], z.real, atol=1e-12)
    assert np.allclose(y[..., 1::2], z.imag, atol=1e-12)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), atol=1e-12)


def test_rotation_only_relative_positions_matter():
    B, n, H, d = 1, 12, 2, 8
    q, k, v = _rand(B, n, H, d), _rand(B, n, H, d), _rand(B, n, H, d)
    gam = oracle.decay_gammas(H)
    o0, s0 = oracle.retention_prefill(q, k, v, gam, 4, pos0=0)
    o1, s1 = oracle.retention_prefill(q, k, v, gam, 4, pos0=517)
    assert np.allclose(o0, o1, atol=1e-10)
    # the state is in absolute (rotated) coordinates, so it does change
    assert not np.allclose(s0, s1, atol=1e-6)


def test_split_prefill_through_state():
    B, n, H, d, m = 2, 20, 2, 8, 12
    q, k, v = _rand(B, n, H, d), _rand(B, n, H, d), _rand(B, n, H, d)
    gam = oracle.decay_gammas(H)
    o_full, s_full = oracle.retention_prefill(q, k, v, gam, 8)
    o_a, s_a = oracle.retention_prefill(q[:, :m], k[:, :m], v[:, :m], gam, 8)
    o_b, s_b = oracle.retention_prefill(q[:, m:], k[:, m:], v[:, m:], gam, 8, pos0=m, state_in=s_a)
    assert np.allclose(np.concatenate([o_a, o_b], axis=1), o_full, atol=1e-12)
    assert np.allclose(s_b, s_full, atol=1e-12)


# ---------------------------------------------------------- gate epilogue
def test_groupnorm_swish_against_torch_library():
    N, H, dv = 7, 3, 16
    o, g = _rand(N, H, dv), _rand(N, H, dv, scale=3.0)
    w, b = _rand(H, dv), _rand(H, dv)
    got = oracle.groupnorm_swish(o, g, w, b, eps=1e-5)
    t = torch.from_numpy(o.reshape(N, H * dv))
    gn = torch.nn.functional.group_norm(t, H, torch.from_numpy(w.ravel()),
                                        torch.from_numpy(b.ravel()), eps=1e-5)
    want = torch.nn.functional.silu(torch.from_numpy(g.reshape(N, H * dv))) * gn
    assert np.allclose(got.reshape(N, H * dv), want.numpy(), atol=1e-12)


def test_groupnorm_swish_hand_values():
    o = np.array([1.0, 2.0, 3.0, 4.0]).reshape(1, 1, 4)
    # mean 2.5, biased variance 1.25; a gate of 0 gives swish(0) = 0
    assert np.all(oracle.groupnorm_swish(o, np.zeros_like(o), eps=0.0) == 0.0)
    big = np.full_like(o, 60.0)          # swish(60) = 60 to double precision
    y = oracle.groupnorm_swish(o, big, eps=0.0).ravel() / 60.0
    assert np.allclose(y, np.array([-1.5, -0.5, 0.5, 1.5]) / math.sqrt(1.25), atol=1e-14)
    # unit gate: swish(1) = 1 / (1 + e^-1)
    y1 = oracle.groupnorm_swish(o, np.ones_like(o), eps=0.0).ravel()
    assert np.allclose(y1, np.array([-1.5, -0.5, 0.5, 1.5]) / math.sqrt(1.25) / (1 + math.exp(-1)),
                       atol=1e-14)


def test_groupnorm_output_moments():
    o = _rand(50, 4, 32, scale=5.0) + 3.0
    y = oracle.groupnorm_swish(o, np.full_like(o, 60.0), eps=1e-5) / 60.0
    assert np.allclose(y.mean(-1), 0.0, atol=1e-12)
    var = o.var(-1)
    assert np.allclose(y.var(-1), var / (var + 1e-5), atol=1e-12)


# ------------------------------------------------------- parity measure
def test_slice_rel_err_measure():
    ref = _rand(2, 5, 3, 4)
    assert slice_rel_err(ref, ref, keep=False) == 0.0
    bad = ref.copy()
    bad[1, 2, 2, 3] += 0.5 * np.abs(ref[1, :, 2, :]).max()
    assert abs(slice_rel_err(bad, ref, keep=False) - 0.5) < 1e-12
    nan = ref.copy()
    nan[0, 0, 0, 0] = np.nan
    assert slice_rel_err(nan, ref, keep=False) == float("inf")


# ---------------------------------------------------------------- gradients
def _loss_and_grads_fd(q, k, v, gam, w, pos0, h=1e-6):
    """Central differences of L = sum(O * w), O from the token-by-token
    recurrence (a form written independently of the gradient formulas)."""
    def loss(q_, k_, v_):
        o, _ = oracle.retention_recurrent(oracle.xpos_rotate(q_, pos0),
                                          oracle.xpos_rotate(k_, pos0), v_, gam)
        return float((o * w).sum())
    grads = []
    for x in (q, k, v):
        g = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [xp if y is x else y for y in (q, k, v)]
            args_m = [xm if y is x else y for y in (q, k, v)]
            g[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        grads.append(g)
    return grads


def test_backward_matches_finite_differences():
    B, n, H, dk, dv = 1, 5, 2, 4, 6
    q, k, v = _rand(B, n, H, dk), _rand(B, n, H, dk), _rand(B, n, H, dv)
    w = _rand(B, n, H, dv)
    gam = [0.9, 0.5]
    fd = _loss_and_grads_fd(q, k, v, gam, w, pos0=3)
    got = oracle.retention_prefill_backward(q, k, v, gam, w, pos0=3)
    for g_fd, g in zip(fd, got):
        assert np.allclose(g, g_fd, rtol=1e-6, atol=1e-7)


def test_backward_gamma_zero_closed_form():
    B, n, H, d = 2, 7, 1, 3
    q, k, v, do = (_rand(B, n, H, d) for _ in range(4))
    dq, dk, dv = oracle.retention_parallel_backward(q, k, v, [0.0], do)
    s = (do * v).sum(-1, keepdims=True)                      # dO_t . v_t
    assert np.allclose(dq, s * k, atol=1e-12)
    assert np.allclose(dk, s * q, atol=1e-12)
    assert np.allclose(dv, (q * k).sum(-1, keepdims=True) * do, atol=1e-12)


def test_backward_gamma_one_reverse_prefix_sums():
    # gamma = 1: dV_s = k_s . sum_{t>=s} q_t^T dO_t, dK_s = sum_{t>=s} (q_t dO_t^T) v_s,
    # dQ_t = dO_t . (sum_{s<=t} v_s^T k_s): prefix sums from the library
    B, n, H, dk, dv = 1, 9, 1, 3, 4
    q, k, v, do = _rand(B, n, H, dk), _rand(B, n, H, dk), _rand(B, n, H, dv), _rand(B, n, H, dv)
    dq, dk_, dv_ = oracle.retention_parallel_backward(q, k, v, [1.0], do)
    qdo = q[..., :, None] * do[..., None, :]                  # [B, n, H, dk, dv]
    rsum = np.flip(np.cumsum(np.flip(qdo, axis=1), axis=1), axis=1)
    assert np.allclose(dv_, np.einsum("bnhk,bnhkv->bnhv", k, rsum), atol=1e-12)
    assert np.allclose(dk_, np.einsum("bnhkv,bnhv->bnhk", rsum, v), atol=1e-12)
    vk = v[..., :, None] * k[..., None, :]                    # [B, n, H, dv, dk]
    psum = np.cumsum(vk, axis=1)
    assert np.allclose(dq, np.einsum("bnhv,bnhvk->bnhk", do, psum), atol=1e-12)


def test_backward_as_forward_calls_on_reversed_sequences():
    """The decomposition the GPU backward uses: dQ is a causal retention of
    (dO, V, K), and dK, dV are causal retentions in reversed time."""
    B, n, H, d = 2, 11, 3, 4
    q, k, v, do = (_rand(B, n, H, d) for _ in range(4))
    gam = [0.9, 0.7, 0.97]
    dq, dk, dv = oracle.retention_parallel_backward(q, k, v, gam, do)
    rev = lambda x: np.flip(x, axis=1)                       # noqa: E731
    fq, _ = oracle.retention_chunkwise(do, v, k, gam, 4)
    fk, _ = oracle.retention_chunkwise(rev(v), rev(do), rev(q), gam, 4)
    fv, _ = oracle.retention_chunkwise(rev(k), rev(q), rev(do), gam, 4)
    assert np.allclose(dq, fq, atol=1e-12)
    assert np.allclose(dk, rev(fk), atol=1e-12)
    assert np.allclose(dv, rev(fv), atol=1e-12)


def test_rotation_backward_is_the_inverse_turn():
    x = _rand(2, 6, 2, 8)
    y = oracle.xpos_rotate(x, 9)
    assert np.allclose(oracle.xpos_rotate_backward(y, 9), x, atol=1e-12)


# ---------------------------------------------------------------- properties
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=60, deadline=None)
@given(B=st.integers(1, 2), n=st.integers(1, 20), H=st.integers(1, 3),
       dk=st.sampled_from([2, 4, 6]), dv=st.sampled_from([2, 4, 6]),
       chunk=st.integers(1, 24), seed=st.integers(0, 2**31 - 1),
       gam=st.lists(st.floats(0.0, 1.0), min_size=3, max_size=3),
       with_state=st.booleans())
def test_three_forms_agree_on_random_shapes(B, n, H, dk, dv, chunk, seed, gam, with_state):
    r = np.random.default_rng(seed)
    q, k = r.standard_normal((B, n, H, dk)), r.standard_normal((B, n, H, dk))
    v = r.standard_normal((B, n, H, dv))
    s0 = r.standard_normal((B, H, dk, dv)) if with_state else None
    g = gam[:H]
    op, sp = oracle.retention_parallel(q, k, v, g, s0)
    orr, sr = oracle.retention_recurrent(q, k, v, g, s0)
    oc, sc = oracle.retention_chunkwise(q, k, v, g, chunk, s0)
    assert np.allclose(op, orr, rtol=1e-10, atol=1e-10)
    assert np.allclose(oc, orr, rtol=1e-10, atol=1e-10)
    assert np.allclose(sp, sr, rtol=1e-10, atol=1e-10)
    assert np.allclose(sc, sr, rtol=1e-10, atol=1e-10)


@settings(max_examples=15, deadline=None)
@given(n=st.integers(1, 6), d=st.sampled_from([2, 4]), seed=st.integers(0, 2**31 - 1),
       g=st.floats(0.05, 1.0), pos0=st.integers(0, 50))
def test_backward_matches_finite_differences_on_random_cases(n, d, seed, g, pos0):
    r = np.random.default_rng(seed)
    q, k, v, w = (r.standard_normal((1, n, 1, d)) for _ in range(4))
    fd = _loss_and_grads_fd(q, k, v, [g], w, pos0)
    got = oracle.retention_prefill_backward(q, k, v, [g], w, pos0=pos0)
    for g_fd, g_an in zip(fd, got):
        assert np.allclose(g_an, g_fd, rtol=1e-5, atol=1e-6)


# ------------------------------------------------------------ the MSR layer
def test_linear_hand_worked_example():
    g = read_golden("linear_2x3x2.txt")
    y = oracle.linear(g["x"].reshape(2, 3), g["w"].reshape(2, 3))
    np.testing.assert_array_equal(y, g["y"].reshape(2, 2))


def test_linear_against_scalar_loops_and_identity():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 4, 5))
    w = rng.standard_normal((6, 5))
    y = oracle.linear(x, w)
    want = np.zeros((3, 4, 6))
    for a in range(3):
        for b in range(4):
            for o in range(6):
                for i in range(5):
                    want[a, b, o] += x[a, b, i] * w[o, i]
    np.testing.assert_allclose(y, want, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(oracle.linear(x, np.eye(5)), x)


def test_msr_layer_wiring_against_per_head_loops():
    # every projection written out per token and head by scalar loops, then the
    # already pinned prefill and a per-token output projection
    rng = np.random.default_rng(6)
    B, n, H, d, hidden = 2, 5, 2, 4, 6
    x = rng.standard_normal((B, n, hidden))
    ws = [rng.standard_normal((H * d, hidden)) * 0.3 for _ in range(4)]
    w_o = rng.standard_normal((hidden, H * d)) * 0.3
    gam = np.array([0.9, 0.6])
    got, st = oracle.msr_layer(x, *ws, w_o, gam, chunk=2, pos0=3)

    proj = []
    for w in ws:
        p = np.zeros((B, n, H, d))
        for b in range(B):
            for t in range(n):
                for h in range(H):
                    for j in range(d):
                        p[b, t, h, j] = sum(x[b, t, i] * w[h * d + j, i] for i in range(hidden))
        proj.append(p)
    q, k, v, g = proj
    o = oracle.retention_recurrent(oracle.xpos_rotate(q, 3), oracle.xpos_rotate(k, 3), v, gam)[0]
    y = oracle.groupnorm_swish(o, g)
    want = np.zeros((B, n, hidden))
    for b in range(B):
        for t in range(n):
            for c in range(hidden):
                want[b, t, c] = sum(y[b, t, h, j] * w_o[c, h * d + j]
                                    for h in range(H) for j in range(d))
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)
    _, want_state = oracle.retention_prefill(q, k, v, gam, 2, pos0=3, gate=g)
    np.testing.assert_allclose(st, want_state, rtol=1e-12, atol=1e-14)


def test_msr_layer_with_identity_weights_is_the_gated_prefill():
    rng = np.random.default_rng(7)
    B, n, H, d = 1, 6, 2, 4
    x = rng.standard_normal((B, n, H * d))
    eye = np.eye(H * d)
    gam = np.array([0.8, 0.95])
    got, _ = oracle.msr_layer(x, eye, eye, eye, eye, eye, gam, chunk=4)
    xs = x.reshape(B, n, H, d)
    want, _ = oracle.retention_prefill(xs, xs, xs, gam, 4, gate=xs)
    np.testing.assert_allclose(got, want.reshape(B, n, H * d), rtol=1e-12, atol=1e-14)
