"""CPU oracle: RetNet multi-scale retention in float64 (test infrastructure).

This module is the yardstick the CUDA library is checked against.  It is
test infrastructure: only tests, the smoke check and the benchmark's
CPU-baseline leg use it; the product path never imports it.

Sources (web pages on RetNet; quoted by title and section):
  [SUM]  "Retentive Network: A Successor to Transformer for Large Language
         Models" -- research summary page, sections "Summary" and "Key points".
         Retention comes from a linear recurrence with exponential decay; it
         has a parallel, a recurrent (O(1) per step, no KV cache) and a
         chunkwise form (parallel inside a chunk, recurrent state passed
         between chunks); every head has its own decay gamma; positions are
         encoded in an xPos-like way; a swish gate and GroupNorm follow.
         "Key points": gamma = 1 - 2^(-5-i); chunk b = 512; head dim 256.
  [CARD] "SpiralAI Spiral-RetNet-3b-base" model card, "Visualization of the
         retention mechanism": the recurrent and parallel modes are
         mathematically equivalent.
  [MED]  "Beyond Transformers: Unveiling the Retentive Network", section
         "Efficient Inference": O(1) inference per token.

The pages name the pieces but print no equations.  The operator written out
here is the plainest reading that all of them support (one head, decay g):

  recurrent   S_t = g S_{t-1} + k_t^T v_t,   o_t = q_t S_t   (row vectors)
  parallel    O = (Q K^T (.) D) V,  D[n, m] = g^(n-m) if n >= m else 0
  chunkwise   per chunk of length L starting at token c0, with local
              indices i, j:  O_c = (Q_c K_c^T (.) D) V_c + (Q_c (.) xi) S_prev,
              xi_i = g^(i+1);  S = g^L S_prev + K_c^T (V_c (.) zeta),
              zeta_j = g^(L-1-j).
  rotation    pairs (2j, 2j+1) of q and k turned by angle pos * theta_j,
              theta_j = 10000^(-2j/d)  (xPos-like relative positions, decay
              taking the place of xPos's length scaling).
  epilogue    Y = swish(G) (.) GroupNorm_H(O), one group per head over d_v.

Layouts: q, k [B, n, H, dk]; v, o, g, y [B, n, H, dv]; state [B, H, dk, dv].
Everything is computed in float64.

Pins (tests/test_oracle.py) hold every function here to something other
than itself: hand-derived worked examples under tests/golden/, closed forms
(gamma table, decay mask), special cases that reduce to textbook routines
(gamma = 1 -> prefix-sum linear attention, gamma = 0 -> diagonal,
d = 2 rotation -> complex multiplication, GroupNorm and SiLU against
torch's library routines), brute-force state sums and the agreement of the
three independently written forms.  The gradients of the parallel form are
pinned by central finite differences of the token-by-token recurrence and by
closed forms at gamma = 0 and gamma = 1 (reverse prefix sums).
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def _f64(x):
    return np.asarray(x, dtype=F64)


# --------------------------------------------------------------------------
# Decay constants  ([SUM] "Key points": gamma = 1 - 2^(-5-i), head index i
# read as 0-based)
# --------------------------------------------------------------------------
def decay_gammas(heads: int) -> np.ndarray:
    """gamma_h = 1 - 2^(-5-h) for h = 0 .. heads-1 (exact in binary)."""
    h = np.arange(heads, dtype=F64)
    return 1.0 - np.power(2.0, -5.0 - h)


# --------------------------------------------------------------------------
# xPos-like rotation  ([SUM] "Summary": positions encoded similar to xPos)
# --------------------------------------------------------------------------
def rotation_thetas(d: int) -> np.ndarray:
    """theta_j = 10000^(-2j/d), j = 0 .. d/2-1."""
    if d % 2:
        raise ValueError("rotation needs an even head dimension")
    j = np.arange(d // 2, dtype=F64)
    return np.power(10000.0, -2.0 * j / d)


def xpos_rotate(x, pos0: int = 0) -> np.ndarray:
    """Rotate adjacent pairs of x [B, n, H, d] by (pos0 + t) * theta_j.

    (x_2j, x_2j+1) -> (x_2j cos a - x_2j+1 sin a, x_2j sin a + x_2j+1 cos a),
    a = (pos0 + t) * theta_j, t = token index.
    """
    x = _f64(x)
    n, d = x.shape[1], x.shape[3]
    theta = rotation_thetas(d)
    pos = pos0 + np.arange(n, dtype=F64)
    ang = pos[:, None] * theta[None, :]                      # [n, d/2]
    c = np.cos(ang)[None, :, None, :]
    s = np.sin(ang)[None, :, None, :]
    even = x[..., 0::2]
    odd = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = even * c - odd * s
    out[..., 1::2] = even * s + odd * c
    return out


# --------------------------------------------------------------------------
# Parallel form  ([SUM] "Summary": the parallel form, used for training)
# --------------------------------------------------------------------------
def decay_mask(n: int, gamma: float) -> np.ndarray:
    """D[a, b] = gamma^(a-b) for a >= b, else 0 (with gamma^0 = 1)."""
    idx = np.arange(n)
    diff = idx[:, None] - idx[None, :]          # a - b
    return np.where(diff >= 0, F64(gamma) ** np.maximum(diff, 0), 0.0)


def retention_parallel(q, k, v, gammas, state_in=None):
    """O = (Q K^T (.) D) V per (batch, head), plus the initial-state term.

    With an initial state S0 the recurrence unrolls to
    o_t = sum_{m<=t} g^(t-m) (q_t . k_m) v_m + g^(t+1) q_t S0, and the state
    after the last token is g^n S0 + sum_m g^(n-1-m) k_m^T v_m.
    Returns (o [B, n, H, dv], state [B, H, dk, dv]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, n, H, dk = q.shape
    dv = v.shape[3]
    gam = _f64(gammas)
    o = np.zeros((B, n, H, dv), dtype=F64)
    state = np.zeros((B, H, dk, dv), dtype=F64)
    for h in range(H):
        g = gam[h]
        D = decay_mask(n, g)
        for b in range(B):
            Q, K, V = q[b, :, h, :], k[b, :, h, :], v[b, :, h, :]
            o[b, :, h, :] = ((Q @ K.T) * D) @ V
            # state after the last token: row n-1 of D weights every key
            w = D[n - 1, :] if n else np.zeros(0)
            state[b, h] = (K * w[:, None]).T @ V
            if state_in is not None:
                S0 = _f64(state_in)[b, h]
                xi = np.power(g, np.arange(1, n + 1, dtype=F64))
                o[b, :, h, :] += (Q * xi[:, None]) @ S0
                state[b, h] += g ** n * S0
    return o, state


# --------------------------------------------------------------------------
# Recurrent form  ([SUM] "Summary": recurrent form, O(1) per step; [MED])
# --------------------------------------------------------------------------
def retention_step(q, k, v, gammas, state):
    """One decode step for every (batch, head).

    q, k [B, H, dk], v [B, H, dv], state [B, H, dk, dv] (not modified).
    S <- g S + k^T v, then o = q S (the current token is included).
    Returns (o [B, H, dv], new_state).
    """
    q, k, v, S = _f64(q), _f64(k), _f64(v), _f64(state)
    g = _f64(gammas)[None, :, None, None]
    S_new = g * S + k[:, :, :, None] * v[:, :, None, :]
    o = np.einsum("bhk,bhkv->bhv", q, S_new)
    return o, S_new


def retention_recurrent(q, k, v, gammas, state_in=None):
    """Token-by-token recurrence over the whole sequence.

    Returns (o [B, n, H, dv], state after the last token [B, H, dk, dv]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, n, H, dk = q.shape
    dv = v.shape[3]
    S = np.zeros((B, H, dk, dv), dtype=F64) if state_in is None else _f64(state_in).copy()
    o = np.zeros((B, n, H, dv), dtype=F64)
    for t in range(n):
        o[:, t], S = retention_step(q[:, t], k[:, t], v[:, t], gammas, S)
    return o, S


# --------------------------------------------------------------------------
# Chunkwise recurrent form  ([SUM] "Summary": parallel within a chunk,
# recurrent state passed between chunks; "Key points": O(dn(b+h)), b = 512)
# --------------------------------------------------------------------------
def retention_chunkwise(q, k, v, gammas, chunk: int, state_in=None):
    """Chunkwise form with chunk length `chunk` (last chunk may be shorter).

    For each chunk [c0, c0 + L) and head decay g, with local indices i, j:
      inner  = (Q_c K_c^T (.) D_L) V_c            (D_L: L x L decay mask)
      cross  = (Q_c (.) xi) S_prev,   xi_i = g^(i+1)
      S      = g^L S_prev + K_c^T (V_c (.) zeta),   zeta_j = g^(L-1-j)
    Returns (o [B, n, H, dv], final state [B, H, dk, dv]).
    """
    if chunk <= 0:
        raise ValueError("chunk must be positive")
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, n, H, dk = q.shape
    dv = v.shape[3]
    gam = _f64(gammas)
    S = np.zeros((B, H, dk, dv), dtype=F64) if state_in is None else _f64(state_in).copy()
    o = np.zeros((B, n, H, dv), dtype=F64)
    for c0 in range(0, n, chunk):
        L = min(chunk, n - c0)
        loc = np.arange(L, dtype=F64)
        for h in range(H):
            g = gam[h]
            D = decay_mask(L, g)
            xi = np.power(g, loc + 1.0)
            zeta = np.power(g, L - 1.0 - loc)
            for b in range(B):
                Q = q[b, c0:c0 + L, h, :]
                K = k[b, c0:c0 + L, h, :]
                V = v[b, c0:c0 + L, h, :]
                S_prev = S[b, h]
                inner = ((Q @ K.T) * D) @ V
                cross = (Q * xi[:, None]) @ S_prev
                o[b, c0:c0 + L, h, :] = inner + cross
                S[b, h] = g ** L * S_prev + K.T @ (V * zeta[:, None])
    return o, S


# --------------------------------------------------------------------------
# Output epilogue  ([SUM] "Summary": swish gate and GroupNorm are added)
# --------------------------------------------------------------------------
def groupnorm_swish(o, gate, weight=None, bias=None, eps: float = 1e-5):
    """Y = swish(G) (.) GroupNorm(O) with one group per head.

    o, gate [..., H, dv].  For each (token, head): mean and biased variance
    over dv; yhat = (o - mean) / sqrt(var + eps) * w + b with per-channel
    affine w, b of shape [H, dv] (defaults 1 and 0); swish(x) = x * sigmoid(x).
    """
    o, gate = _f64(o), _f64(gate)
    mean = o.mean(axis=-1, keepdims=True)
    var = ((o - mean) ** 2).mean(axis=-1, keepdims=True)
    yhat = (o - mean) / np.sqrt(var + eps)
    if weight is not None:
        yhat = yhat * _f64(weight)
    if bias is not None:
        yhat = yhat + _f64(bias)
    swish = gate / (1.0 + np.exp(-gate))
    return swish * yhat


# --------------------------------------------------------------------------
# Whole prefill pass: rotation -> chunkwise retention -> (gate epilogue)
# --------------------------------------------------------------------------
# --------------------------------------------------------------------------
# Gradients of the parallel form  ([SUM] "Summary": the parallel form is the
# one used for training).  The pages print no backward pass; these are the
# derivatives of O = (Q K^T (.) D) V (zero initial state) written out with
# the same D, by the product rule on each factor.
# --------------------------------------------------------------------------
def retention_parallel_backward(q, k, v, gammas, d_out):
    """Gradients of O = (Q K^T (.) D) V with respect to Q, K and V.

    With A = Q K^T (.) D and dA = (dO V^T) (.) D (D is constant):
        dV = A^T dO,   dQ = dA K,   dK = dA^T Q,
    per (batch, head).  Returns (dq, dk, dv) in the layouts of q, k, v.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(d_out)
    B, n, H, _ = q.shape
    gam = _f64(gammas)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for h in range(H):
        D = decay_mask(n, gam[h])
        for b in range(B):
            Q, K, V, dO = q[b, :, h, :], k[b, :, h, :], v[b, :, h, :], do[b, :, h, :]
            A = (Q @ K.T) * D
            dA = (dO @ V.T) * D
            dv[b, :, h, :] = A.T @ dO
            dq[b, :, h, :] = dA @ K
            dk[b, :, h, :] = dA.T @ Q
    return dq, dk, dv


def xpos_rotate_backward(dy, pos0: int = 0) -> np.ndarray:
    """Gradient of xpos_rotate: each pair's rotation is orthogonal, so the
    gradient is the pair turned back by the same angle (R^T dy)."""
    dy = _f64(dy)
    n, d = dy.shape[1], dy.shape[3]
    theta = rotation_thetas(d)
    pos = pos0 + np.arange(n, dtype=F64)
    ang = pos[:, None] * theta[None, :]
    c = np.cos(ang)[None, :, None, :]
    s = np.sin(ang)[None, :, None, :]
    even = dy[..., 0::2]
    odd = dy[..., 1::2]
    out = np.empty_like(dy)
    out[..., 0::2] = even * c + odd * s
    out[..., 1::2] = -even * s + odd * c
    return out


def retention_prefill_backward(q, k, v, gammas, d_out, pos0: int = 0, rotate: bool = True):
    """Gradients of O = retention(R q, R k, v) (zero initial state, no
    epilogue) with respect to the raw q, k and v, by the chain rule through
    the rotation.  Returns (dq, dk, dv)."""
    if rotate:
        qr, kr = xpos_rotate(q, pos0), xpos_rotate(k, pos0)
    else:
        qr, kr = _f64(q), _f64(k)
    dqr, dkr, dv = retention_parallel_backward(qr, kr, v, gammas, d_out)
    if rotate:
        return xpos_rotate_backward(dqr, pos0), xpos_rotate_backward(dkr, pos0), dv
    return dqr, dkr, dv


def retention_prefill(q, k, v, gammas, chunk: int, pos0: int = 0, rotate: bool = True,
                      state_in=None, gate=None, weight=None, bias=None, eps: float = 1e-5):
    """The hot path in page order: rotate q, k; chunkwise retention; epilogue.

    Returns (out, state): out is Y when `gate` is given, else O.
    """
    if rotate:
        q = xpos_rotate(q, pos0)
        k = xpos_rotate(k, pos0)
    o, state = retention_chunkwise(q, k, v, gammas, chunk, state_in)
    if gate is not None:
        o = groupnorm_swish(o, gate, weight, bias, eps)
    return o, state


# --------------------------------------------------------------------------
# The multi-scale retention layer  ([SUM] "Summary": retention replaces
# multi-head attention; a swish gate and GroupNorm are added.  "Key points":
# the 200M models have hidden size 1024.)  The input is projected to the
# queries, keys, values and the gate input by dense weights, and the gated,
# normalised retention output is projected back.
# --------------------------------------------------------------------------
def linear(x, w):
    """y = x W^T: x [..., in], w [out, in] (a linear layer's weight)."""
    return _f64(x) @ _f64(w).T


def msr_layer(x, w_q, w_k, w_v, w_g, w_o, gammas, chunk: int, pos0: int = 0,
              state_in=None, weight=None, bias=None, eps: float = 1e-5):
    """x [B, n, hidden]; w_q, w_k, w_v, w_g [H d, hidden]; w_o [hidden, H d].

    q, k, v, g = x W_q^T, x W_k^T, x W_v^T, x W_g^T (reshaped [B, n, H, d]);
    y = swish(g) (.) GroupNorm(retention(R q, R k, v)) as retention_prefill
    computes it; returns (y W_o^T [B, n, hidden], final state).
    """
    x = _f64(x)
    B, n, _ = x.shape
    H = len(gammas)
    d = w_q.shape[0] // H
    q, k, v, g = (linear(x, w).reshape(B, n, H, d) for w in (w_q, w_k, w_v, w_g))
    y, state = retention_prefill(q, k, v, gammas, chunk, pos0=pos0, state_in=state_in, gate=g,
                                 weight=weight, bias=bias, eps=eps)
    return linear(y.reshape(B, n, H * d), w_o), state
