"""Pins for the fp64 oracle: facts fixed by the mathematics of softmax attention,
not by the oracle's own code.

Each pin takes an ``oracle.Oracle`` and raises ``AssertionError`` when the oracle
disagrees. ``test_oracle_pins.py`` runs them on the real oracle and
``test_oracle_planted.py`` runs them on copies of the oracle with one planted
mistake each, to show that every such mistake trips at least one pin.

Sources of the facts:
  * closed forms of the definition (page "PyTorch-CUDA-v2.9镜像中使用FlashAttention提升训练速度",
    the Attention(Q,K,V) formula): Q = 0 gives the mean of the visible values; a row
    that sees one key returns that key's value; one-hot keys with a large score select
    one value row; constant value rows pass through unchanged;
  * invariants of the softmax gradient: rows of dS sum to zero, so sum_j dK_j = 0 and
    sum_j dV_j = sum_i dO_i; shifting K by u shifts LSE_i by scale * q_i . u; etc.;
  * central finite differences of L = <O, dO> (the backward is the gradient of L);
  * torch's fp64 CPU scaled_dot_product_attention and autograd, as an independent
    library implementation of the same definition.

The key-padding pins (`key_padding_mask`, True = padded key: accepted by the attention layer
of page "PyTorch-CUDA-v2.9镜像中使用FlashAttention提升训练速度", applied with masked_fill(-inf) on
every head and query by the reference layer of page "Flash Attention 3.7 核心原理与实战" §4.2)
use: no flags set is no mask at all; padded keys' K and V rows do not matter and
get zero gradients; a single unpadded key is returned exactly; a fully padded batch entry
gives O = 0, LSE = -inf and zero gradients; finite differences; torch's SDPA with the combined
boolean mask.

The variable-length pins (`lengths`, each sample's real length: the dynamic batching of page
"告别OOM和训练慢…" §6) use: full lengths are no restriction at all; an entry of length L is the
problem truncated to its first L tokens, with zero outputs, -inf LSE and zero gradients past
it; a zero-length entry is all zeros; finite differences.

The dropout pins (`dropout_p` of page "告别OOM和训练慢…" §4.2; F.dropout on the softmax
weights before the product with V in the reference layer of page "Flash Attention 3.7 核心原理
与实战" §4.2) pin the generator by the known-answer vectors of Philox4x32-10 (Salmon, Moraes,
Dror and Shaw, SC 2011, as published with the authors' Random123 library), the keep flags by
their documented counter/byte layout computed from those pinned outputs, p = 0 as no dropout
at all, the dropped fraction by a binomial bound, and the arithmetic by torch autograd in
fp64 with the same flags as an explicit multiplicative mask and by finite differences.

The ALiBi pins (linear bias -m_h |i - j| on the scaled scores, the `alibi_slopes` parameter
of page "告别OOM和训练慢…(含A100环境配置)" §4.2) use the same kinds of facts: closed forms
where the scores are the bias alone, the limit of a bias so steep that each row sees only
itself, finite differences, zero slopes, and torch's SDPA with the bias as a float mask.
"""
from __future__ import annotations

import math

import numpy as np
import torch

# (causal, (left, right)) mask modes exercised by the pins
MODES = [
    (False, (-1, -1)),
    (True, (-1, -1)),
    (False, (2, 0)),
    (False, (1, 1)),
    (False, (0, 2)),
    (True, (3, -1)),
]


def _rng(seed):
    return np.random.default_rng(seed)


def _visible_count(i, N, causal, window):
    """Number of keys row i sees: the width of the band [i-left, i+right] clipped to [0, N)."""
    left, right = window
    if causal:
        right = 0 if (right < 0 or right > 0) else right
    lo = 0 if left < 0 else max(0, i - left)
    hi = N - 1 if right < 0 else min(N - 1, i + right)
    return hi - lo + 1, lo, hi


def pin_single_key(orc):
    """N = 1: O = V, LSE = scale q.k, dQ = dK = 0, dV = dO (any mask mode)."""
    r = _rng(1)
    q, k, v, do = (r.standard_normal((2, 3, 1, 5)) for _ in range(4))
    scale = 0.37
    for causal, window in MODES:
        o, lse = orc.fwd(q, k, v, scale, causal, window)
        np.testing.assert_allclose(o, v, rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse, scale * np.sum(q * k, axis=-1), rtol=1e-14, atol=1e-14)
        dq, dk, dv = orc.bwd(q, k, v, do, scale, causal, window)
        np.testing.assert_allclose(dq, 0.0, atol=1e-15)
        np.testing.assert_allclose(dk, 0.0, atol=1e-15)
        np.testing.assert_allclose(dv, do, rtol=0, atol=1e-15)


def pin_zero_queries(orc):
    """Q = 0: every visible score is 0, so O_i is the plain mean of the visible V rows
    and LSE_i = ln(number of visible keys), for every mask mode."""
    r = _rng(2)
    B, H, N, d = 1, 2, 9, 3
    q = np.zeros((B, H, N, d))
    k = r.standard_normal((B, H, N, d))
    v = r.standard_normal((B, H, N, d))
    for causal, window in MODES:
        o, lse = orc.fwd(q, k, v, 0.5, causal, window)
        for i in range(N):
            cnt, lo, hi = _visible_count(i, N, causal, window)
            np.testing.assert_allclose(o[:, :, i], v[:, :, lo:hi + 1].mean(axis=2),
                                       rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(lse[:, :, i], math.log(cnt), rtol=0, atol=1e-13)


def pin_causal_first_row(orc):
    """Causal row 0 sees only key 0: O_0 = V_0, LSE_0 = scale q_0.k_0 and dQ_0 = 0."""
    r = _rng(3)
    q, k, v, do = (r.standard_normal((2, 2, 6, 4)) for _ in range(4))
    scale = 0.6
    o, lse = orc.fwd(q, k, v, scale, True)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[:, :, 0], scale * np.sum(q[:, :, 0] * k[:, :, 0], axis=-1),
                               rtol=1e-14, atol=1e-14)
    dq, _, _ = orc.bwd(q, k, v, do, scale, True)
    np.testing.assert_allclose(dq[:, :, 0], 0.0, atol=1e-15)


def pin_one_hot_keys(orc):
    """K_j = c e_j, Q_i = e_{pi(i)}, c * scale = 30: row i scores 30 on key pi(i) and 0
    elsewhere, so LSE_i = ln(e^30 + N - 1) exactly and O_i = V_{pi(i)} up to N e^-30."""
    N, d = 6, 8
    c, scale = 256.0, 30.0 / 256.0
    perm = np.array([3, 0, 5, 1, 4, 2])
    k = np.zeros((1, 1, N, d))
    q = np.zeros((1, 1, N, d))
    for j in range(N):
        k[0, 0, j, j] = c
    for i in range(N):
        q[0, 0, i, perm[i]] = 1.0
    v = _rng(4).standard_normal((1, 1, N, d))
    o, lse = orc.fwd(q, k, v, scale)
    np.testing.assert_allclose(lse[0, 0], math.log(math.exp(30.0) + N - 1), rtol=0, atol=1e-13)
    tol = 2 * N * math.exp(-30.0) * np.abs(v).max()
    np.testing.assert_allclose(o[0, 0], v[0, 0, perm], rtol=0, atol=tol)


def pin_constant_values(orc):
    """All V rows equal w: O_i = w, and dP_ij = dO_i . w is constant along j, so dS = 0
    and dQ = dK = 0, for every mask mode."""
    r = _rng(5)
    B, H, N, d = 1, 2, 7, 4
    q = r.standard_normal((B, H, N, d))
    k = r.standard_normal((B, H, N, d))
    w = r.standard_normal((B, H, 1, d))
    v = np.repeat(w, N, axis=2)
    do = r.standard_normal((B, H, N, d))
    for causal, window in MODES:
        o, _ = orc.fwd(q, k, v, 0.8, causal, window)
        np.testing.assert_allclose(o, v, rtol=1e-13, atol=1e-13)
        dq, dk, _ = orc.bwd(q, k, v, do, 0.8, causal, window)
        np.testing.assert_allclose(dq, 0.0, atol=1e-12)
        np.testing.assert_allclose(dk, 0.0, atol=1e-12)


def pin_two_keys_logistic(orc):
    """Two keys, no mask, d = 1: P_i0 is the logistic function of s_i0 - s_i1, so
    O_i = sigma(s_i0 - s_i1) v_0 + sigma(s_i1 - s_i0) v_1 and LSE_i = s_i1 + ln(1 + e^(s_i0 - s_i1))."""
    q = np.array([0.3, -1.2]).reshape(1, 1, 2, 1)
    k = np.array([1.5, -0.4]).reshape(1, 1, 2, 1)
    v = np.array([2.0, -3.0]).reshape(1, 1, 2, 1)
    scale = 0.9
    o, lse = orc.fwd(q, k, v, scale)
    for i in range(2):
        s0 = scale * q[0, 0, i, 0] * k[0, 0, 0, 0]
        s1 = scale * q[0, 0, i, 0] * k[0, 0, 1, 0]
        p0 = 1.0 / (1.0 + math.exp(s1 - s0))
        assert abs(o[0, 0, i, 0] - (p0 * 2.0 + (1 - p0) * -3.0)) < 1e-14
        assert abs(lse[0, 0, i] - (s1 + math.log1p(math.exp(s0 - s1)))) < 1e-14


def pin_finite_differences(orc):
    """dQ, dK, dV equal central finite differences of L = <O, dO> on tiny inputs, for
    every mask mode, to 1e-6 relative."""
    h = 1e-6
    for (N, d, seed) in [(1, 3, 11), (2, 1, 12), (5, 3, 13), (8, 4, 14)]:
        r = _rng(seed)
        q, k, v, do = (r.standard_normal((1, 1, N, d)) for _ in range(4))
        scale = 0.7
        for causal, window in MODES:
            grads = orc.bwd(q, k, v, do, scale, causal, window)

            def L(qq, kk, vv):
                o, _ = orc.fwd(qq, kk, vv, scale, causal, window)
                return float(np.sum(o * do))

            for which, g in enumerate(grads):
                fd = np.zeros_like(q)
                for idx in np.ndindex(q.shape):
                    args = [q.copy(), k.copy(), v.copy()]
                    args[which][idx] += h
                    lp = L(*args)
                    args[which][idx] -= 2 * h
                    lm = L(*args)
                    fd[idx] = (lp - lm) / (2 * h)
                err = np.abs(fd - g).max()
                ref = max(1.0, np.abs(g).max())
                assert err <= 1e-6 * ref, (N, d, causal, window, which, err)


def pin_gradient_invariants(orc):
    """Per head: sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i (every row sees a key);
    <Q, dQ>_F = <K, dK>_F (scores are bilinear in Q and K)."""
    r = _rng(6)
    B, H, N, d = 2, 1, 33, 8
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    for causal, window in MODES:
        dq, dk, dv = orc.bwd(q, k, v, do, 0.35, causal, window)
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)
        np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), rtol=1e-12, atol=1e-11)
        lhs = np.sum(q * dq, axis=(2, 3))
        rhs = np.sum(k * dk, axis=(2, 3))
        np.testing.assert_allclose(lhs, rhs, rtol=1e-11, atol=1e-11)


def pin_shift_invariants(orc):
    """K_j -> K_j + u leaves O unchanged and shifts LSE_i by scale q_i . u;
    V_j -> V_j + w shifts every O_i by w (rows of P sum to one)."""
    r = _rng(7)
    B, H, N, d = 1, 2, 17, 5
    q, k, v = (r.standard_normal((B, H, N, d)) for _ in range(3))
    u = r.standard_normal((B, H, 1, d))
    w = r.standard_normal((B, H, 1, d))
    scale = 0.45
    for causal, window in MODES:
        o, lse = orc.fwd(q, k, v, scale, causal, window)
        o2, lse2 = orc.fwd(q, k + u, v, scale, causal, window)
        np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse2 - lse, scale * np.sum(q * u, axis=-1), atol=1e-12)
        o3, _ = orc.fwd(q, k, v + w, scale, causal, window)
        np.testing.assert_allclose(o3 - o, np.broadcast_to(w, o.shape), atol=1e-12)


def pin_key_permutation(orc):
    """Without a mask, permuting the key/value rows together changes nothing."""
    r = _rng(8)
    q, k, v = (r.standard_normal((1, 2, 13, 6)) for _ in range(3))
    perm = r.permutation(13)
    o, lse = orc.fwd(q, k, v, 0.5)
    o2, lse2 = orc.fwd(q, k[:, :, perm], v[:, :, perm], 0.5)
    np.testing.assert_allclose(o2, o, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=1e-13, atol=1e-13)


def _band_mask(N, causal, window):
    """Boolean (N, N) mask built from torch's tril/triu band routines."""
    left, right = window
    if causal:
        right = 0 if (right < 0 or right > 0) else right
    m = torch.ones(N, N, dtype=torch.bool)
    if right >= 0:
        m = torch.tril(m, diagonal=right)
    if left >= 0:
        m = torch.triu(m, diagonal=-left)
    return m


def pin_library_sdpa(orc):
    """torch's fp64 CPU scaled_dot_product_attention (and autograd through it) gives the
    same O and gradients; torch.logsumexp of the masked scores gives the same LSE."""
    r = _rng(9)
    B, H, N, d = 2, 2, 19, 7
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    scale = 0.41
    for causal, window in MODES:
        mask = _band_mask(N, causal, window)
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask,
                                                              scale=scale)
        to.backward(torch.tensor(do))
        scores = (torch.tensor(q) @ torch.tensor(k).transpose(-1, -2)) * scale
        tlse = torch.logsumexp(scores.masked_fill(~mask, float("-inf")), dim=-1)
        o, lse = orc.fwd(q, k, v, scale, causal, window)
        dq, dk, dv = orc.bwd(q, k, v, do, scale, causal, window)
        np.testing.assert_allclose(o, to.detach().numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, tlse.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-11, atol=1e-11)


def _alibi_slopes(H):
    """The geometric slopes of the ALiBi paper: 2^(-8 h / H) for h = 1..H."""
    return np.array([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)])


def pin_alibi_two_keys(orc):
    """Q = 0 and N = 2: the scores are the bias alone, so row 0 weighs key 1 by e^-m
    against 1: O_0 = (v_0 + e^-m v_1) / (1 + e^-m), LSE_0 = ln(1 + e^-m); row 1 the same
    with the keys swapped."""
    r = _rng(11)
    H = 3
    slopes = np.array([0.3, 1.7, 4.0])
    q = np.zeros((1, H, 2, 4))
    k, v = (r.standard_normal((1, H, 2, 4)) for _ in range(2))
    o, lse = orc.fwd(q, k, v, 0.5, False, (-1, -1), slopes)
    for h, m in enumerate(slopes):
        w = math.exp(-m)
        np.testing.assert_allclose(o[0, h, 0], (v[0, h, 0] + w * v[0, h, 1]) / (1 + w), rtol=1e-13)
        np.testing.assert_allclose(o[0, h, 1], (v[0, h, 1] + w * v[0, h, 0]) / (1 + w), rtol=1e-13)
        np.testing.assert_allclose(lse[0, h], [math.log1p(w)] * 2, rtol=1e-13)


def pin_alibi_steep_bias(orc):
    """A slope of 60 with scores of order one: every other key is damped by e^-60 or more,
    so each row returns its own value, O_i = v_i, and LSE_i = scale q_i . k_i, in every mask
    mode (the diagonal is always visible)."""
    r = _rng(12)
    q, k, v = (0.3 * r.standard_normal((1, 2, 9, 4)) for _ in range(3))
    slopes = np.array([60.0, 80.0])
    for causal, window in MODES:
        o, lse = orc.fwd(q, k, v, 0.5, causal, window, slopes)
        np.testing.assert_allclose(o, v, rtol=0, atol=1e-20)
        np.testing.assert_allclose(lse, 0.5 * np.sum(q * k, axis=-1), rtol=1e-14, atol=1e-14)


def pin_alibi_zero_slopes(orc):
    """Zero slopes are no bias at all: bit-identical results."""
    r = _rng(13)
    q, k, v, do = (r.standard_normal((1, 2, 7, 3)) for _ in range(4))
    for causal, window in MODES:
        a = orc.fwd(q, k, v, 0.6, causal, window)
        b = orc.fwd(q, k, v, 0.6, causal, window, np.zeros(2))
        ga = orc.bwd(q, k, v, do, 0.6, causal, window)
        gb = orc.bwd(q, k, v, do, 0.6, causal, window, np.zeros(2))
        for x, y in zip(a + ga, b + gb):
            assert np.array_equal(x, y)


def pin_alibi_finite_differences(orc):
    """With a bias, the backward is still the gradient of L = <O, dO>: central
    differences in every entry of Q, K, V (the bias does not depend on them)."""
    r = _rng(14)
    B, H, N, d = 1, 2, 5, 3
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    slopes = np.array([0.7, 2.5])
    scale, eps = 0.45, 1e-6
    for causal, window in MODES[:3]:
        grads = orc.bwd(q, k, v, do, scale, causal, window, slopes)
        for which in range(3):
            num = np.zeros_like(q)
            for idx in np.ndindex(q.shape):
                args = [q.copy(), k.copy(), v.copy()]
                args[which][idx] += eps
                lp = np.sum(orc.fwd(*args, scale, causal, window, slopes)[0] * do)
                args[which][idx] -= 2 * eps
                lm = np.sum(orc.fwd(*args, scale, causal, window, slopes)[0] * do)
                num[idx] = (lp - lm) / (2 * eps)
            np.testing.assert_allclose(grads[which], num, rtol=1e-6, atol=1e-7)


def pin_alibi_library_sdpa(orc):
    """torch's fp64 SDPA with the bias -m_h |i - j| (and -inf where masked) as a float
    mask, and autograd through it, give the same O, LSE and gradients."""
    r = _rng(15)
    B, H, N, d = 2, 3, 17, 6
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    slopes = _alibi_slopes(H)
    scale = 0.35
    idx = torch.arange(N, dtype=torch.float64)
    dist = (idx[:, None] - idx[None, :]).abs()
    bias = -torch.tensor(slopes)[:, None, None] * dist[None]
    for causal, window in MODES:
        band = _band_mask(N, causal, window)
        fmask = bias.masked_fill(~band, float("-inf"))
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=fmask,
                                                              scale=scale)
        to.backward(torch.tensor(do))
        scores = (torch.tensor(q) @ torch.tensor(k).transpose(-1, -2)) * scale + fmask
        tlse = torch.logsumexp(scores, dim=-1)
        o, lse = orc.fwd(q, k, v, scale, causal, window, slopes)
        dq, dk, dv = orc.bwd(q, k, v, do, scale, causal, window, slopes)
        np.testing.assert_allclose(o, to.detach().numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, tlse.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-11, atol=1e-11)


def _padding(B, N, seed):
    """Seeded key-padding flags with key 0 of every batch entry unpadded (so that every row,
    causal ones included, sees at least one key), about a third of the rest padded."""
    r = _rng(seed)
    pad = r.random((B, N)) < 0.35
    pad[:, 0] = False
    return pad


def pin_padding_none_set(orc):
    """All flags False is no padding at all: bit-identical results in every mode."""
    r = _rng(21)
    q, k, v, do = (r.standard_normal((2, 2, 9, 3)) for _ in range(4))
    none = np.zeros((2, 9), dtype=bool)
    for causal, window in MODES:
        a = orc.fwd(q, k, v, 0.7, causal, window)
        b = orc.fwd(q, k, v, 0.7, causal, window, key_padding=none)
        ga = orc.bwd(q, k, v, do, 0.7, causal, window)
        gb = orc.bwd(q, k, v, do, 0.7, causal, window, key_padding=none)
        for x, y in zip(a + ga, b + gb):
            assert np.array_equal(x, y)


def pin_padding_keys_do_not_matter(orc):
    """Changing the K and V rows of padded keys changes nothing; their dK and dV are 0."""
    r = _rng(22)
    B, H, N, d = 2, 2, 11, 4
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    pad = _padding(B, N, 23)
    k2, v2 = k.copy(), v.copy()
    k2[pad[:, None, :, None].repeat(H, 1).repeat(d, 3)] += 5.0
    v2[pad[:, None, :, None].repeat(H, 1).repeat(d, 3)] -= 3.0
    for causal, window in MODES:
        o, lse = orc.fwd(q, k, v, 0.5, causal, window, key_padding=pad)
        o2, lse2 = orc.fwd(q, k2, v2, 0.5, causal, window, key_padding=pad)
        np.testing.assert_allclose(o2, o, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(lse2, lse, rtol=1e-13, atol=1e-13)
        dq, dk, dv = orc.bwd(q, k, v, do, 0.5, causal, window, key_padding=pad)
        dq2, _, _ = orc.bwd(q, k2, v2, do, 0.5, causal, window, key_padding=pad)
        np.testing.assert_allclose(dq2, dq, rtol=1e-12, atol=1e-12)
        for b in range(B):
            assert np.all(dk[b][:, pad[b]] == 0.0) and np.all(dv[b][:, pad[b]] == 0.0)


def pin_padding_single_key(orc):
    """Only key 0 unpadded: a row that sees key 0 returns v_0 with LSE = scale q_i . k_0;
    a row that does not (a window that ends before it) has O = 0 and LSE = -inf."""
    r = _rng(24)
    B, H, N, d = 1, 2, 7, 3
    q, k, v = (r.standard_normal((B, H, N, d)) for _ in range(3))
    pad = np.ones((B, N), dtype=bool)
    pad[:, 0] = False
    for causal, window in MODES:
        o, lse = orc.fwd(q, k, v, 0.9, causal, window, key_padding=pad)
        for i in range(N):
            _, lo, hi = _visible_count(i, N, causal, window)
            if lo <= 0 <= hi:
                np.testing.assert_allclose(o[0, :, i], v[0, :, 0], rtol=1e-14, atol=1e-15)
                np.testing.assert_allclose(lse[0, :, i], 0.9 * np.sum(q[0, :, i] * k[0, :, 0], -1),
                                           rtol=1e-14, atol=1e-14)
            else:
                assert np.all(o[0, :, i] == 0.0) and np.all(lse[0, :, i] == -np.inf)


def pin_padding_whole_entry(orc):
    """A batch entry whose every key is padded: O = 0, LSE = -inf and zero gradients for it,
    while the other entry is untouched by the flags of this one."""
    r = _rng(25)
    q, k, v, do = (r.standard_normal((2, 2, 6, 3)) for _ in range(4))
    pad = np.zeros((2, 6), dtype=bool)
    pad[1] = True
    o, lse = orc.fwd(q, k, v, 0.5, False, (-1, -1), key_padding=pad)
    dq, dk, dv = orc.bwd(q, k, v, do, 0.5, False, (-1, -1), key_padding=pad)
    assert np.all(o[1] == 0.0) and np.all(lse[1] == -np.inf)
    assert np.all(dq[1] == 0.0) and np.all(dk[1] == 0.0) and np.all(dv[1] == 0.0)
    o0, lse0 = orc.fwd(q[:1], k[:1], v[:1], 0.5)
    np.testing.assert_array_equal(o[0], o0[0])
    np.testing.assert_array_equal(lse[0], lse0[0])


def pin_padding_finite_differences(orc):
    """With padded keys, the backward is still the gradient of L = <O, dO>."""
    r = _rng(26)
    B, H, N, d = 2, 1, 5, 2
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    pad = np.array([[False, True, False, False, True], [False, False, True, True, False]])
    scale, eps = 0.6, 1e-6
    for causal, window in MODES[:3]:
        grads = orc.bwd(q, k, v, do, scale, causal, window, key_padding=pad)
        for which in range(3):
            num = np.zeros_like(q)
            for idx in np.ndindex(q.shape):
                args = [q.copy(), k.copy(), v.copy()]
                args[which][idx] += eps
                lp = np.sum(orc.fwd(*args, scale, causal, window, key_padding=pad)[0] * do)
                args[which][idx] -= 2 * eps
                lm = np.sum(orc.fwd(*args, scale, causal, window, key_padding=pad)[0] * do)
                num[idx] = (lp - lm) / (2 * eps)
            np.testing.assert_allclose(grads[which], num, rtol=1e-6, atol=1e-7)


def pin_padding_library_sdpa(orc):
    """torch's fp64 SDPA with the band mask and the padding combined into one boolean mask
    (and autograd through it) gives the same O, LSE and gradients."""
    r = _rng(27)
    B, H, N, d = 2, 2, 15, 5
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    pad = _padding(B, N, 28)
    scale = 0.4
    keep = torch.tensor(~pad)[:, None, None, :]
    for causal, window in MODES:
        mask = _band_mask(N, causal, window)[None, None] & keep
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask,
                                                              scale=scale)
        to.backward(torch.tensor(do))
        scores = (torch.tensor(q) @ torch.tensor(k).transpose(-1, -2)) * scale
        tlse = torch.logsumexp(scores.masked_fill(~mask, float("-inf")), dim=-1)
        o, lse = orc.fwd(q, k, v, scale, causal, window, key_padding=pad)
        dq, dk, dv = orc.bwd(q, k, v, do, scale, causal, window, key_padding=pad)
        np.testing.assert_allclose(o, to.detach().numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, tlse.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-11, atol=1e-11)


def pin_self_similarity(orc):
    """k = v = q (the page "显存神技：必学FlashAttention！" comparison input): each row's own
    key has the largest score |q_i|^2 scale among keys of no larger norm, so O is finite,
    LSE_i >= scale |q_i|^2 (the diagonal is one term of the sum) and the invariants hold."""
    r = _rng(10)
    q = r.standard_normal((1, 2, 11, 4))
    for causal, window in MODES:
        o, lse = orc.fwd(q, q, q, 0.5, causal, window)
        assert np.all(np.isfinite(o))
        assert np.all(lse >= 0.5 * np.sum(q * q, axis=-1) - 1e-12)


def pin_lengths_full_is_identity(orc):
    """lengths = N for every entry is no restriction: bit-identical results."""
    r = _rng(41)
    q, k, v, do = (r.standard_normal((2, 2, 13, 4)) for _ in range(4))
    for causal, window in MODES[:4]:
        a = orc.fwd(q, k, v, 0.5, causal, window)
        b = orc.fwd(q, k, v, 0.5, causal, window, lengths=[13, 13])
        ga = orc.bwd(q, k, v, do, 0.5, causal, window)
        gb = orc.bwd(q, k, v, do, 0.5, causal, window, lengths=[13, 13])
        for x, y in zip(a + ga, b + gb):
            assert np.array_equal(x, y)


def pin_lengths_truncated_problem(orc):
    """An entry of real length L is the same problem truncated to its first L tokens: its
    outputs and gradients there equal those of the truncated inputs; past L, O = 0,
    LSE = -inf and every gradient row is zero."""
    r = _rng(42)
    B, H, N, d = 3, 2, 17, 5
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    lens = [17, 9, 1]
    for causal, window in MODES:
        o, lse = orc.fwd(q, k, v, 0.45, causal, window, lengths=lens)
        dq, dk, dv = orc.bwd(q, k, v, do, 0.45, causal, window, lengths=lens)
        for b, L in enumerate(lens):
            sl = (slice(b, b + 1), slice(None), slice(0, L))
            ot, lt = orc.fwd(q[sl], k[sl], v[sl], 0.45, causal, window)
            gt = orc.bwd(q[sl], k[sl], v[sl], do[sl], 0.45, causal, window)
            np.testing.assert_allclose(o[sl], ot, rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(lse[b:b + 1, :, :L], lt, rtol=1e-13, atol=1e-13)
            for g, t in zip((dq, dk, dv), gt):
                np.testing.assert_allclose(g[sl], t, rtol=1e-12, atol=1e-12)
            assert np.all(o[b, :, L:] == 0.0) and np.all(np.isneginf(lse[b, :, L:]))
            for g in (dq, dk, dv):
                assert np.all(g[b, :, L:] == 0.0)


def pin_lengths_zero_entry(orc):
    """A zero-length entry: O = 0, LSE = -inf, zero gradients; the others are unaffected."""
    r = _rng(43)
    q, k, v, do = (r.standard_normal((2, 1, 7, 3)) for _ in range(4))
    o, lse = orc.fwd(q, k, v, 0.7, True, lengths=[7, 0])
    g = orc.bwd(q, k, v, do, 0.7, True, lengths=[7, 0])
    o1, lse1 = orc.fwd(q[:1], k[:1], v[:1], 0.7, True)
    assert np.all(o[1] == 0.0) and np.all(np.isneginf(lse[1]))
    np.testing.assert_allclose(o[:1], o1, rtol=1e-14, atol=1e-14)
    for x in g:
        assert np.all(x[1] == 0.0)


def pin_lengths_finite_differences(orc):
    """With variable lengths, the backward is still the gradient of L = <O, dO>."""
    h = 1e-6
    r = _rng(44)
    q, k, v, do = (r.standard_normal((2, 1, 6, 2)) for _ in range(4))
    lens = [6, 4]
    for causal, window in MODES[:3]:
        grads = orc.bwd(q, k, v, do, 0.6, causal, window, lengths=lens)

        def L(qq, kk, vv):
            o, _ = orc.fwd(qq, kk, vv, 0.6, causal, window, lengths=lens)
            return float(np.sum(o * do))

        for which, g in enumerate(grads):
            fd = np.zeros_like(q)
            for idx in np.ndindex(q.shape):
                args = [q.copy(), k.copy(), v.copy()]
                args[which][idx] += h
                lp = L(*args)
                args[which][idx] -= 2 * h
                lm = L(*args)
                fd[idx] = (lp - lm) / (2 * h)
            err = np.abs(fd - g).max()
            assert err <= 1e-6 * max(1.0, np.abs(g).max()), (causal, window, which, err)


# Philox4x32-10 known-answer vectors: (counter, key) -> output, the three published with
# the generator (all-zero, all-one and pi-digit inputs).
PHILOX_KAT = [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000), (0x00000000, 0x00000000),
     (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff, 0xffffffff, 0xffffffff, 0xffffffff), (0xffffffff, 0xffffffff),
     (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
]


def pin_philox_known_answers(orc):
    """The generator reproduces the published known-answer vectors of Philox4x32-10."""
    for ctr, key, want in PHILOX_KAT:
        assert tuple(orc.philox4x32_10(ctr, key)) == want, (ctr, key)


def pin_dropout_mask_layout(orc):
    """The keep flag of (query i, key j) of head bh is byte j mod 4 of output word
    (j mod 16) / 4 of Philox4x32-10 at counter (j / 16, i, bh, offset) and key (seed low,
    seed high), compared with t = floor(256 p + 1/2): kept iff byte >= t."""
    seed, offset, N = 0x0123456789ABCDEF, 77, 40
    for p, bh in [(0.1, 0), (0.5, 5), (0.97, 3)]:
        t = math.floor(256 * p + 0.5)
        m = orc.dropout_mask(seed, offset, bh, N, p)
        for i in range(N):
            for j in range(N):
                words = orc.philox4x32_10((j // 16, i, bh, offset),
                                          (seed & 0xFFFFFFFF, seed >> 32))
                byte = (words[(j % 16) // 4] >> (8 * (j % 4))) & 0xFF
                assert m[i, j] == (1 if byte >= t else 0), (p, bh, i, j)


def pin_dropout_zero_is_identity(orc):
    """p = 0 (and any p < 1/512, which rounds to no threshold) is no dropout at all:
    bit-identical outputs and gradients."""
    r = _rng(21)
    q, k, v, do = (r.standard_normal((1, 2, 21, 5)) for _ in range(4))
    for causal, window in MODES[:3]:
        o, lse = orc.fwd(q, k, v, 0.4, causal, window)
        g = orc.bwd(q, k, v, do, 0.4, causal, window)
        for p in (0.0, 0.0019):
            o2, lse2 = orc.fwd(q, k, v, 0.4, causal, window, dropout=(p, 5, 6))
            g2 = orc.bwd(q, k, v, do, 0.4, causal, window, dropout=(p, 5, 6))
            assert np.array_equal(o, o2) and np.array_equal(lse, lse2)
            for a, b in zip(g, g2):
                assert np.array_equal(a, b)


def pin_dropout_keep_fraction(orc):
    """Over 256 x 256 flags the dropped fraction is t / 256 within five binomial standard
    deviations; flags differ between heads, offsets and seeds."""
    n = 256 * 256
    for p in (0.1, 0.3, 0.5):
        t = math.floor(256 * p + 0.5)
        m = orc.dropout_mask(99, 0, 1, 256, p)
        dropped = n - int(m.sum())
        sigma = math.sqrt(n * (t / 256) * (1 - t / 256))
        assert abs(dropped - n * t / 256) <= 5 * sigma, (p, dropped)
    a = orc.dropout_mask(99, 0, 1, 64, 0.5)
    for other in (orc.dropout_mask(99, 0, 2, 64, 0.5), orc.dropout_mask(99, 1, 1, 64, 0.5),
                  orc.dropout_mask(98, 0, 1, 64, 0.5)):
        assert not np.array_equal(a, other)


def _dropout_factor(orc, B, H, N, p, seed, offset):
    """Z / (1 - p') per head as a (B, H, N, N) array, from the oracle's keep flags."""
    t = math.floor(256 * p + 0.5)
    z = np.stack([orc.dropout_mask(seed, offset, bh, N, p) for bh in range(B * H)])
    return (z.astype(np.float64) * (256.0 / (256.0 - t))).reshape(B, H, N, N)


def pin_dropout_library(orc):
    """torch in fp64: O = (softmax(masked scores) o Z / (1 - p')) V with the oracle's keep
    flags as an explicit factor, LSE unchanged by dropout, and autograd through that
    expression for dQ, dK, dV."""
    r = _rng(22)
    B, H, N, d = 2, 2, 37, 6
    q, k, v, do = (r.standard_normal((B, H, N, d)) for _ in range(4))
    scale, p, seed, offset = 0.37, 0.2, 1234, 9
    zf = torch.tensor(_dropout_factor(orc, B, H, N, p, seed, offset))
    for causal, window in MODES:
        mask = _band_mask(N, causal, window)
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        s = (tq @ tk.transpose(-1, -2)) * scale
        s = s.masked_fill(~mask, float("-inf"))
        to = (torch.softmax(s, dim=-1) * zf) @ tv
        to.backward(torch.tensor(do))
        tlse = torch.logsumexp(s.detach(), dim=-1)
        o, lse = orc.fwd(q, k, v, scale, causal, window, dropout=(p, seed, offset))
        dq, dk, dv = orc.bwd(q, k, v, do, scale, causal, window, dropout=(p, seed, offset))
        np.testing.assert_allclose(o, to.detach().numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, tlse.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-11, atol=1e-11)


def pin_dropout_finite_differences(orc):
    """With dropout (fixed seed, so fixed flags), the backward is the gradient of
    L = <O, dO>: central finite differences, every mask mode."""
    h = 1e-6
    for (N, d, seed) in [(5, 3, 31), (18, 2, 32)]:
        r = _rng(seed)
        q, k, v, do = (r.standard_normal((1, 1, N, d)) for _ in range(4))
        scale, drop = 0.6, (0.4, 555, 3)
        for causal, window in MODES:
            grads = orc.bwd(q, k, v, do, scale, causal, window, dropout=drop)

            def L(qq, kk, vv):
                o, _ = orc.fwd(qq, kk, vv, scale, causal, window, dropout=drop)
                return float(np.sum(o * do))

            for which, g in enumerate(grads):
                fd = np.zeros_like(q)
                for idx in np.ndindex(q.shape):
                    args = [q.copy(), k.copy(), v.copy()]
                    args[which][idx] += h
                    lp = L(*args)
                    args[which][idx] -= 2 * h
                    lm = L(*args)
                    fd[idx] = (lp - lm) / (2 * h)
                err = np.abs(fd - g).max()
                ref = max(1.0, np.abs(g).max())
                assert err <= 1e-6 * ref, (N, d, causal, window, which, err)


ALL_PINS = [
    pin_single_key,
    pin_zero_queries,
    pin_causal_first_row,
    pin_one_hot_keys,
    pin_constant_values,
    pin_two_keys_logistic,
    pin_finite_differences,
    pin_gradient_invariants,
    pin_shift_invariants,
    pin_key_permutation,
    pin_library_sdpa,
    pin_self_similarity,
    pin_alibi_two_keys,
    pin_alibi_steep_bias,
    pin_alibi_zero_slopes,
    pin_alibi_finite_differences,
    pin_alibi_library_sdpa,
    pin_padding_none_set,
    pin_padding_keys_do_not_matter,
    pin_padding_single_key,
    pin_padding_whole_entry,
    pin_padding_finite_differences,
    pin_padding_library_sdpa,
    pin_lengths_full_is_identity,
    pin_lengths_truncated_problem,
    pin_lengths_zero_entry,
    pin_lengths_finite_differences,
    pin_philox_known_answers,
    pin_dropout_mask_layout,
    pin_dropout_zero_is_identity,
    pin_dropout_keep_fraction,
    pin_dropout_library,
    pin_dropout_finite_differences,
]
