"""Pins for the fp64 oracle: checks against facts fixed outside the oracle.

Each ``pin_*`` function takes a loaded oracle library (the real one, or a
deliberately broken copy built by the mutation tests) and raises
AssertionError when the oracle disagrees with the fact it pins.  None of them
restates the oracle's own formula: they use closed forms, invariances of the
definition, the online-softmax ledger the pages describe (FlashAttention,
Playable, EP 04), hand-worked tiny cases and torch's own fp64 attention.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

RNG_SEED = 1234


def _rand(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return (g.standard_normal(shape) * scale).astype(np.float32)


def _run(lib, q, k, v, scale, causal, rows=None):
    return oracle.attention_fwd(q, k, v, scale, causal, rows=rows, lib=lib)


# ---------------------------------------------------------------- closed forms

def pin_hand_worked(lib):
    """N=2, d=1, scale=1, worked by hand.

    q = [ln 3, 0], k = [1, 0], v = [4, 8]:
      row 0 scores [ln 3, 0] -> softmax [3/4, 1/4] -> o = 3 + 2 = 5, lse = ln 4
      row 1 scores [0, 0]    -> softmax [1/2, 1/2] -> o = 6,         lse = ln 2
    causal: row 0 sees only key 0 -> o = 4, lse = ln 3; row 1 unchanged.
    """
    q = np.array([math.log(3.0), 0.0], dtype=np.float64)
    # ln 3 is not exact in fp32; carry the fp32 value through the hand result.
    q32 = q.astype(np.float32)
    a = float(q32[0])  # the score of row 0 against key 0
    Q = q32.reshape(1, 1, 2, 1)
    K = np.array([1.0, 0.0], dtype=np.float32).reshape(1, 1, 2, 1)
    V = np.array([4.0, 8.0], dtype=np.float32).reshape(1, 1, 2, 1)
    o, lse = _run(lib, Q, K, V, 1.0, False)
    w0 = math.exp(a) / (math.exp(a) + 1.0)
    assert abs(o[0, 0, 0, 0] - (4 * w0 + 8 * (1 - w0))) < 1e-13, o
    assert abs(o[0, 0, 0, 0] - 5.0) < 1e-6
    assert abs(o[0, 0, 1, 0] - 6.0) < 1e-14
    assert abs(lse[0, 0, 0] - math.log(math.exp(a) + 1.0)) < 1e-14
    assert abs(lse[0, 0, 1] - math.log(2.0)) < 1e-14
    o, lse = _run(lib, Q, K, V, 1.0, True)
    assert o[0, 0, 0, 0] == 4.0
    assert abs(lse[0, 0, 0] - a) < 1e-14
    assert abs(o[0, 0, 1, 0] - 6.0) < 1e-14
    assert abs(lse[0, 0, 1] - math.log(2.0)) < 1e-14


def pin_q_zero_mean_of_v(lib):
    """Q = 0 makes every score equal: O_i is the mean of the allowed V rows and
    lse_i = ln(#allowed keys), whatever the scale."""
    B, H, N, d = 1, 2, 37, 8
    q = np.zeros((B, H, N, d), np.float32)
    k = _rand((B, H, N, d), 1)
    v = _rand((B, H, N, d), 2)
    for causal in (False, True):
        o, lse = _run(lib, q, k, v, 0.7, causal)
        for i in range(N):
            n_allowed = i + 1 if causal else N
            want = v[:, :, :n_allowed].astype(np.float64).mean(axis=2)
            np.testing.assert_allclose(o[:, :, i], want, rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[:, :, i], math.log(n_allowed), rtol=0, atol=1e-13)


def pin_single_key(lib):
    """N = 1: the only key gets weight 1, so O = V_0 and lse = scale * q . k_0."""
    q = _rand((2, 3, 1, 16), 3)
    k = _rand((2, 3, 1, 16), 4)
    v = _rand((2, 3, 1, 16), 5)
    for causal in (False, True):
        o, lse = _run(lib, q, k, v, 0.3, causal)
        np.testing.assert_array_equal(o, v.astype(np.float64))
        want = 0.3 * np.einsum("bhnd,bhnd->bhn", q.astype(np.float64), k.astype(np.float64))
        np.testing.assert_allclose(lse, want, rtol=0, atol=1e-13)


def pin_causal_row0(lib):
    """Causal row 0 sees only key 0: O_0 = V_0 exactly, lse_0 = scale * q_0 . k_0."""
    q = _rand((1, 2, 50, 32), 6, 3.0)
    k = _rand((1, 2, 50, 32), 7)
    v = _rand((1, 2, 50, 32), 8)
    o, lse = _run(lib, q, k, v, 0.25, True)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0].astype(np.float64))
    want = 0.25 * (q[:, :, 0].astype(np.float64) * k[:, :, 0].astype(np.float64)).sum(-1)
    np.testing.assert_allclose(lse[:, :, 0], want, rtol=0, atol=1e-13)


# ---------------------------------------------------------------- invariances

def pin_affine_v(lib):
    """Softmax weights sum to 1, so O(a V + b) = a O(V) + b (b a constant row)."""
    q = _rand((1, 2, 40, 8), 9, 2.0)
    k = _rand((1, 2, 40, 8), 10)
    v = _rand((1, 2, 40, 8), 11)
    a, bvec = 0.5, np.linspace(-2, 2, 8).astype(np.float32)
    v2 = (a * v + bvec).astype(np.float32)  # exact: a is a power of two... up to fp32 add
    for causal in (False, True):
        o1, l1 = _run(lib, q, k, v, 0.4, causal)
        o2, l2 = _run(lib, q, k, v2, 0.4, causal)
        # reference through the fp32 values actually passed
        ones = np.ones_like(v)
        o_one, _ = _run(lib, q, k, ones, 0.4, causal)
        np.testing.assert_allclose(o_one, 1.0, rtol=0, atol=1e-13)
        np.testing.assert_allclose(o2, a * o1 + bvec, rtol=0, atol=1e-6)
        np.testing.assert_array_equal(l1, l2)


def pin_key_permutation(lib):
    """Non-causal attention is a sum over keys: permuting K and V rows together
    changes nothing."""
    q = _rand((1, 1, 33, 16), 12, 2.0)
    k = _rand((1, 1, 33, 16), 13)
    v = _rand((1, 1, 33, 16), 14)
    perm = np.random.default_rng(15).permutation(33)
    o1, l1 = _run(lib, q, k, v, 0.5, False)
    o2, l2 = _run(lib, q, k[:, :, perm], v[:, :, perm], 0.5, False)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def pin_future_keys_ignored(lib):
    """Causal row i must not depend on keys/values after i."""
    q = _rand((1, 1, 30, 8), 16, 2.0)
    k = _rand((1, 1, 30, 8), 17)
    v = _rand((1, 1, 30, 8), 18)
    o1, l1 = _run(lib, q, k, v, 0.6, True)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 20:] = 100.0
    v2[:, :, 20:] = -50.0
    o2, l2 = _run(lib, q, k2, v2, 0.6, True)
    np.testing.assert_array_equal(o1[:, :, :20], o2[:, :, :20])
    np.testing.assert_array_equal(l1[:, :, :20], l2[:, :, :20])
    assert np.abs(o1[:, :, 20:] - o2[:, :, 20:]).max() > 1.0


def pin_softmax_shift(lib):
    """Adding one vector w to every key adds scale*q_i.w to every score of row i:
    O is unchanged and lse_i moves by exactly that amount."""
    q = _rand((1, 2, 24, 8), 19)
    k = _rand((1, 2, 24, 8), 20)
    v = _rand((1, 2, 24, 8), 21)
    w = np.array([0.5, -1.0, 0.25, 2.0, 0.0, -0.5, 1.0, 0.125], np.float32)
    k2 = (k + w).astype(np.float32)
    for causal in (False, True):
        o1, l1 = _run(lib, q, k, v, 0.8, causal)
        o2, l2 = _run(lib, q, k2, v, 0.8, causal)
        # fp32 rounding of k + w perturbs scores by ~1e-7; compare at that level
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-5)
        shift = 0.8 * (q.astype(np.float64) @ w.astype(np.float64))
        np.testing.assert_allclose(l2 - l1, shift, rtol=0, atol=1e-5)


def pin_lse_bounds(lib):
    """max_j s_ij <= lse_i <= max_j s_ij + ln(#allowed keys)."""
    q = _rand((1, 1, 64, 16), 22, 3.0)
    k = _rand((1, 1, 64, 16), 23)
    v = _rand((1, 1, 64, 16), 24)
    s = 0.5 * (q[0, 0].astype(np.float64) @ k[0, 0].astype(np.float64).T)
    for causal in (False, True):
        _, lse = _run(lib, q, k, v, 0.5, causal)
        for i in range(64):
            allowed = s[i, : i + 1] if causal else s[i]
            assert allowed.max() - 1e-12 <= lse[0, 0, i] <= allowed.max() + math.log(len(allowed)) + 1e-12


def pin_row_subset(lib):
    """Asking for a subset of rows returns exactly those rows of the full run."""
    q = _rand((2, 2, 70, 8), 25)
    k = _rand((2, 2, 70, 8), 26)
    v = _rand((2, 2, 70, 8), 27)
    rows = np.array([[[0, 5, 69], [1, 2, 3]], [[68, 0, 30], [7, 7, 7]]], np.int64)
    for causal in (False, True):
        of, lf = _run(lib, q, k, v, 0.3, causal)
        os_, ls = _run(lib, q, k, v, 0.3, causal, rows=rows)
        for b in range(2):
            for h in range(2):
                np.testing.assert_array_equal(os_[b, h], of[b, h, rows[b, h]])
                np.testing.assert_array_equal(ls[b, h], lf[b, h, rows[b, h]])


# ---------------------------------------------------------------- online ledger (pages)

def online_ledger(scores, values, tile, rescale=True):
    """The tile-by-tile ledger of FlashAttention, Playable (EP 04): a running max m,
    a running sum l and a rescale of everything accumulated whenever a tile
    brings a bigger max.  With ``rescale=False`` it is the naive streamer that
    the page shows going wrong."""
    m, l = -math.inf, 0.0
    acc = np.zeros(values.shape[1])
    for t0 in range(0, len(scores), tile):
        s = scores[t0:t0 + tile]
        m_new = max(m, float(s.max()))
        r = math.exp(m - m_new) if (rescale and m != -math.inf) else 1.0
        e = np.exp(s - m_new)
        l = l * r + float(e.sum())
        acc = acc * r + e @ values[t0:t0 + tile]
        m = m_new
    return acc / l, m + math.log(l)


def pin_online_ledger(lib):
    """Online softmax equals the all-at-once softmax (the page claims agreement
    to 15 decimals); rows are built so that later tiles bring larger maxima."""
    N, d = 96, 4
    rng = np.random.default_rng(28)
    q = np.zeros((1, 1, N, d), np.float32)
    q[0, 0, :, 0] = 1.0
    k = np.zeros((1, 1, N, d), np.float32)
    # increasing trend + noise: the running max keeps growing across tiles
    k[0, 0, :, 0] = (np.linspace(0, 12, N) + rng.standard_normal(N)).astype(np.float32)
    v = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    o, lse = _run(lib, q, k, v, 1.0, False)
    scores = k[0, 0, :, 0].astype(np.float64)
    for tile in (1, 3, 64):
        o_led, lse_led = online_ledger(scores, v[0, 0].astype(np.float64), tile)
        np.testing.assert_allclose(o[0, 0, 0], o_led, rtol=0, atol=1e-13)
        assert abs(lse[0, 0, 0] - lse_led) < 1e-13


def check_no_rescale_fails():
    """Negative control (EP 04): the streamer without rescale is far off on the
    same row, so the ledger comparison above has teeth."""
    N, d = 96, 4
    rng = np.random.default_rng(28)
    scores = rng.standard_normal(N)
    scores[-8:] += 4.0  # the last tile brings a bigger max
    values = rng.standard_normal((N, d))
    values[:-8] += 1.0
    values[-8:] -= 1.0
    good, _ = online_ledger(scores, values, 8)
    bad, _ = online_ledger(scores, values, 8, rescale=False)
    return float(np.abs(bad - good).max() / np.abs(good).max())


# ---------------------------------------------------------------- library cross-check

def pin_torch_sdpa(lib):
    """torch's fp64 math attention and logsumexp agree with the oracle."""
    for (B, H, N, d, causal, seed) in [(1, 2, 65, 16, False, 29), (2, 1, 130, 32, True, 30),
                                        (1, 1, 257, 64, True, 31)]:
        q = _rand((B, H, N, d), seed, 2.0)
        k = _rand((B, H, N, d), seed + 100)
        v = _rand((B, H, N, d), seed + 200)
        scale = 1.0 / math.sqrt(d)
        o, lse = _run(lib, q, k, v, scale, causal)
        qt, kt, vt = (torch.from_numpy(x).double() for x in (q, k, v))
        ot = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=scale)
        s = scale * qt @ kt.transpose(-1, -2)
        if causal:
            s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
        lt = torch.logsumexp(s, dim=-1)
        np.testing.assert_allclose(o, ot.numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lt.numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------- decode over a key/value cache
# New tokens attend to the cached keys ("FlashAttention: Tiled & Fused", card
# "KV Cache: Why Generation Speeds Up"); query i of nq sits at position
# nk - nq + i.

def _dec(lib, q, k, v, scale, causal):
    return oracle.attention_decode(q, k, v, scale, causal, lib=lib)


def pin_decode_hand_worked(lib):
    """One query, two cached keys, d = 1, scale = 1: q = 1, k = [0, ln 3],
    v = [4, 8] -> weights [1/4, 3/4], o = 1 + 6 = 7, lse = ln 4 (with the fp32
    value of ln 3 carried through)."""
    a = float(np.float32(math.log(3.0)))
    q = np.ones((1, 1, 1, 1), np.float32)
    k = np.array([0.0, a], np.float32).reshape(1, 1, 2, 1)
    v = np.array([4.0, 8.0], np.float32).reshape(1, 1, 2, 1)
    for causal in (False, True):  # the only query is the last position: the mask changes nothing
        o, lse = _dec(lib, q, k, v, 1.0, causal)
        w1 = math.exp(a) / (1.0 + math.exp(a))
        assert abs(o[0, 0, 0, 0] - (4 * (1 - w1) + 8 * w1)) < 1e-13, o
        assert abs(o[0, 0, 0, 0] - 7.0) < 1e-6
        assert abs(lse[0, 0, 0] - math.log(1.0 + math.exp(a))) < 1e-14


def pin_decode_closed_forms(lib):
    """q = 0: o_i is the mean of the keys query i may use (nk - nq + i + 1 of
    them under the causal mask) and lse_i = ln of their count.  nk = 1: o = v_0
    and lse = scale * q . k_0."""
    B, H, nq, nk, d = 2, 2, 5, 23, 8
    k = _rand((B, H, nk, d), 40)
    v = _rand((B, H, nk, d), 41)
    q = np.zeros((B, H, nq, d), np.float32)
    for causal in (False, True):
        o, lse = _dec(lib, q, k, v, 0.9, causal)
        for i in range(nq):
            n_allowed = nk - nq + i + 1 if causal else nk
            np.testing.assert_allclose(o[:, :, i], v[:, :, :n_allowed].astype(np.float64).mean(axis=2),
                                       rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[:, :, i], math.log(n_allowed), rtol=0, atol=1e-13)
    q1 = _rand((B, H, 1, d), 42)
    o, lse = _dec(lib, q1, k[:, :, :1], v[:, :, :1], 0.3, True)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0].astype(np.float64))
    want = 0.3 * np.einsum("bhd,bhd->bh", q1[:, :, 0].astype(np.float64), k[:, :, 0].astype(np.float64))
    np.testing.assert_allclose(lse[:, :, 0], want, rtol=0, atol=1e-13)


def pin_decode_is_the_last_rows_of_prefill(lib):
    """The queries of a decode step are the last nq rows of the full attention
    over the whole sequence: decoding them against the cache must give the
    full computation's rows nk - nq .. nk - 1, causal or not."""
    B, H, nk, d, nq = 1, 3, 70, 16, 4
    qf = _rand((B, H, nk, d), 50)
    k = _rand((B, H, nk, d), 51)
    v = _rand((B, H, nk, d), 52)
    rows = np.broadcast_to(np.arange(nk - nq, nk, dtype=np.int64), (B, H, nq))
    for causal in (False, True):
        o_full, lse_full = _run(lib, qf, k, v, 0.2, causal, rows=rows)
        o, lse = _dec(lib, qf[:, :, nk - nq:], k, v, 0.2, causal)
        np.testing.assert_allclose(o, o_full, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, lse_full, rtol=0, atol=1e-13)


def pin_decode_future_keys_ignored(lib):
    """Under the causal mask query i must not depend on cached keys past its
    position nk - nq + i; without the mask it depends on all of them."""
    B, H, nq, nk, d = 1, 2, 6, 40, 8
    q = _rand((B, H, nq, d), 60)
    k = _rand((B, H, nk, d), 61)
    v = _rand((B, H, nk, d), 62)
    o, lse = _dec(lib, q, k, v, 0.5, True)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, nk - nq + 1:] += 3.0  # every key after query 0's position
    v2[:, :, nk - nq + 1:] -= 2.0
    o2, lse2 = _dec(lib, q, k2, v2, 0.5, True)
    np.testing.assert_array_equal(o2[:, :, 0], o[:, :, 0])
    np.testing.assert_array_equal(lse2[:, :, 0], lse[:, :, 0])
    assert np.abs(o2[:, :, 1:] - o[:, :, 1:]).max() > 1e-3
    o3, _ = _dec(lib, q, k2, v2, 0.5, False)
    o4, _ = _dec(lib, q, k, v, 0.5, False)
    assert np.abs(o3 - o4).max() > 1e-3


def pin_decode_torch_sdpa(lib):
    """torch's fp64 math attention with an explicit boolean mask (query i may
    use keys <= nk - nq + i) and the scale passed in, and torch.logsumexp."""
    B, H, nq, nk, d = 2, 2, 7, 300, 32
    q = _rand((B, H, nq, d), 70)
    k = _rand((B, H, nk, d), 71)
    v = _rand((B, H, nk, d), 72)
    tq, tk, tv = (torch.from_numpy(x.astype(np.float64)) for x in (q, k, v))
    pos = torch.arange(nk - nq, nk).view(nq, 1)
    for causal in (False, True):
        mask = (torch.arange(nk).view(1, nk) <= pos) if causal else torch.ones(nq, nk, dtype=torch.bool)
        o_ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=0.17)
        s = (tq @ tk.transpose(-1, -2)) * 0.17
        lse_ref = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1)
        o, lse = _dec(lib, q, k, v, 0.17, causal)
        np.testing.assert_allclose(o, o_ref.numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref.numpy(), rtol=0, atol=1e-12)


# --------------------------------------------------------------- backward pass
# The gradient of the exact function (the pages name training as what the
# method enables; they give no backward formulas).

def _bwd(lib, q, k, v, do, scale, causal):
    return oracle.attention_bwd(q, k, v, do, scale, causal, lib=lib)


def pin_bwd_torch_autograd(lib):
    """torch's fp64 autograd through its math attention (explicit scale)."""
    for (B, H, N, d, causal, seed) in [(1, 2, 33, 8, False, 80), (2, 1, 70, 16, True, 81)]:
        q, k, v, do = (_rand((B, H, N, d), seed + i) for i in range(4))
        dq, dk, dv = _bwd(lib, q, k, v, do, 0.35, causal)
        tq, tk, tv = (torch.from_numpy(x.astype(np.float64)).requires_grad_() for x in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.35)
        o.backward(torch.from_numpy(do.astype(np.float64)))
        for got, want in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            np.testing.assert_allclose(got, want.numpy(), rtol=0, atol=1e-12)


def pin_bwd_finite_differences(lib):
    """Central differences of L = sum(O * dO), computed with the forward
    oracle, against the gradients at a few entries of q, k and v."""
    B, H, N, d = 1, 1, 6, 3
    q, k, v, do = (_rand((B, H, N, d), 90 + i) for i in range(4))
    for causal in (False, True):
        dq, dk, dv = _bwd(lib, q, k, v, do, 0.8, causal)

        def loss(qq, kk, vv):
            o, _ = _run(lib, qq, kk, vv, 0.8, causal)
            return float((o * do.astype(np.float64)).sum())

        h = 2.0 ** -10  # float32 inputs: steps of 2^-10 are exact, the loss is smooth
        for (which, grad) in ((0, dq), (1, dk), (2, dv)):
            for (i, t) in ((0, 0), (3, 2), (5, 1)):
                args = [q.copy(), k.copy(), v.copy()]
                args[which][0, 0, i, t] += h
                up = loss(*args)
                args[which][0, 0, i, t] -= 2 * h
                dn = loss(*args)
                fd = (up - dn) / (2 * h)
                assert abs(fd - grad[0, 0, i, t]) < 2e-5, (which, i, t, fd, grad[0, 0, i, t])


def pin_bwd_invariants(lib):
    """Rows of dS sum to zero, so the key gradients of a head sum to zero and
    constant keys give no query gradient; rows of P sum to one, so the value
    gradients of a head sum to the sum of dO; the gradients are linear in dO
    and vanish with it."""
    B, H, N, d = 1, 2, 29, 8
    q, k, v, do, do2 = (_rand((B, H, N, d), 100 + i) for i in range(5))
    # upstream gradients on a 2^-8 grid, so that 2 do - 3 do2 is exact in fp32
    do, do2 = (np.round(x * 256.0).astype(np.float32) / np.float32(256.0) for x in (do, do2))
    for causal in (False, True):
        dq, dk, dv = _bwd(lib, q, k, v, do, 0.5, causal)
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
        np.testing.assert_allclose(dv.sum(axis=2), do.astype(np.float64).sum(axis=2), atol=1e-12)
        kc = np.broadcast_to(k[:, :, :1], k.shape).copy()
        dqc, _, _ = _bwd(lib, q, kc, v, do, 0.5, causal)
        np.testing.assert_allclose(dqc, 0.0, atol=1e-12)
        z = _bwd(lib, q, k, v, np.zeros_like(do), 0.5, causal)
        for g in z:
            assert np.abs(g).max() == 0.0
        g1 = _bwd(lib, q, k, v, do2, 0.5, causal)
        gs = _bwd(lib, q, k, v, (2 * do - 3 * do2).astype(np.float32), 0.5, causal)
        for a, b, c in zip((dq, dk, dv), g1, gs):
            np.testing.assert_allclose(c, 2 * a - 3 * b, atol=1e-11)


def _bwd_rows(lib, q, k, v, do, scale, causal, qrows, krows):
    return oracle.attention_bwd_rows(q, k, v, do, scale, causal, qrows, krows, lib=lib)


def pin_bwd_rows_torch_autograd(lib):
    """The row-sampled gradients against torch's fp64 autograd through its
    math attention, on rows that include the first and last of each head; the
    last case spreads the scores over about +-1000, where exp without the row
    max overflows."""
    for (B, H, N, d, causal, seed, scale) in [(1, 2, 41, 8, False, 120, 0.45), (2, 1, 67, 16, True, 121, 0.45),
                                              (1, 1, 30, 8, True, 122, 40.0)]:
        q, k, v, do = (_rand((B, H, N, d), seed + i) for i in range(4))
        g = np.random.default_rng(seed)
        qrows = np.stack([np.stack([np.r_[0, N - 1, g.choice(N, 5, replace=False)] for _ in range(H)])
                          for _ in range(B)])
        krows = np.stack([np.stack([np.r_[N - 1, 0, g.choice(N, 4, replace=False)] for _ in range(H)])
                          for _ in range(B)])
        dq, dk, dv = _bwd_rows(lib, q, k, v, do, scale, causal, qrows, krows)
        tq, tk, tv = (torch.from_numpy(x.astype(np.float64)).requires_grad_() for x in (q, k, v))
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        o.backward(torch.from_numpy(do.astype(np.float64)))
        for got, full, rows in ((dq, tq.grad, qrows), (dk, tk.grad, krows), (dv, tv.grad, krows)):
            want = np.take_along_axis(full.numpy(), rows[..., None], axis=2)
            np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def pin_bwd_rows_match_full_gradients(lib):
    """The row-sampled gradients equal the full-matrix oracle's rows, on a
    head with a ragged length and on every row of a small one."""
    for (N, causal, seed) in [(37, True, 130), (37, False, 131), (12, True, 132)]:
        q, k, v, do = (_rand((1, 2, N, 8), seed + i) for i in range(4))
        rows = np.broadcast_to(np.arange(N), (1, 2, N)).copy()
        dq, dk, dv = _bwd(lib, q, k, v, do, 0.6, causal)
        rq, rk, rv = _bwd_rows(lib, q, k, v, do, 0.6, causal, rows, rows[:, :, ::-1].copy())
        np.testing.assert_allclose(rq, dq, rtol=0, atol=1e-12)
        np.testing.assert_allclose(rk, dk[:, :, ::-1], rtol=0, atol=1e-12)
        np.testing.assert_allclose(rv, dv[:, :, ::-1], rtol=0, atol=1e-12)


# ------------------------------------------------- merging partial results
def pin_merge_is_attention_over_the_union(lib):
    """Attention over a key set split into parts, merged by log-sum-exp,
    equals attention over the whole set (the forward oracle on the keys of
    each part, then the merge, against the forward oracle on all keys), for
    uneven parts and a part whose keys are all masked for some rows."""
    B, H, N, d = 1, 2, 50, 8
    q, k, v = (_rand((B, H, N, d), 110 + i) for i in range(3))
    o_ref, lse_ref = _run(lib, q, k, v, 0.4, False)
    bounds = [0, 7, 30, 50]
    parts_o, parts_l = [], []
    for a, b in zip(bounds, bounds[1:]):
        # queries against the keys [a, b): the decode oracle with nq = N and no mask
        o_p, l_p = oracle.attention_decode(q, k[:, :, a:b], v[:, :, a:b], 0.4, False, lib=lib)
        parts_o.append(o_p.astype(np.float32))
        parts_l.append(l_p.astype(np.float32))
    o, lse = oracle.lse_merge(np.stack(parts_o), np.stack(parts_l), lib=lib)
    # the parts were rounded to fp32 before the merge: agreement to fp32 precision
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=2e-6)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=2e-6)
    # a part with no usable key (lse = -inf) changes nothing
    o2, lse2 = oracle.lse_merge(np.stack(parts_o + [np.full_like(parts_o[0], 7.0)]),
                                np.stack(parts_l + [np.full_like(parts_l[0], -np.inf)]), lib=lib)
    np.testing.assert_array_equal(o2, o)
    np.testing.assert_array_equal(lse2, lse)
    # one part is the identity
    o3, lse3 = oracle.lse_merge(np.stack(parts_o[:1]), np.stack(parts_l[:1]), lib=lib)
    np.testing.assert_allclose(o3, parts_o[0], rtol=0, atol=1e-7)
    np.testing.assert_allclose(lse3, parts_l[0], rtol=0, atol=1e-6)


BWD_PINS = [pin_bwd_torch_autograd, pin_bwd_finite_differences, pin_bwd_invariants, pin_bwd_rows_torch_autograd,
            pin_bwd_rows_match_full_gradients]

DECODE_PINS = [pin_decode_hand_worked, pin_decode_closed_forms, pin_decode_is_the_last_rows_of_prefill,
               pin_decode_future_keys_ignored, pin_decode_torch_sdpa]

ALL_PINS = [
    pin_hand_worked, pin_q_zero_mean_of_v, pin_single_key, pin_causal_row0, pin_affine_v,
    pin_key_permutation, pin_future_keys_ignored, pin_softmax_shift, pin_lse_bounds,
    pin_row_subset, pin_online_ledger, pin_torch_sdpa,
] + DECODE_PINS + BWD_PINS + [pin_merge_is_attention_over_the_union]
