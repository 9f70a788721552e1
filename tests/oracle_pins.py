"""Checks that pin the fp64 oracle to facts fixed outside itself.

Each ``pin_*`` function takes an oracle front end (``oracle.Oracle``) and
raises AssertionError when it disagrees with a closed form, an invariant the
lecture page states, finite differences, a library special case or a worked
fixture.  ``tests/test_oracle.py`` runs them against the real oracle;
``tests/test_oracle_mutants.py`` compiles deliberately broken copies of the
oracle and checks that every planted mistake trips at least one pin.

Page cited throughout: "Let's build GPT: from scratch, in code, spelled out"
(the lecture page with the chapter list and corrections).  The local-window
pins (``pin_window_*``) follow the minGPT README page's reference notes on
GPT-3 (alternating dense and locally banded sparse attention), read as: token
t sees positions t-window < s <= t.  The dropout pins (``pin_dropout_*``) follow
the lecture's chapter "scaling up the model! creating a few variables. adding
dropout", read as inverted dropout on the attention weights with a Philox4x32-10
keep mask (one call per 4 x 4 block of (query t, key s) pairs: counter (s/4, t/4,
b*n_head+h, 0), key = seed, byte s%4 of word t%4, kept iff that byte >= theta =
round(256 p); kept weights scaled by 1/(1 - theta/256)); the generator's own bits
are pinned by the published known-answer vectors of Philox4x32-10
(``tests/golden/philox4x32_10_kat.json``).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _split(qkv, n_head):
    """View qkv[B,T,3C] as q, k, v of shape [B, n_head, T, hs] (heads as a batch dim)."""
    B, T, C3 = qkv.shape
    C = C3 // 3
    hs = C // n_head
    x = qkv.reshape(B, T, 3, n_head, hs)
    return [np.ascontiguousarray(x[:, :, i].transpose(0, 2, 1, 3)) for i in range(3)]


def pin_single_token(orc):
    """T=1: a token sees only itself, so its weight is exactly 1 and y = v;
    lse is the one visible score q.k / sqrt(hs) (chapter 'version 4')."""
    B, n_head, hs = 3, 2, 8
    C = n_head * hs
    qkv = _rng(1).standard_normal((B, 1, 3 * C))
    y, lse = orc.forward(qkv, n_head)
    assert np.array_equal(y, qkv[:, :, 2 * C:]), "T=1 must return V exactly"
    q, k, _ = _split(qkv, n_head)
    score = (q * k).sum(-1) / math.sqrt(hs)          # [B, nh, 1]
    assert np.allclose(lse, score, rtol=0, atol=1e-14)


def pin_uniform_scores_prefix_mean(orc):
    """Zero queries make every score equal: the weights become the lecture's
    version-1 average of the past context, y[t] = mean(v_0..v_t), and the
    normaliser is t+1 (lse = ln(t+1))."""
    B, T, n_head, hs = 2, 19, 3, 5
    C = n_head * hs
    qkv = _rng(2).standard_normal((B, T, 3 * C))
    qkv[:, :, :C] = 0.0
    y, lse = orc.forward(qkv, n_head)
    v = qkv[:, :, 2 * C:]
    for b in range(B):
        for t in range(T):
            acc = np.zeros(C)
            for s in range(t + 1):       # version 1: a for loop over the past
                acc += v[b, s]
            assert np.allclose(y[b, t], acc / (t + 1), rtol=0, atol=1e-13)
    expect = np.log(np.arange(1, T + 1, dtype=np.float64))
    assert np.allclose(lse, np.broadcast_to(expect, lse.shape), rtol=0, atol=1e-14)


def pin_tril_average_fixture(orc):
    """Golden fixture: with equal affinities the weights are the
    lower-triangular averaging matrix of chapters 'version 2'/'version 3'.
    One-hot values (v_s = e_s) expose the weights in y."""
    fx = json.load(open(os.path.join(GOLDEN, "tril_average_T5.json")))
    T = fx["T"]
    W = np.array([[float(eval(x)) for x in row] for row in fx["weights_exact"]])  # fractions like "1/3"
    n_head, hs = 1, T
    C = hs
    qkv = np.zeros((1, T, 3 * C))
    qkv[0, :, 2 * C:] = np.eye(T)
    qkv[0, :, C:2 * C] = _rng(3).standard_normal((T, C))   # keys are irrelevant when q = 0
    y, _ = orc.forward(qkv, n_head)
    assert np.allclose(y[0], W, rtol=0, atol=1e-15)
    P = orc.probs(qkv, n_head, 0, 0)
    assert np.allclose(P, W, rtol=0, atol=1e-15)


def pin_rows_are_distributions(orc):
    """Softmax rows sum to one, the future (s > t) has weight exactly zero and
    the diagonal is visible (correction to 00:57:00: the future cannot
    communicate; a token is not in its own future)."""
    B, T, n_head, hs = 2, 23, 2, 6
    C = n_head * hs
    qkv = 2.0 * _rng(4).standard_normal((B, T, 3 * C))
    for b in range(B):
        for h in range(n_head):
            P = orc.probs(qkv, n_head, b, h)
            assert np.allclose(P.sum(1), 1.0, rtol=0, atol=1e-14)
            assert np.all(P[np.triu_indices(T, 1)] == 0.0)
            assert np.all(np.diag(P) > 0.0)
            assert np.all(P >= 0.0)


def pin_weights_from_softmax_of_scaled_scores(orc):
    """Brute force on a tiny case: each weight is exp(score)/sum over the
    visible row, with score = q.k/sqrt(head_size) (note 6, correction to
    01:20:05), evaluated one element at a time with Python floats."""
    T, n_head, hs = 4, 2, 3
    C = n_head * hs
    qkv = _rng(5).standard_normal((1, T, 3 * C))
    for h in range(n_head):
        P = orc.probs(qkv, n_head, 0, h)
        for t in range(T):
            sc = []
            for s in range(t + 1):
                dot = sum(qkv[0, t, h * hs + d] * qkv[0, s, C + h * hs + d] for d in range(hs))
                sc.append(dot / math.sqrt(hs))
            den = sum(math.exp(x) for x in sc)
            for s in range(t + 1):
                assert abs(P[t, s] - math.exp(sc[s]) / den) < 1e-14


def pin_worked_two_heads(orc):
    """Golden fixture: a T=2, two-head case worked by hand (scale sqrt(hs) = 2,
    not sqrt(C)); also recomputed here from its closed form."""
    fx = json.load(open(os.path.join(GOLDEN, "worked_T2_two_heads.json")))
    qkv = np.array(fx["qkv"])
    y, lse = orc.forward(qkv, fx["n_head"])
    assert np.allclose(y, np.array(fx["y"]), rtol=0, atol=1e-13)
    assert np.allclose(lse, np.array(fx["lse"]), rtol=0, atol=1e-13)
    # closed form of head 0 at t=1: weights (1, 3)/(1+3)
    v0, v1 = qkv[0, 0, 16:20], qkv[0, 1, 16:20]
    assert np.allclose(y[0, 1, 0:4], 0.25 * v0 + 0.75 * v1, rtol=0, atol=1e-13)


def pin_causality(orc):
    """Perturbing tokens after position t leaves everything at positions <= t
    unchanged: y, lse and dq (the future cannot communicate)."""
    B, T, n_head, hs = 2, 17, 2, 4
    C = n_head * hs
    r = _rng(6)
    qkv = r.standard_normal((B, T, 3 * C))
    dy = r.standard_normal((B, T, C))
    y0, l0 = orc.forward(qkv, n_head)
    g0 = orc.backward(qkv, dy, n_head)
    for t in (0, 5, 11):
        q2 = qkv.copy()
        d2 = dy.copy()
        q2[:, t + 1:] += r.standard_normal(q2[:, t + 1:].shape)
        d2[:, t + 1:] += r.standard_normal(d2[:, t + 1:].shape)
        y1, l1 = orc.forward(q2, n_head)
        g1 = orc.backward(q2, d2, n_head)
        assert np.array_equal(y1[:, :t + 1], y0[:, :t + 1])
        assert np.array_equal(l1[:, :, :t + 1], l0[:, :, :t + 1])
        assert np.array_equal(g1[:, :t + 1, :C], g0[:, :t + 1, :C])
        assert not np.allclose(y1[:, t + 1:], y0[:, t + 1:])


def pin_batch_independence(orc):
    """No communication across the batch dimension (note 3)."""
    B, T, n_head, hs = 3, 9, 2, 4
    C = n_head * hs
    r = _rng(7)
    qkv = r.standard_normal((B, T, 3 * C))
    dy = r.standard_normal((B, T, C))
    y0, l0 = orc.forward(qkv, n_head)
    g0 = orc.backward(qkv, dy, n_head)
    q2, d2 = qkv.copy(), dy.copy()
    q2[1] = r.standard_normal(q2[1].shape)
    d2[1] = r.standard_normal(d2[1].shape)
    y1, l1 = orc.forward(q2, n_head)
    g1 = orc.backward(q2, d2, n_head)
    for b in (0, 2):
        assert np.array_equal(y1[b], y0[b]) and np.array_equal(l1[b], l0[b])
        assert np.array_equal(g1[b], g0[b])


def pin_head_permutation(orc):
    """Heads are a batch dimension (exercise EX1): permuting the heads of q, k
    and v together permutes the heads of y, lse and dqkv the same way."""
    B, T, n_head, hs = 2, 11, 4, 3
    C = n_head * hs
    r = _rng(8)
    qkv = r.standard_normal((B, T, 3 * C))
    dy = r.standard_normal((B, T, C))
    perm = np.array([2, 0, 3, 1])

    def permute_cols(x, parts):
        x = x.reshape(B, T, parts, n_head, hs)[:, :, :, perm]
        return x.reshape(B, T, parts * C)

    y0, l0 = orc.forward(qkv, n_head)
    g0 = orc.backward(qkv, dy, n_head)
    y1, l1 = orc.forward(permute_cols(qkv, 3), n_head)
    g1 = orc.backward(permute_cols(qkv, 3), permute_cols(dy, 1), n_head)
    assert np.array_equal(y1, permute_cols(y0, 1))
    assert np.array_equal(l1, l0[:, perm])
    assert np.array_equal(g1, permute_cols(g0, 3))


def pin_set_semantics(orc):
    """Attention has no notion of space (note 2): shuffling the tokens before
    position t leaves y[t] and lse[t] unchanged."""
    B, T, n_head, hs = 1, 12, 2, 5
    C = n_head * hs
    r = _rng(9)
    qkv = r.standard_normal((B, T, 3 * C))
    y0, l0 = orc.forward(qkv, n_head)
    t = 9
    perm = r.permutation(t)
    q2 = qkv.copy()
    q2[:, :t] = qkv[:, perm]
    y1, l1 = orc.forward(q2, n_head)
    assert np.allclose(y1[:, t], y0[:, t], rtol=0, atol=1e-13)
    assert np.allclose(l1[:, :, t], l0[:, :, t], rtol=0, atol=1e-13)


def pin_finite_differences(orc):
    """The backward is the gradient of L = sum(y * dy): central differences in
    fp64 (h = 1e-6) agree with it for every input element."""
    for (B, T, n_head, hs, seed) in ((1, 5, 2, 4, 10), (1, 8, 1, 3, 11)):
        C = n_head * hs
        r = _rng(seed)
        qkv = r.standard_normal((B, T, 3 * C))
        G = r.standard_normal((B, T, C))
        grad = orc.backward(qkv, G, n_head)
        h = 1e-6
        fd = np.zeros_like(qkv)
        flat = qkv.reshape(-1)
        for i in range(flat.size):
            xp = flat.copy()
            xm = flat.copy()
            xp[i] += h
            xm[i] -= h
            yp, _ = orc.forward(xp.reshape(qkv.shape), n_head)
            ym, _ = orc.forward(xm.reshape(qkv.shape), n_head)
            fd.reshape(-1)[i] = ((yp * G).sum() - (ym * G).sum()) / (2 * h)
        err = np.abs(fd - grad).max() / np.abs(grad).max()
        assert err < 1e-6, f"finite-difference mismatch {err:.3e}"


def pin_row_identity(orc):
    """The backward's row term: rowsum(dY o y) equals rowsum(P o dP) with dP = dY V^T, because
    y = P V (the lecture's weighted aggregation); y from the forward, P from the weights
    routine, element sums in fp64."""
    B, T, n_head, hs = 2, 23, 3, 6
    C = n_head * hs
    r = _rng(41)
    qkv = r.standard_normal((B, T, 3 * C)) * 1.3
    dy = r.standard_normal((B, T, C))
    y, _ = orc.forward(qkv, n_head)
    _, _, v = _split(qkv, n_head)
    for b in range(B):
        for h in range(n_head):
            P = orc.probs(qkv, n_head, b, h)
            dyh = dy[b, :, h * hs:(h + 1) * hs]
            lhs = (dyh * y[b, :, h * hs:(h + 1) * hs]).sum(axis=1)
            rhs = (P * (dyh @ v[b, h].T)).sum(axis=1)
            assert np.allclose(lhs, rhs, rtol=0, atol=1e-12)


def pin_library_special_case(orc):
    """A different implementation of the same function: PyTorch's
    scaled_dot_product_attention(is_causal=True) and autograd, in fp64 on
    the CPU (its default scale is 1/sqrt(head_size))."""
    B, T, n_head, hs = 2, 37, 3, 8
    C = n_head * hs
    r = _rng(12)
    qkv = r.standard_normal((B, T, 3 * C))
    dy = r.standard_normal((B, T, C))
    x = torch.tensor(qkv, dtype=torch.float64, requires_grad=True)
    q, k, v = x.split(C, dim=2)
    heads = lambda a: a.view(B, T, n_head, hs).transpose(1, 2)
    out = torch.nn.functional.scaled_dot_product_attention(heads(q), heads(k), heads(v), is_causal=True)
    y_ref = out.transpose(1, 2).reshape(B, T, C)
    (y_ref * torch.tensor(dy)).sum().backward()
    y, lse = orc.forward(qkv, n_head)
    g = orc.backward(qkv, dy, n_head)
    assert np.abs(y - y_ref.detach().numpy()).max() < 1e-12
    assert np.abs(g - x.grad.numpy()).max() < 1e-12
    # lse against torch.logsumexp of the masked scaled scores
    qh, kh = heads(q).detach(), heads(k).detach()
    s = qh @ kh.transpose(-1, -2) / math.sqrt(hs)
    s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
    assert np.abs(lse - torch.logsumexp(s, -1).numpy()).max() < 1e-12


def pin_regression_fixture(orc):
    """Regression fixture written by tests/golden/make_golden.py from this
    oracle: catches any later change to the oracle's arithmetic."""
    fx = json.load(open(os.path.join(GOLDEN, "oracle_small_seeded.json")))
    qkv, dy = np.array(fx["qkv"]), np.array(fx["dy"])
    y, lse = orc.forward(qkv, fx["n_head"])
    g = orc.backward(qkv, dy, fx["n_head"])
    assert np.allclose(y, fx["y"], rtol=0, atol=1e-13)
    assert np.allclose(lse, fx["lse"], rtol=0, atol=1e-13)
    assert np.allclose(g, fx["dqkv"], rtol=0, atol=1e-13)


def pin_empty(orc):
    """Empty batch or sequence: nothing to compute, shapes preserved."""
    y, lse = orc.forward(np.zeros((0, 4, 12)), 2)
    assert y.shape == (0, 4, 4) and lse.shape == (0, 2, 4)
    y, lse = orc.forward(np.zeros((2, 0, 12)), 2)
    assert y.shape == (2, 0, 4) and lse.shape == (2, 2, 0)
    g = orc.backward(np.zeros((2, 0, 12)), np.zeros((2, 0, 4)), 2)
    assert g.shape == (2, 0, 12)


# ---- local window (banded) attention ------------------------------------------

def pin_window_one(orc):
    """window = 1: each token sees only itself, so y = v exactly, lse = q.k/sqrt(hs),
    and the backward is dV = dy, dQ = dK = 0 (the softmax of one element has zero
    derivative)."""
    B, T, n_head, hs = 2, 11, 2, 4
    C = n_head * hs
    r = _rng(30)
    qkv = r.standard_normal((B, T, 3 * C))
    dy = r.standard_normal((B, T, C))
    y, lse = orc.forward(qkv, n_head, window=1)
    assert np.array_equal(y, qkv[:, :, 2 * C:])
    q, k, _ = _split(qkv, n_head)
    assert np.allclose(lse, (q * k).sum(-1) / math.sqrt(hs), rtol=0, atol=1e-14)
    g = orc.backward(qkv, dy, n_head, window=1)
    assert np.allclose(g[:, :, 2 * C:], dy, rtol=0, atol=1e-15)
    assert np.abs(g[:, :, :2 * C]).max() < 1e-15


def pin_window_covers_all(orc):
    """A window at least T wide hides nothing the causal mask does not: the
    results equal the causal oracle's bit for bit."""
    B, T, n_head, hs = 2, 13, 2, 3
    C = n_head * hs
    r = _rng(31)
    qkv = r.standard_normal((B, T, 3 * C))
    dy = r.standard_normal((B, T, C))
    y0, l0 = orc.forward(qkv, n_head)
    g0 = orc.backward(qkv, dy, n_head)
    for w in (T, T + 5):
        y, l = orc.forward(qkv, n_head, window=w)
        assert np.array_equal(y, y0) and np.array_equal(l, l0)
        assert np.array_equal(orc.backward(qkv, dy, n_head, window=w), g0)


def pin_window_uniform_scores(orc):
    """Zero queries: the weights are uniform over the band, so y[t] is the mean of
    v over max(0, t-window+1)..t and lse[t] = ln(band size)."""
    B, T, n_head, hs, w = 2, 17, 2, 3, 5
    C = n_head * hs
    qkv = _rng(32).standard_normal((B, T, 3 * C))
    qkv[:, :, :C] = 0.0
    y, lse = orc.forward(qkv, n_head, window=w)
    v = qkv[:, :, 2 * C:]
    for t in range(T):
        lo = max(0, t - w + 1)
        total = np.zeros((B, C))
        for s in range(lo, t + 1):
            total += v[:, s]
        assert np.allclose(y[:, t], total / (t - lo + 1), rtol=0, atol=1e-14)
        assert np.allclose(lse[:, :, t], math.log(t - lo + 1), rtol=0, atol=1e-14)


def pin_window_locality(orc):
    """Tokens before the band of position t (s <= t-window) do not reach it:
    perturbing them leaves y[t], lse[t] bit-identical; perturbing a token inside
    the band changes y[t]."""
    B, T, n_head, hs, w = 1, 16, 2, 4, 4
    C = n_head * hs
    r = _rng(33)
    qkv = r.standard_normal((B, T, 3 * C))
    y0, l0 = orc.forward(qkv, n_head, window=w)
    t = 12
    q2 = qkv.copy()
    q2[:, :t - w + 1] += r.standard_normal(q2[:, :t - w + 1].shape)
    y1, l1 = orc.forward(q2, n_head, window=w)
    assert np.array_equal(y1[:, t], y0[:, t]) and np.array_equal(l1[:, :, t], l0[:, :, t])
    q3 = qkv.copy()
    q3[:, t - w + 1] += 1.0
    y2, _ = orc.forward(q3, n_head, window=w)
    assert not np.allclose(y2[:, t], y0[:, t])


def pin_window_library_special_case(orc):
    """A different implementation: PyTorch scaled_dot_product_attention with an
    explicit boolean band mask, and autograd, in fp64 on the CPU."""
    B, T, n_head, hs, w = 2, 29, 2, 8, 7
    C = n_head * hs
    r = _rng(34)
    qkv = r.standard_normal((B, T, 3 * C))
    dy = r.standard_normal((B, T, C))
    x = torch.tensor(qkv, dtype=torch.float64, requires_grad=True)
    q, k, v = x.split(C, dim=2)
    heads = lambda a: a.view(B, T, n_head, hs).transpose(1, 2)
    tt = torch.arange(T)
    band = (tt[None, :] <= tt[:, None]) & (tt[None, :] > tt[:, None] - w)   # [t, s] visible
    out = torch.nn.functional.scaled_dot_product_attention(heads(q), heads(k), heads(v), attn_mask=band)
    y_ref = out.transpose(1, 2).reshape(B, T, C)
    (y_ref * torch.tensor(dy)).sum().backward()
    y, lse = orc.forward(qkv, n_head, window=w)
    g = orc.backward(qkv, dy, n_head, window=w)
    assert np.abs(y - y_ref.detach().numpy()).max() < 1e-12
    assert np.abs(g - x.grad.numpy()).max() < 1e-12
    s = heads(q).detach() @ heads(k).detach().transpose(-1, -2) / math.sqrt(hs)
    s = s.masked_fill(~band, float("-inf"))
    assert np.abs(lse - torch.logsumexp(s, -1).numpy()).max() < 1e-12


def pin_window_finite_differences(orc):
    """The windowed backward is the gradient of sum(y * dy): central differences."""
    B, T, n_head, hs, w = 1, 7, 2, 3, 3
    C = n_head * hs
    r = _rng(35)
    qkv = r.standard_normal((B, T, 3 * C))
    G = r.standard_normal((B, T, C))
    grad = orc.backward(qkv, G, n_head, window=w)
    h = 1e-6
    fd = np.zeros_like(qkv)
    flat = qkv.reshape(-1)
    for i in range(flat.size):
        xp = flat.copy()
        xm = flat.copy()
        xp[i] += h
        xm[i] -= h
        yp, _ = orc.forward(xp.reshape(qkv.shape), n_head, window=w)
        ym, _ = orc.forward(xm.reshape(qkv.shape), n_head, window=w)
        fd.reshape(-1)[i] = ((yp * G).sum() - (ym * G).sum()) / (2 * h)
    err = np.abs(fd - grad).max() / np.abs(grad).max()
    assert err < 1e-6, f"finite-difference mismatch {err:.3e}"


# ---- dropout on the attention weights --------------------------------------------

def _mask_probe(orc, p, seed, T=64, n_head=2):
    """Zero queries (uniform weights) and v = the identity (hs = T): then
    y[t][h*T + s] = f(t, s) / (t + 1) exposes the dropout factor f of every weight."""
    hs = T
    C = n_head * hs
    qkv = np.zeros((1, T, 3 * C))
    qkv[0, :, C:2 * C] = _rng(40).standard_normal((T, C))   # keys: irrelevant when q = 0
    for h in range(n_head):
        qkv[0, :, 2 * C + h * hs:2 * C + (h + 1) * hs] = np.eye(T)
    y, _ = orc.forward(qkv, n_head, dropout=p, seed=seed)
    f = np.zeros((n_head, T, T))
    for h in range(n_head):
        f[h] = y[0, :, h * hs:(h + 1) * hs] * (np.arange(T)[:, None] + 1)
    return f


def _theta(p):
    """The 8-bit drop threshold: round(256 p), at most 255."""
    return min(255, math.floor(256 * p + 0.5))


def pin_dropout_mask_and_scale(orc):
    """Inverted dropout with p applied in steps of 1/256: every visible weight is
    either 0 or scaled by exactly 1/(1 - theta/256), theta = round(256 p) (77 for
    p = 0.3); none above the diagonal; the keep rate is 1 - theta/256 (binomial, 5
    sigma); the two heads get different masks."""
    p = 0.3
    f = _mask_probe(orc, p, seed=11)
    T = f.shape[1]
    tril = np.tril(np.ones((T, T), dtype=bool))
    vals = f[:, tril]
    assert _theta(p) == 77
    p = _theta(p) / 256.0
    kept = np.abs(vals - 1.0 / (1.0 - p)) < 1e-12
    dropped = np.abs(vals) < 1e-15
    assert np.all(kept | dropped)
    assert np.all(np.abs(f[:, ~tril]) < 1e-15)
    n = vals.size
    rate = kept.mean()
    assert abs(rate - (1 - p)) < 5 * math.sqrt(p * (1 - p) / n)
    assert not np.array_equal(kept.reshape(2, -1)[0], kept.reshape(2, -1)[1])


def pin_dropout_counter_layout(orc):
    """Weight (t, s) of batch-head pair bh is kept iff byte s%4 (least significant
    first) of word t%4 of Philox4x32-10 at counter (s/4, t/4, bh, 0) under key (seed
    low, seed high) is >= round(256 p): the mapping the CUDA path must follow too."""
    p, seed = 0.45, (7 << 32) | 12345
    f = _mask_probe(orc, p, seed=seed, T=48, n_head=2)
    thr = _theta(p)
    assert thr == 115
    for h in range(2):
        for t in range(48):
            for s_ in range(t + 1):
                r = orc.philox([s_ // 4, t // 4, h, 0], [seed & 0xFFFFFFFF, seed >> 32])
                assert (((r[t % 4] >> (8 * (s_ % 4))) & 0xFF) >= thr) == (f[h, t, s_] > 0), (h, t, s_)


def pin_dropout_lse_unchanged_and_unbiased(orc):
    """lse is that of the undropped weights (bit-identical); averaged over many
    seeds the output approaches the undropped output (inverted dropout is unbiased)."""
    B, T, n_head, hs, p = 1, 12, 1, 4, 0.5
    C = n_head * hs
    qkv = _rng(41).standard_normal((B, T, 3 * C))
    y0, l0 = orc.forward(qkv, n_head)
    acc = np.zeros_like(y0)
    N = 400
    for k in range(N):
        y, l = orc.forward(qkv, n_head, dropout=p, seed=1000 + k)
        assert np.array_equal(l, l0)
        acc += y
    mean = acc / N
    # per element the estimator's std is at most max|v| * sqrt(p/(1-p)) / sqrt(N)
    bound = 5 * np.abs(qkv[:, :, 2 * C:]).max() * math.sqrt(p / (1 - p)) / math.sqrt(N)
    assert np.abs(mean - y0).max() < bound


def pin_dropout_finite_differences(orc):
    """With the mask fixed by the seed, the backward is the gradient of sum(y * dy)."""
    B, T, n_head, hs, p, seed = 1, 6, 2, 3, 0.4, 99
    C = n_head * hs
    r = _rng(42)
    qkv = r.standard_normal((B, T, 3 * C))
    G = r.standard_normal((B, T, C))
    grad = orc.backward(qkv, G, n_head, dropout=p, seed=seed)
    h = 1e-6
    fd = np.zeros_like(qkv)
    flat = qkv.reshape(-1)
    for i in range(flat.size):
        xp = flat.copy()
        xm = flat.copy()
        xp[i] += h
        xm[i] -= h
        yp, _ = orc.forward(xp.reshape(qkv.shape), n_head, dropout=p, seed=seed)
        ym, _ = orc.forward(xm.reshape(qkv.shape), n_head, dropout=p, seed=seed)
        fd.reshape(-1)[i] = ((yp * G).sum() - (ym * G).sum()) / (2 * h)
    err = np.abs(fd - grad).max() / np.abs(grad).max()
    assert err < 1e-6, f"finite-difference mismatch {err:.3e}"


def pin_philox_statistics(orc):
    """The generator's words look uniform: mean, every bit's frequency and a 16-bin
    chi-square over 4096 counters (4 words each) within generous bounds."""
    words = []
    for i in range(4096):
        words += orc.philox([i, 3 * i, 7, 0], [0x1234, 0x5678])
    w = np.array(words, dtype=np.float64)
    n = w.size
    u = w / 2.0 ** 32
    assert abs(u.mean() - 0.5) < 5 * math.sqrt(1 / 12 / n)
    wi = np.array(words, dtype=np.uint64)
    for bit in range(32):
        freq = ((wi >> bit) & 1).mean()
        assert abs(freq - 0.5) < 5 * math.sqrt(0.25 / n)
    counts = np.bincount((u * 16).astype(int), minlength=16)
    chi2 = ((counts - n / 16) ** 2 / (n / 16)).sum()
    assert chi2 < 50  # 15 degrees of freedom: P(chi2 > 50) is about 1e-5


def pin_philox_known_answers(orc):
    """Philox4x32-10 reproduces the generator's published known-answer vectors
    (the Random123 library's list for philox4x32 with 10 rounds, which accompanies
    Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011): the
    round count, both multipliers, the word permutation and the key schedule are
    all fixed by these three outputs."""
    fx = json.load(open(os.path.join(GOLDEN, "philox4x32_10_kat.json")))
    assert fx["rounds"] == 10 and len(fx["vectors"]) == 3
    for v in fx["vectors"]:
        ctr = [int(w, 16) for w in v["ctr"]]
        key = [int(w, 16) for w in v["key"]]
        want = [int(w, 16) for w in v["out"]]
        got = [int(w) for w in orc.philox(ctr, key)]
        assert got == want, f"philox({v['ctr']}, {v['key']}) = {[f'{w:08x}' for w in got]}, want {v['out']}"


ALL_PINS = [
    pin_row_identity,
    pin_single_token, pin_uniform_scores_prefix_mean, pin_tril_average_fixture,
    pin_rows_are_distributions, pin_weights_from_softmax_of_scaled_scores,
    pin_worked_two_heads, pin_causality, pin_batch_independence, pin_head_permutation,
    pin_set_semantics, pin_finite_differences, pin_library_special_case,
    pin_regression_fixture, pin_empty,
    pin_window_one, pin_window_covers_all, pin_window_uniform_scores, pin_window_locality,
    pin_window_library_special_case, pin_window_finite_differences,
    pin_dropout_mask_and_scale, pin_dropout_counter_layout, pin_dropout_lse_unchanged_and_unbiased,
    pin_dropout_finite_differences, pin_philox_statistics, pin_philox_known_answers,
]
