"""Pins of the fp64 oracle against facts the pages and mathematics fix.

Each test is chosen so that a plausible mistake in the oracle fails it:
  * a dropped residual / wrong sign / transposed weight  -> closed forms at N=1, N=2
  * a wrong softmax scale or key source (input vs output) -> N=2 closed form
  * an off-by-one in the lowbit block ranges              -> brute-force coverage,
                                                             blocked == naive
  * a wrong head split or missing mask                    -> textbook causal layer
  * a tanh-approximate GELU or misplaced eps              -> GELU / RMS values
Source of the method: "Recurrent Transformer" paper page (www.lshu.cn/news/403416):
paper §2 (notation: RMS, Attn), §2.1 (Transformer layer), §2.2 (RT layer,
temporary and persistent pairs), notes §4.2 (blocked schedule, exactness).
"""
import math
import os

import numpy as np
import pytest

import rtinputs
from oracle import rt_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _problem(B, N, d, H, d_ff, sigma=0.02, seed=0):
    W = rtinputs.weights(seed, d, d_ff, sigma=sigma, dtype="f32")
    x = rtinputs.x_batch(seed, range(B), N, d, dtype="f32")
    return x, W


def _relerr(a, b):
    return np.max(np.abs(a - b)) / np.max(np.abs(b))


# --------------------------------------------------------------------------
# scalar building blocks, against textbook values
# --------------------------------------------------------------------------
def test_gelu_matches_normal_cdf_values():
    # GELU(y) = y * Phi(y); Phi(1) = 0.8413447460685429, Phi(2) = 0.9772498680518208
    # (standard normal table values). The tanh approximation gives 0.841192 at 1.
    g = O.gelu(np.array([0.0, 1.0, -1.0, 2.0]))
    assert g[0] == 0.0
    assert abs(g[1] - 0.8413447460685429) < 1e-15
    assert abs(g[2] - (-1.0) * (1 - 0.8413447460685429)) < 1e-15
    assert abs(g[3] - 2 * 0.9772498680518208) < 1e-15


def test_rms_definition():
    # RMS(x) = x / sqrt(mean x^2 + eps): [3, 4] has mean square 12.5.
    r = O.rms(np.array([3.0, 4.0]))
    np.testing.assert_allclose(r, np.array([3.0, 4.0]) / math.sqrt(12.5 + 1e-6), rtol=0, atol=1e-15)
    # output has mean square 1 up to the eps term
    v = np.random.default_rng(1).standard_normal(64) * 5
    r = O.rms(v)
    ms = np.mean(v * v)
    assert abs(np.mean(r * r) - ms / (ms + 1e-6)) < 1e-14


# --------------------------------------------------------------------------
# the schedule
# --------------------------------------------------------------------------
def test_lowbit_worked_example_from_pages():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "lowbit_worked_example.txt"))
            if l.strip() and not l.startswith("#")]
    for t, lb, q0, q1 in (map(int, r) for r in rows):
        assert O.lowbit(t) == lb
        blocks = {tt: (keys, qs) for tt, keys, qs in O.lowbit_blocks(16)}
        keys, qs = blocks[t]
        assert qs == list(range(q0, q1 + 1))
        assert keys == list(range(t - lb + 1, t + 1))


def test_lowbit_values():
    assert [O.lowbit(t) for t in range(1, 17)] == [1, 2, 1, 4, 1, 2, 1, 8, 1, 2, 1, 4, 1, 2, 1, 16]
    with pytest.raises(ValueError):
        O.lowbit(0)


@pytest.mark.parametrize("N", list(range(1, 65)) + [100, 127, 128, 129, 255, 256])
def test_schedule_covers_every_causal_pair_exactly_once(N):
    count = np.zeros((N + 1, N + 1), dtype=np.int64)
    for t, keys, queries in O.lowbit_blocks(N):
        for j in queries:
            assert t < j, "a fold must happen before its query is finalised"
            for i in keys:
                assert i <= t, "a key can only be folded once revealed"
                count[j, i] += 1
    for j in range(1, N + 1):
        for i in range(1, N + 1):
            assert count[j, i] == (1 if i < j else 0), (j, i)


# --------------------------------------------------------------------------
# exactness of the blocked schedule (notes §4.2: equal up to FP reordering)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("N", [1, 2, 3, 7, 8, 64])
def test_blocked_equals_naive(N):
    x, W = _problem(2, N, 16, 2, 32, sigma=0.3)
    zn, Kn, Vn = O.rt_layer(x, W, 2)
    zb, Kb, Vb = O.rt_layer_blocked(x, W, 2)
    for a, b in ((zb, zn), (Kb, Kn), (Vb, Vn)):
        assert _relerr(a, b) < 1e-12


def test_blocked_equals_naive_peaky_attention():
    # sigma = 0.2 at d=64 makes softmax peaky, exercising the max-rescaling path.
    x, W = _problem(2, 40, 64, 2, 128, sigma=0.2)
    zn, Kn, Vn = O.rt_layer(x, W, 2)
    zb, Kb, Vb = O.rt_layer_blocked(x, W, 2)
    for a, b in ((zb, zn), (Kb, Kn), (Vb, Vn)):
        assert _relerr(a, b) < 1e-12
    # confirm peakiness: over all queries and heads, some query puts most of
    # its mass on one key and the score spread is wide
    best, spread = 0.0, 0.0
    for t in range(1, 40):
        r = O.rms(x[0, t])
        q = r @ W["W_q"].T
        for h in range(2):
            sl = slice(32 * h, 32 * h + 32)
            s = (Kn[0, :t, sl] @ q[sl]) / math.sqrt(32)
            p = np.exp(s - s.max()); p /= p.sum()
            best, spread = max(best, p.max()), max(spread, s.max() - s.min())
    assert best > 0.5 and spread > 8


# --------------------------------------------------------------------------
# the fold on its own
# --------------------------------------------------------------------------
def test_block_fold_equals_direct_softmax_and_is_associative():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((5, 8)); k = rng.standard_normal((7, 8)); v = rng.standard_normal((7, 8))
    sc = 0.7
    m0 = np.full(5, -np.inf); l0 = np.zeros(5); o0 = np.zeros((5, 8))
    m, l, o = O.block_fold(q, k, v, m0, l0, o0, sc)
    # direct: softmax rows (explicit loops)
    for a in range(5):
        s = [sc * sum(q[a, e] * k[i, e] for e in range(8)) for i in range(7)]
        mx = max(s)
        w = [math.exp(si - mx) for si in s]
        ref = [sum(w[i] * v[i, e] for i in range(7)) / sum(w) for e in range(8)]
        np.testing.assert_allclose(o[a] / l[a], ref, rtol=1e-13, atol=1e-14)
        assert abs(m[a] - mx) < 1e-14 * abs(mx)
    # two halves folded one after the other = one fold
    m1, l1, o1 = O.block_fold(q, k[:3], v[:3], m0, l0, o0, sc)
    m2, l2, o2 = O.block_fold(q, k[3:], v[3:], m1, l1, o1, sc)
    np.testing.assert_allclose(o2 / l2[:, None], o / l[:, None], rtol=1e-13)


# --------------------------------------------------------------------------
# closed forms (pure-Python loops, independent of the oracle's helpers)
# --------------------------------------------------------------------------
def _py_rms(v):
    ms = sum(e * e for e in v) / len(v)
    return [e / math.sqrt(ms + 1e-6) for e in v]


def _py_mv(Wm, v):
    return [sum(Wm[i][j] * v[j] for j in range(len(v))) for i in range(len(Wm))]


def _py_gelu(y):
    return 0.5 * y * (1.0 + math.erf(y / math.sqrt(2.0)))


def _py_layer_tail(x, a, W):
    """u = x + W_o a ; z = u + W_2 GELU(W_1 RMS(u))."""
    u = [xi + oi for xi, oi in zip(x, _py_mv(W["W_o"], a))]
    h = [_py_gelu(e) for e in _py_mv(W["W_1"], _py_rms(u))]
    return [ui + mi for ui, mi in zip(u, _py_mv(W["W_2"], h))]


def test_N1_closed_form_single_token_layer():
    # With one position, softmax over the single temporary key is 1, so
    # a = v~ = W_v RMS(x), and the layer is one pre-norm layer on one token.
    d, H, d_ff = 8, 2, 16
    x, W = _problem(3, 1, d, H, d_ff, sigma=0.4)
    z, K, V = O.rt_layer(x, W, H)
    Wl = {k: v.tolist() for k, v in W.items()}
    for b in range(3):
        xb = x[b, 0].tolist()
        a = _py_mv(Wl["W_v"], _py_rms(xb))
        zb = _py_layer_tail(xb, a, Wl)
        np.testing.assert_allclose(z[b, 0], zb, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(K[b, 0], _py_mv(Wl["W_k"], _py_rms(zb)), rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(V[b, 0], _py_mv(Wl["W_v"], _py_rms(zb)), rtol=1e-13, atol=1e-14)


def test_N2_closed_form_persistent_key_from_output():
    # Position 2 attends to {persistent (k1, v1) from z1} + {temporary (k~2, v~2)}.
    # Two-way softmax = logistic: a = sig(s1 - s2) v1 + sig(s2 - s1) v~2, per head,
    # with s = <k, q> / sqrt(d_h).
    d, H, d_ff = 8, 2, 16
    dh = d // H
    x, W = _problem(2, 2, d, H, d_ff, sigma=0.5)
    z, K, V = O.rt_layer(x, W, H)
    Wl = {k: v.tolist() for k, v in W.items()}
    sig = lambda y: 1.0 / (1.0 + math.exp(-y))
    for b in range(2):
        x1, x2 = x[b, 0].tolist(), x[b, 1].tolist()
        z1 = _py_layer_tail(x1, _py_mv(Wl["W_v"], _py_rms(x1)), Wl)
        k1 = _py_mv(Wl["W_k"], _py_rms(z1)); v1 = _py_mv(Wl["W_v"], _py_rms(z1))
        r2 = _py_rms(x2)
        q2 = _py_mv(Wl["W_q"], r2); kt = _py_mv(Wl["W_k"], r2); vt = _py_mv(Wl["W_v"], r2)
        a = []
        for h in range(H):
            sl = slice(h * dh, (h + 1) * dh)
            s1 = sum(p * r for p, r in zip(q2[sl], k1[sl])) / math.sqrt(dh)
            s2 = sum(p * r for p, r in zip(q2[sl], kt[sl])) / math.sqrt(dh)
            a += [sig(s1 - s2) * e1 + sig(s2 - s1) * e2 for e1, e2 in zip(v1[sl], vt[sl])]
        z2 = _py_layer_tail(x2, a, Wl)
        np.testing.assert_allclose(z[b, 0], z1, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(z[b, 1], z2, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(K[b, 0], k1, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(V[b, 1], _py_mv(Wl["W_v"], _py_rms(z2)), rtol=1e-12, atol=1e-13)


def test_decode_step_N1_closed_form():
    # an empty cache: the step is the single-token layer of the closed form above
    d, H, d_ff = 8, 2, 16
    x, W = _problem(3, 1, d, H, d_ff, sigma=0.4)
    Wl = {k: v.tolist() for k, v in W.items()}
    z, k, v = O.rt_decode_step(x[:, 0], W, H, np.zeros((3, 0, d)), np.zeros((3, 0, d)))
    for b in range(3):
        xb = x[b, 0].tolist()
        zb = _py_layer_tail(xb, _py_mv(Wl["W_v"], _py_rms(xb)), Wl)
        np.testing.assert_allclose(z[b], zb, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(k[b], _py_mv(Wl["W_k"], _py_rms(zb)), rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(v[b], _py_mv(Wl["W_v"], _py_rms(zb)), rtol=1e-13, atol=1e-14)


def test_decode_from_empty_cache_reproduces_the_layer():
    # Autoregressive consistency: feeding each step's own (k_t, v_t) back as
    # cache reproduces the whole-sequence layer (naive definition and the
    # blocked schedule), peaky attention included.
    for sigma in (0.02, 0.3):
        x, W = _problem(2, 19, 16, 2, 32, sigma=sigma)
        z, K, V = O.rt_layer(x, W, 2)
        zb, Kb, Vb = O.rt_layer_blocked(x, W, 2)
        Kc = np.zeros((2, 0, 16)); Vc = np.zeros((2, 0, 16))
        for t in range(19):
            zt, kt, vt = O.rt_decode_step(x[:, t], W, 2, Kc, Vc)
            for ref, got in ((z[:, t], zt), (K[:, t], kt), (V[:, t], vt), (zb[:, t], zt)):
                np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)
            Kc = np.concatenate([Kc, kt[:, None]], axis=1)
            Vc = np.concatenate([Vc, vt[:, None]], axis=1)


# --------------------------------------------------------------------------
# gradients (rt_layer_backward): central finite differences of rt_layer
# --------------------------------------------------------------------------
def _loss(x, W, H, dz, dK, dV):
    z, K, V = O.rt_layer(x, W, H)
    return float(np.sum(z * dz) + np.sum(K * dK) + np.sum(V * dV))


def test_checkpoint_recompute_rebuilds_the_persistent_pairs():
    # the sequential layer and the one-step parallel rebuild from its z agree
    x, W = _problem(3, 11, 16, 2, 32, sigma=0.3)
    z, K, V = O.rt_layer(x, W, 2)
    Kr, Vr = O.recompute_kv(z, W)
    np.testing.assert_allclose(Kr, K, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(Vr, V, rtol=1e-13, atol=1e-14)
    # and a persistent pair depends on its own position's output only
    z2 = z.copy(); z2[:, 5] += 1.0
    K2, _ = O.recompute_kv(z2, W)
    assert np.array_equal(np.delete(K2, 5, axis=1), np.delete(Kr, 5, axis=1))


def test_backward_matches_finite_differences():
    B, N, d, H, d_ff = 2, 4, 8, 2, 16
    x, W = _problem(B, N, d, H, d_ff, sigma=0.5)
    rng = np.random.default_rng(7)
    dz, dK, dV = (rng.standard_normal((B, N, d)) for _ in range(3))
    dx, dW, (z, K, V) = O.rt_layer_backward(x, W, H, dz, dK, dV)
    zr, Kr, Vr = O.rt_layer(x, W, H)
    np.testing.assert_allclose(z, zr, rtol=1e-12, atol=1e-13)      # the restated forward is the layer
    np.testing.assert_allclose(K, Kr, rtol=1e-12, atol=1e-13)
    h = 1e-5
    for idx in [(0, 0, 0), (1, 3, 5), (0, 2, 7), (1, 1, 2)]:
        xp = x.copy(); xp[idx] += h
        xm = x.copy(); xm[idx] -= h
        fd = (_loss(xp, W, H, dz, dK, dV) - _loss(xm, W, H, dz, dK, dV)) / (2 * h)
        assert abs(fd - dx[idx]) <= 1e-6 * max(1.0, abs(fd)), (idx, fd, dx[idx])
    for name, idx in [("W_q", (1, 2)), ("W_k", (3, 0)), ("W_v", (5, 6)), ("W_o", (0, 7)), ("W_1", (9, 4)),
                      ("W_2", (6, 13))]:
        Wp = {k: v.copy() for k, v in W.items()}; Wp[name][idx] += h
        Wm = {k: v.copy() for k, v in W.items()}; Wm[name][idx] -= h
        fd = (_loss(x, Wp, H, dz, dK, dV) - _loss(x, Wm, H, dz, dK, dV)) / (2 * h)
        assert abs(fd - dW[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, dW[name][idx])


def test_backward_is_causal():
    # a gradient on z at position s reaches only the inputs of positions <= s
    B, N, d, H, d_ff = 1, 6, 8, 2, 16
    x, W = _problem(B, N, d, H, d_ff, sigma=0.4)
    dz = np.zeros((B, N, d)); dz[0, 3] = 1.0
    zero = np.zeros((B, N, d))
    dx, _, _ = O.rt_layer_backward(x, W, H, dz, zero, zero)
    assert np.all(dx[0, 4:] == 0.0)
    assert np.all(np.abs(dx[0, :4]).max(axis=-1) > 0.0)


# --------------------------------------------------------------------------
# the paper's own parameterisation (rt_layer_pages): pure-Python closed forms
# --------------------------------------------------------------------------
def _py_rms_unit(v):
    """sqrt(D) v / ||v||_2 (paper §2 notation), no eps."""
    n = math.sqrt(sum(e * e for e in v))
    return [e * math.sqrt(len(v)) / n for e in v]


def _py_heads_rms_unit(v, H):
    dh = len(v) // H
    out = []
    for h in range(H):
        out += _py_rms_unit(v[h * dh:(h + 1) * dh])
    return out


def _py_pages_tail(x, a, W, L):
    """u = x + W_o a / sqrt(L); z = u + W_2 GELU(W_1 RMS(u)) / sqrt(L)."""
    c = 1.0 / math.sqrt(L)
    u = [xi + c * oi for xi, oi in zip(x, _py_mv(W["W_o"], a))]
    h = [_py_gelu(e) for e in _py_mv(W["W_1"], _py_rms_unit(u))]
    return [ui + c * mi for ui, mi in zip(u, _py_mv(W["W_2"], h))]


def test_pages_parameterisation_N1_N2_closed_forms():
    # N = 1: one key, a = v~ = W_v RMS(x). N = 2: per head a two-way softmax
    # (logistic) of the unscaled scores <k1, q2>, <k~2, q2> with per-head
    # unit-RMS keys and queries (|score| <= d_h by Cauchy-Schwarz).
    d, H, d_ff, L = 8, 2, 16, 4
    dh = d // H
    x, W = _problem(2, 2, d, H, d_ff, sigma=0.5)
    z, K, V = O.rt_layer_pages(x, W, H, L=L)
    Wl = {k: v.tolist() for k, v in W.items()}
    sig = lambda y: 1.0 / (1.0 + math.exp(-y))
    for b in range(2):
        x1, x2 = x[b, 0].tolist(), x[b, 1].tolist()
        r1 = _py_rms_unit(x1)
        z1 = _py_pages_tail(x1, _py_mv(Wl["W_v"], r1), Wl, L)
        rz1 = _py_rms_unit(z1)
        k1 = _py_heads_rms_unit(_py_mv(Wl["W_k"], rz1), H)
        v1 = _py_mv(Wl["W_v"], rz1)
        r2 = _py_rms_unit(x2)
        q2 = _py_heads_rms_unit(_py_mv(Wl["W_q"], r2), H)
        kt = _py_heads_rms_unit(_py_mv(Wl["W_k"], r2), H)
        vt = _py_mv(Wl["W_v"], r2)
        a = []
        for h in range(H):
            sl = slice(h * dh, (h + 1) * dh)
            s1 = sum(p * r for p, r in zip(q2[sl], k1[sl]))
            s2 = sum(p * r for p, r in zip(q2[sl], kt[sl]))
            assert abs(s1) <= dh + 1e-9 and abs(s2) <= dh + 1e-9
            a += [sig(s1 - s2) * e1 + sig(s2 - s1) * e2 for e1, e2 in zip(v1[sl], vt[sl])]
        z2 = _py_pages_tail(x2, a, Wl, L)
        np.testing.assert_allclose(z[b, 0], z1, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(K[b, 0], k1, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(V[b, 0], v1, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(z[b, 1], z2, rtol=1e-11, atol=1e-12)
        rz2 = _py_rms_unit(z2)
        np.testing.assert_allclose(K[b, 1], _py_heads_rms_unit(_py_mv(Wl["W_k"], rz2), H), rtol=1e-11, atol=1e-12)


def test_pages_parameterisation_standard_layer_reduction():
    # kv_source="input" is the paper's standard layer (§2.1): one masked score
    # matrix per head with per-head unit-RMS q and k and no softmax scale
    B, N, d, H, d_ff, L = 2, 9, 16, 4, 32, 3
    dh = d // H
    x, W = _problem(B, N, d, H, d_ff, sigma=0.3)
    z, K, V = O.rt_layer_pages(x, W, H, L=L, kv_source="input")
    unit = lambda v: v * np.sqrt(v.shape[-1]) / np.sqrt(np.sum(v * v, axis=-1, keepdims=True))
    r = unit(x)
    q = unit((r @ W["W_q"].T).reshape(B, N, H, dh)).transpose(0, 2, 1, 3)
    k = unit((r @ W["W_k"].T).reshape(B, N, H, dh)).transpose(0, 2, 1, 3)
    v = (r @ W["W_v"].T).reshape(B, N, H, dh).transpose(0, 2, 1, 3)
    S = q @ k.transpose(0, 1, 3, 2)
    S = np.where(np.triu(np.ones((N, N), dtype=bool), k=1), -np.inf, S)
    P = np.exp(S - S.max(axis=-1, keepdims=True))
    P /= P.sum(axis=-1, keepdims=True)
    a = (P @ v).transpose(0, 2, 1, 3).reshape(B, N, d)
    u = x + (a @ W["W_o"].T) / np.sqrt(L)
    hid = unit(u) @ W["W_1"].T
    zr = u + ((0.5 * hid * (1.0 + np.vectorize(math.erf)(hid / math.sqrt(2.0)))) @ W["W_2"].T) / np.sqrt(L)
    np.testing.assert_allclose(z, zr, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(K, k.transpose(0, 2, 1, 3).reshape(B, N, d), rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# standard-layer special case (paper §2.1): a textbook causal pre-norm layer
# written as one masked score matrix per head
# --------------------------------------------------------------------------
def _textbook_causal_layer(x, W, H):
    B, N, d = x.shape
    dh = d // H
    ms = np.mean(x * x, axis=-1, keepdims=True)
    r = x / np.sqrt(ms + 1e-6)
    q = (r @ W["W_q"].T).reshape(B, N, H, dh).transpose(0, 2, 1, 3)
    k = (r @ W["W_k"].T).reshape(B, N, H, dh).transpose(0, 2, 1, 3)
    v = (r @ W["W_v"].T).reshape(B, N, H, dh).transpose(0, 2, 1, 3)
    S = q @ k.transpose(0, 1, 3, 2) / np.sqrt(dh)                 # [B,H,N,N]
    mask = np.triu(np.ones((N, N), dtype=bool), k=1)              # key index > query index
    S = np.where(mask, -np.inf, S)
    P = np.exp(S - S.max(axis=-1, keepdims=True))
    P /= P.sum(axis=-1, keepdims=True)
    a = (P @ v).transpose(0, 2, 1, 3).reshape(B, N, d)
    u = x + a @ W["W_o"].T
    ru = u / np.sqrt(np.mean(u * u, axis=-1, keepdims=True) + 1e-6)
    pre = ru @ W["W_1"].T
    from scipy.stats import norm
    y = u + (pre * norm.cdf(pre)) @ W["W_2"].T
    return y, k.transpose(0, 2, 1, 3).reshape(B, N, d), v.transpose(0, 2, 1, 3).reshape(B, N, d)


@pytest.mark.parametrize("N,H", [(1, 1), (5, 2), (33, 4)])
def test_input_kv_source_is_the_textbook_transformer_layer(N, H):
    x, W = _problem(2, N, 16, H, 48, sigma=0.3)
    z, K, V = O.rt_layer(x, W, H, kv_source="input")
    zt, Kt, Vt = _textbook_causal_layer(x, W, H)
    assert _relerr(z, zt) < 1e-12
    assert _relerr(K, Kt) < 1e-12
    assert _relerr(V, Vt) < 1e-12


def test_rt_reduces_to_transformer_when_branches_vanish_and_differs_otherwise():
    # With W_o = 0 and W_2 = 0 the layer output equals its input (z = x), so the
    # persistent pair from z equals the one from x.
    x, W = _problem(2, 12, 16, 2, 32, sigma=0.3)
    W0 = dict(W, W_o=np.zeros_like(W["W_o"]), W_2=np.zeros_like(W["W_2"]))
    a = O.rt_layer(x, W0, 2)
    b = O.rt_layer(x, W0, 2, kv_source="input")
    for u, v in zip(a, b):
        assert _relerr(u, v) < 1e-14
    zr, _, _ = O.rt_layer(x, W, 2)
    zt, _, _ = O.rt_layer(x, W, 2, kv_source="input")
    assert np.max(np.abs(zr - zt)) > 1e-6


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------
def test_prefix_batch_permutation_and_causality():
    x, W = _problem(3, 20, 16, 2, 32, sigma=0.3)
    z, K, V = O.rt_layer(x, W, 2)
    # prefix: running the first 11 positions gives the first 11 outputs
    zp, Kp, Vp = O.rt_layer(x[:, :11], W, 2)
    np.testing.assert_array_equal(zp, z[:, :11])
    np.testing.assert_array_equal(Kp, K[:, :11])
    # batch permutation permutes outputs (sequences are independent)
    perm = [2, 0, 1]
    zq, _, _ = O.rt_layer(x[perm], W, 2)
    np.testing.assert_allclose(zq, z[perm], rtol=1e-14, atol=1e-14)
    # causality: perturbing x at position 15 leaves positions < 15 unchanged
    x2 = x.copy(); x2[:, 14] += 1.0
    z2, _, _ = O.rt_layer(x2, W, 2)
    np.testing.assert_array_equal(z2[:, :14], z[:, :14])
    assert np.max(np.abs(z2[:, 14:] - z[:, 14:])) > 1e-3


def test_stack_chains_layers():
    vocab, d, H, d_ff = 50, 16, 2, 32
    E = rtinputs.embedding(0, vocab, d, dtype="f32")
    ids = np.stack([rtinputs.token_ids(0, b, 6, vocab) for b in range(2)])
    layers = [rtinputs.weights(0, d, d_ff, sigma=0.3, dtype="f32", layer=i) for i in range(3)]
    zs, kv = O.rt_stack(ids, E, layers, H)
    x = E[ids]
    for i, W in enumerate(layers):
        x, K, V = O.rt_layer(x, W, H)
        np.testing.assert_array_equal(K, kv[i][0])
    np.testing.assert_array_equal(x, zs)


def test_embedding_lookup_row_by_row():
    # The stack's front end is a table lookup (the token id selects a row of
    # the embedding table; RT paper §6.1 feeds the embedded tokens to the
    # first layer). Hand-chosen ids -- the first and last rows of the table,
    # repeats, and a [B, N] layout -- are checked one by one against a loop
    # that copies the row by explicit index, so a transposed table, an
    # off-by-one id or a flattened batch axis fails.
    vocab, d = 7, 5
    E = np.arange(vocab * d, dtype=np.float64).reshape(vocab, d) * 0.5 - 3.0
    ids = np.array([[0, 6, 3], [6, 6, 0]], dtype=np.int32)
    x = O.embed(ids, E)
    assert x.shape == (2, 3, d)
    for b in range(ids.shape[0]):
        for n in range(ids.shape[1]):
            row = [E[int(ids[b, n]), e] for e in range(d)]
            assert list(x[b, n]) == row
    # row 0 of the table is -3.0, -2.5, ... and row vocab-1 ends at the last entry
    assert list(x[0, 0]) == [-3.0, -2.5, -2.0, -1.5, -1.0]
    assert x[0, 1, -1] == E.flat[-1] == (vocab * d - 1) * 0.5 - 3.0


# --------------------------------------------------------------------------
# block-wise (chunked) recurrence: the two ends of the depth/speed trade-off
# --------------------------------------------------------------------------
def test_chunked_recurrence_with_chunks_of_one_is_the_rt_layer():
    x, W = _problem(2, 13, 32, 2, 64, sigma=0.2)
    got = O.rt_layer_chunked(x, W, 2, 1)
    ref = O.rt_layer(x, W, 2)
    for g, r in zip(got, ref):
        assert _relerr(g, r) < 1e-12


@pytest.mark.parametrize("N,C", [(9, 9), (9, 16)])
def test_chunked_recurrence_with_one_chunk_is_the_standard_layer(N, C):
    # every pair temporary: the causal pre-norm Transformer layer (its own
    # textbook pin is test_input_kv_source_is_the_textbook_transformer_layer)
    x, W = _problem(2, N, 32, 2, 64, sigma=0.2)
    z, K, V = O.rt_layer_chunked(x, W, 2, C)
    zr, _, _ = O.rt_layer(x, W, 2, kv_source="input")
    assert _relerr(z, zr) < 1e-12
    Kr, Vr = O.recompute_kv(z, W)               # persistent pairs of the outputs
    assert _relerr(K, Kr) < 1e-12 and _relerr(V, Vr) < 1e-12


def test_chunked_recurrence_two_positions_closed_form():
    # N = 2 in one chunk of 2: position 2 sees the TEMPORARY pairs of
    # positions 1 and 2 (with C = 1 it would see position 1's persistent pair)
    x, W = _problem(1, 2, 16, 1, 32, sigma=0.3)
    z, _, _ = O.rt_layer_chunked(x, W, 1, 2)
    r = O.rms(x[0])
    q, kt, vt = r @ W["W_q"].T, r @ W["W_k"].T, r @ W["W_v"].T
    s = np.array([q[1] @ kt[0], q[1] @ kt[1]]) / 4.0
    p = np.exp(s - s.max())
    p /= p.sum()
    a = p[0] * vt[0] + p[1] * vt[1]
    u = x[0, 1] + W["W_o"] @ a
    z2 = u + W["W_2"] @ O.gelu(W["W_1"] @ O.rms(u))
    assert _relerr(z[0, 1], z2) < 1e-12
    # position 1 attends to its own temporary pair only: a_1 = v~_1
    u1 = x[0, 0] + W["W_o"] @ vt[0]
    assert _relerr(z[0, 0], u1 + W["W_2"] @ O.gelu(W["W_1"] @ O.rms(u1))) < 1e-12


def test_chunked_recurrence_is_causal_and_chunk_local():
    x, W = _problem(1, 12, 32, 2, 64, sigma=0.2)
    z, _, _ = O.rt_layer_chunked(x, W, 2, 4)
    x2 = x.copy()
    x2[:, 9] += 1.0                              # chunk 2 (positions 9..12, 1-based)
    z2, _, _ = O.rt_layer_chunked(x2, W, 2, 4)
    np.testing.assert_array_equal(z2[:, :9], z[:, :9])
    assert np.max(np.abs(z2[:, 9:] - z[:, 9:])) > 1e-3
