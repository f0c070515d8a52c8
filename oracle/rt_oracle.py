"""Plain fp64 CPU oracle for one Recurrent Transformer (RT) layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or runs
this module: only the tests, the smoke check and the benchmark's CPU-baseline
leg do. It shares no code with the CUDA library.

Source (cited as [RT ...] below): "Recurrent Transformer" paper page,
www.lshu.cn/news/403416 -- a reader's summary notes ("notes") followed by a
translation of the paper ("paper").

  [RT paper §2, notation]    RMS(x) = sqrt(D) x / ||x||_2; the Attn operator
                             sum_i v_i exp<k_i,q> / sum_j exp<k_j,q>; multi-head
                             = the single-head rule per head, then the usual
                             output projection; pre-LN residual branches.
  [RT paper §2.1]            standard causal pre-norm Transformer layer.
  [RT paper §2.2]            RT layer: query and a *temporary* (k, v) from the
                             layer input x_i; *persistent* (k_i, v_i) from the
                             layer output z_i, stored for all later positions.
  [RT notes §2.2]            temporary vs persistent key/value pairs.
  [RT notes §4.1]            naive schedule: query t attends to all revealed KV.
  [RT paper §6.4]            backward pass (its body is missing from the
                             extracted text): gradients here are the exact
                             derivatives of the forward definition.
  [RT paper §7.3]            decoding: a new token costs one query against
                             the cached persistent pairs, as in a standard
                             Transformer (the recurrence is over positions
                             already in the cache).
  [RT notes §4.2]            blocked schedule: queries precomputed; when
                             (k_t, v_t) is revealed a block is folded into the
                             online-softmax statistics (m, l, o) of a batch of
                             future queries; block size = largest power of two
                             dividing t; exact up to floating-point reordering.

Readings where the pages are silent or garbled (the concrete layer follows the
single-layer configuration: pre-RMSNorm with eps 1e-6 and unit gain, no QK
norm, softmax scale 1/sqrt(d_h), no 1/sqrt(L) residual scaling):
  * RMS(v) = v / sqrt(mean(v^2) + 1e-6).
  * GELU is the exact erf form.
  * persistent k_t = W_k RMS(z_t), v_t = W_v RMS(z_t): the same projections
    as the temporary pair, applied to the output (the equations are cut off
    in the extracted text of §2.2).
  * a revealed block at step t folds keys (t - lowbit(t), t] into queries
    (t, t + lowbit(t)] (clipped at N); the notes' example "(k4, v4) updates
    a5..a8" is the query side of t = 4.
  * heads are contiguous slices of width d_h = d / H; their outputs are
    concatenated and multiplied by W_o.

Conventions: positions are 1-based in the comments (as on the pages) and
0-based in the arrays. Weights use nn.Linear orientation [out][in], y = W r.
All arithmetic is float64.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

EPS = 1e-6


# --------------------------------------------------------------------------
# building blocks
# --------------------------------------------------------------------------
def rms(v: np.ndarray) -> np.ndarray:
    """Root-mean-square normalisation over the last axis [RT paper §2,
    notation: RMS(x) = sqrt(D) x/||x||], with eps inside the square root and
    unit gain."""
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + EPS)


def gelu(y: np.ndarray) -> np.ndarray:
    """Exact GELU, y * Phi(y) = y/2 (1 + erf(y / sqrt 2))."""
    return 0.5 * y * (1.0 + erf(y / np.sqrt(2.0)))


def lowbit(t: int) -> int:
    """Largest power of two dividing t (t >= 1) [RT notes §4.2]."""
    if t < 1:
        raise ValueError("lowbit is defined for t >= 1")
    return t & -t


def mlp(u: np.ndarray, W: dict) -> np.ndarray:
    """W_2 GELU(W_1 RMS(u)) [RT paper §2.1, the MLP branch]."""
    return gelu(rms(u) @ W["W_1"].T) @ W["W_2"].T


def _heads(a: np.ndarray, H: int) -> np.ndarray:
    """[..., d] -> [..., H, d_h] (contiguous head slices)."""
    return a.reshape(a.shape[:-1] + (H, a.shape[-1] // H))


# --------------------------------------------------------------------------
# naive schedule = the definition of the layer
# --------------------------------------------------------------------------
def rt_layer(x: np.ndarray, W: dict, H: int, kv_source: str = "output"):
    """RT layer forward, naive per-step schedule [RT paper §2.2; notes §4.1].

    x: [B, N, d] float64. Returns (z, K, V), each [B, N, d]; K and V hold the
    persistent pairs (k_t, v_t), head h in columns h*d_h .. (h+1)*d_h - 1.

    For t = 1..N and every sequence b:
        r = RMS(x_t); q = W_q r; temporary k~ = W_k r, v~ = W_v r
        per head: a_h = Attn({(k_i, v_i): i < t} + {(k~, v~)}, q_h)
                  with scores <k, q_h> / sqrt(d_h)
        u = x_t + W_o a;  z_t = u + W_2 GELU(W_1 RMS(u))
        persistent (k_t, v_t) = (W_k RMS(s_t), W_v RMS(s_t))
    with s_t = z_t (the RT layer, kv_source="output") or s_t = x_t
    (kv_source="input": the persistent pair is the temporary one, i.e. the
    standard Transformer layer of [RT paper §2.1]).
    """
    if kv_source not in ("output", "input"):
        raise ValueError(kv_source)
    x = np.asarray(x, dtype=np.float64)
    B, N, d = x.shape
    dh = d // H
    scale = 1.0 / np.sqrt(dh)
    z = np.empty_like(x)
    Kp = np.empty((B, H, N, dh))          # persistent keys, per head
    Vp = np.empty((B, H, N, dh))
    for t in range(N):                    # position t+1
        r = rms(x[:, t])
        q = _heads(r @ W["W_q"].T, H)     # [B, H, dh]
        kt = _heads(r @ W["W_k"].T, H)
        vt = _heads(r @ W["W_v"].T, H)
        keys = np.concatenate([Kp[:, :, :t], kt[:, :, None]], axis=2)   # [B,H,t+1,dh]
        vals = np.concatenate([Vp[:, :, :t], vt[:, :, None]], axis=2)
        s = np.einsum("bhe,bhie->bhi", q, keys) * scale
        s = s - s.max(axis=-1, keepdims=True)
        w = np.exp(s)
        a = np.einsum("bhi,bhie->bhe", w, vals) / w.sum(axis=-1)[..., None]
        u = x[:, t] + a.reshape(B, d) @ W["W_o"].T
        zt = u + mlp(u, W)
        z[:, t] = zt
        src = zt if kv_source == "output" else x[:, t]
        rs = rms(src)
        Kp[:, :, t] = _heads(rs @ W["W_k"].T, H)
        Vp[:, :, t] = _heads(rs @ W["W_v"].T, H)
    K = Kp.transpose(0, 2, 1, 3).reshape(B, N, d)
    V = Vp.transpose(0, 2, 1, 3).reshape(B, N, d)
    return z, K, V


def rt_decode_step(x_t: np.ndarray, W: dict, H: int, K_prev: np.ndarray, V_prev: np.ndarray):
    """One autoregressive step of the RT layer [RT paper §7.3, §2.2].

    x_t: [B, d] inputs of position t; K_prev, V_prev: [B, t-1, d] persistent
    pairs of positions 1..t-1 (head h in columns h*d_h .. (h+1)*d_h - 1).
    Returns (z_t, k_t, v_t), each [B, d]: the new position's output and its
    persistent pair, which the caller appends to the cache.

    Query and temporary pair from RMS(x_t); per head, attention over the cached
    keys plus the temporary key with scores <k, q_h> / sqrt(d_h); then W_o,
    residual, MLP, and (k_t, v_t) = (W_k RMS(z_t), W_v RMS(z_t)).
    """
    x_t = np.asarray(x_t, dtype=np.float64)
    B, d = x_t.shape
    dh = d // H
    K_prev = np.asarray(K_prev, dtype=np.float64).reshape(B, -1, H, dh).transpose(0, 2, 1, 3)   # [B,H,t-1,dh]
    V_prev = np.asarray(V_prev, dtype=np.float64).reshape(B, -1, H, dh).transpose(0, 2, 1, 3)
    r = rms(x_t)
    q = _heads(r @ W["W_q"].T, H)
    k_tmp = _heads(r @ W["W_k"].T, H)
    v_tmp = _heads(r @ W["W_v"].T, H)
    keys = np.concatenate([K_prev, k_tmp[:, :, None]], axis=2)       # [B,H,t,dh]
    vals = np.concatenate([V_prev, v_tmp[:, :, None]], axis=2)
    s = np.einsum("bhe,bhie->bhi", q, keys) / np.sqrt(dh)
    w = np.exp(s - s.max(axis=-1, keepdims=True))
    a = np.einsum("bhi,bhie->bhe", w, vals) / w.sum(axis=-1)[..., None]
    u = x_t + a.reshape(B, d) @ W["W_o"].T
    z_t = u + mlp(u, W)
    rz = rms(z_t)
    return z_t, rz @ W["W_k"].T, rz @ W["W_v"].T


# --------------------------------------------------------------------------
# activation-checkpoint recompute and gradients (groundwork for training)
# --------------------------------------------------------------------------
def recompute_kv(z: np.ndarray, W: dict) -> tuple:
    """Persistent pairs of every position rebuilt from the stored layer
    outputs in one parallel step [RT paper §6.1, activation checkpointing:
    with x stored, z is kept for free as the next layer's input and the
    persistent pairs are rebuilt from it in parallel]: K = RMS(z) W_k^T,
    V = RMS(z) W_v^T, each [B, N, d]."""
    rz = rms(np.asarray(z, dtype=np.float64))
    return rz @ W["W_k"].T, rz @ W["W_v"].T


# --------------------------------------------------------------------------
# gradients of the layer (groundwork for the backward pass)
# --------------------------------------------------------------------------
def rt_layer_backward(x: np.ndarray, W: dict, H: int, dz: np.ndarray, dK: np.ndarray, dV: np.ndarray):
    """Gradients of the RT layer [RT paper §2.2] for upstream gradients dz, dK,
    dV (each [B, N, d]): returns (dx [B, N, d], dW dict of the weight
    gradients) of the scalar sum(z*dz) + sum(K*dK) + sum(V*dV).

    The forward is the naive definition of rt_layer restated in float64
    PyTorch CPU ops, and the gradients are PyTorch's reverse-mode derivatives
    of it (the pages' own backward, paper §6.4, is missing from the extracted
    text). Every persistent pair k_i, v_i receives gradient from all later
    positions' attention, so the reverse pass runs over positions in reverse.
    """
    import torch
    f64 = torch.float64
    xt = torch.tensor(np.asarray(x, dtype=np.float64), dtype=f64, requires_grad=True)
    Wt = {k: torch.tensor(np.asarray(v, dtype=np.float64), dtype=f64, requires_grad=True) for k, v in W.items()}
    B, N, d = xt.shape
    dh = d // H

    def rms_t(v):
        return v / torch.sqrt(torch.mean(v * v, dim=-1, keepdim=True) + EPS)

    def heads_t(v):
        return v.reshape(v.shape[:-1] + (H, dh))

    zs, ks, vs = [], [], []
    for t in range(N):
        r = rms_t(xt[:, t])
        q = heads_t(r @ Wt["W_q"].T)
        kt = heads_t(r @ Wt["W_k"].T)
        vt = heads_t(r @ Wt["W_v"].T)
        keys = torch.stack(ks + [kt], dim=2)            # [B, H, t+1, dh]
        vals = torch.stack(vs + [vt], dim=2)
        sc = torch.einsum("bhe,bhie->bhi", q, keys) / np.sqrt(dh)
        w = torch.softmax(sc, dim=-1)
        a = torch.einsum("bhi,bhie->bhe", w, vals).reshape(B, d)
        u = xt[:, t] + a @ Wt["W_o"].T
        hid = rms_t(u) @ Wt["W_1"].T
        zt = u + (0.5 * hid * (1.0 + torch.erf(hid / np.sqrt(2.0)))) @ Wt["W_2"].T
        rz = rms_t(zt)
        zs.append(zt)
        ks.append(heads_t(rz @ Wt["W_k"].T))
        vs.append(heads_t(rz @ Wt["W_v"].T))
    z = torch.stack(zs, dim=1)
    K = torch.stack(ks, dim=1).reshape(B, N, d)
    V = torch.stack(vs, dim=1).reshape(B, N, d)
    loss = (z * torch.tensor(dz, dtype=f64)).sum() + (K * torch.tensor(dK, dtype=f64)).sum() + \
        (V * torch.tensor(dV, dtype=f64)).sum()
    loss.backward()
    dW = {k: v.grad.numpy().copy() for k, v in Wt.items()}
    return xt.grad.numpy().copy(), dW, (z.detach().numpy(), K.detach().numpy(), V.detach().numpy())


# --------------------------------------------------------------------------
# the paper's own parameterisation (not the single-layer configuration)
# --------------------------------------------------------------------------
def rms_unit(v: np.ndarray) -> np.ndarray:
    """RMS(v) = sqrt(D) v / ||v||_2 over the last axis of width D, exactly as
    written in [RT paper §2, notation] (no eps, unit gain)."""
    return v * np.sqrt(v.shape[-1]) / np.linalg.norm(v, axis=-1, keepdims=True)


def rt_layer_pages(x: np.ndarray, W: dict, H: int, L: int = 1, kv_source: str = "output"):
    """RT layer in the paper's own parameterisation [RT paper §2 notation,
    §2.1, §2.2]; naive per-step schedule.

    Per position t and sequence b, with RMS = rms_unit and RMS_h = rms_unit
    over each head's d_h entries (the query/key normalisation, applied per
    head as the multi-head rule applies the single-head construction per head):
        r = RMS(x_t); q = RMS_h(W_q r); k~ = RMS_h(W_k r); v~ = W_v r
        per head: a_h = Attn(cached pairs + (k~, v~), q_h), scores <k, q_h>
                  (no softmax scale)
        u = x_t + W_o a / sqrt(L);  z_t = u + W_2 GELU(W_1 RMS(u)) / sqrt(L)
        persistent k_t = RMS_h(W_k RMS(s_t)), v_t = W_v RMS(s_t)
    with s_t = z_t (kv_source="output") or x_t ("input": the standard layer
    of [RT paper §2.1]). The persistent-pair equations are cut off in the
    extracted §2.2; they are read as the temporary ones applied to s_t.
    Returns (z, K, V), each [B, N, d].
    """
    if kv_source not in ("output", "input"):
        raise ValueError(kv_source)
    x = np.asarray(x, dtype=np.float64)
    B, N, d = x.shape
    dh = d // H
    inv_sqrt_L = 1.0 / np.sqrt(L)
    z = np.empty_like(x)
    Kp = np.empty((B, H, N, dh))
    Vp = np.empty((B, H, N, dh))
    for t in range(N):
        r = rms_unit(x[:, t])
        q = rms_unit(_heads(r @ W["W_q"].T, H))
        kt = rms_unit(_heads(r @ W["W_k"].T, H))
        vt = _heads(r @ W["W_v"].T, H)
        keys = np.concatenate([Kp[:, :, :t], kt[:, :, None]], axis=2)
        vals = np.concatenate([Vp[:, :, :t], vt[:, :, None]], axis=2)
        s = np.einsum("bhe,bhie->bhi", q, keys)
        w = np.exp(s - s.max(axis=-1, keepdims=True))
        a = np.einsum("bhi,bhie->bhe", w, vals) / w.sum(axis=-1)[..., None]
        u = x[:, t] + (a.reshape(B, d) @ W["W_o"].T) * inv_sqrt_L
        zt = u + (gelu(rms_unit(u) @ W["W_1"].T) @ W["W_2"].T) * inv_sqrt_L
        z[:, t] = zt
        rs = rms_unit(zt if kv_source == "output" else x[:, t])
        Kp[:, :, t] = rms_unit(_heads(rs @ W["W_k"].T, H))
        Vp[:, :, t] = _heads(rs @ W["W_v"].T, H)
    K = Kp.transpose(0, 2, 1, 3).reshape(B, N, d)
    V = Vp.transpose(0, 2, 1, 3).reshape(B, N, d)
    return z, K, V


# --------------------------------------------------------------------------
# block-wise (chunked) recurrence
# --------------------------------------------------------------------------
def rt_layer_chunked(x: np.ndarray, W: dict, H: int, C: int):
    """RT layer with the recurrence executed block-wise, in chunks of C
    positions [RT notes §8 and paper §9 (discussion and conclusion): running the recurrence over blocks of steps
    trades depth for speed; named as future work without a definition].

    Reading (ours): the positions are cut into consecutive chunks of C; a
    position's persistent pair (from its output z) becomes visible only to
    the positions of later chunks, and inside its own chunk a position
    attends to the temporary pairs (from the inputs x) of the chunk's
    positions up to and including itself. Per position t of chunk c
    (positions c*C .. c*C + C - 1):
        keys = {(k_i, v_i): i < c*C} + {(k~_s, v~_s): c*C <= s <= t}
    and everything else is the layer of rt_layer. C = 1 is rt_layer itself;
    C >= N is the standard causal Transformer layer of [RT paper §2.1] (every
    pair temporary), whose persistent pairs are then W_{k,v} RMS(z).
    Naive schedule, fp64. Returns (z, K, V), each [B, N, d].
    """
    if C < 1:
        raise ValueError("chunk length C >= 1")
    x = np.asarray(x, dtype=np.float64)
    B, N, d = x.shape
    dh = d // H
    scale = 1.0 / np.sqrt(dh)
    z = np.empty_like(x)
    Kp = np.empty((B, H, N, dh))
    Vp = np.empty((B, H, N, dh))
    r = rms(x)
    Qt = _heads(r @ W["W_q"].T, H)              # [B, N, H, dh]
    Kt = _heads(r @ W["W_k"].T, H)
    Vt = _heads(r @ W["W_v"].T, H)
    for c0 in range(0, N, C):
        c1 = min(N, c0 + C)
        for t in range(c0, c1):
            keys = np.concatenate([Kp[:, :, :c0], Kt[:, c0:t + 1].transpose(0, 2, 1, 3)], axis=2)
            vals = np.concatenate([Vp[:, :, :c0], Vt[:, c0:t + 1].transpose(0, 2, 1, 3)], axis=2)
            sc = np.einsum("bhe,bhie->bhi", Qt[:, t], keys) * scale
            sc = sc - sc.max(axis=-1, keepdims=True)
            w = np.exp(sc)
            a = np.einsum("bhi,bhie->bhe", w, vals) / w.sum(axis=-1)[..., None]
            u = x[:, t] + a.reshape(B, d) @ W["W_o"].T
            z[:, t] = u + mlp(u, W)
        rz = rms(z[:, c0:c1])                    # the chunk's persistent pairs, revealed together
        Kp[:, :, c0:c1] = _heads(rz @ W["W_k"].T, H).transpose(0, 2, 1, 3)
        Vp[:, :, c0:c1] = _heads(rz @ W["W_v"].T, H).transpose(0, 2, 1, 3)
    K = Kp.transpose(0, 2, 1, 3).reshape(B, N, d)
    V = Vp.transpose(0, 2, 1, 3).reshape(B, N, d)
    return z, K, V


# --------------------------------------------------------------------------
# blocked (lowbit) schedule, in the pages' order
# --------------------------------------------------------------------------
def lowbit_blocks(N: int):
    """The blocks of the exact blocked schedule for a length-N sequence
    [RT notes §4.2]: for t = 1..N, (t, keys, queries) with keys = (t - lb, t]
    and queries = (t, min(t + lb, N)], lb = lowbit(t). 1-based positions."""
    out = []
    for t in range(1, N + 1):
        lb = lowbit(t)
        keys = list(range(t - lb + 1, t + 1))
        queries = list(range(t + 1, min(t + lb, N) + 1))
        out.append((t, keys, queries))
    return out


def _fold(m, l, o, s, v):
    """Online-softmax merge of scores s [..., n] with values v [..., n, dh]
    into running max m, normaliser l and numerator o [RT notes §4.2: running
    maximum m, normalisation factor l, numerator vector o]."""
    m_new = np.maximum(m, s.max(axis=-1))
    alpha = np.where(np.isneginf(m), 0.0, np.exp(m - m_new))
    p = np.exp(s - m_new[..., None])
    l_new = l * alpha + p.sum(axis=-1)
    o_new = o * alpha[..., None] + np.einsum("...i,...ie->...e", p, v)
    return m_new, l_new, o_new


def rt_layer_blocked(x: np.ndarray, W: dict, H: int):
    """RT layer forward with the exact blocked schedule [RT notes §4.2;
    paper §5]. Same outputs as rt_layer up to floating-point reordering.

    1. Queries and temporary pairs are computed for all positions up front
       (they depend only on x).
    2. Accumulators start empty: m = -inf, l = 0, o = 0.
    3. For t = 1..N: merge the temporary pair of t into its accumulator,
       finalise a_t = o/l, compute u, z_t and the persistent (k_t, v_t), then
       fold keys (t - lb, t] into the accumulators of queries (t, t + lb].
    """
    x = np.asarray(x, dtype=np.float64)
    B, N, d = x.shape
    dh = d // H
    scale = 1.0 / np.sqrt(dh)
    r = rms(x)
    Q = _heads(r @ W["W_q"].T, H)         # [B, N, H, dh]
    Kt = _heads(r @ W["W_k"].T, H)
    Vt = _heads(r @ W["W_v"].T, H)
    m = np.full((B, N, H), -np.inf)
    l = np.zeros((B, N, H))
    o = np.zeros((B, N, H, dh))
    z = np.empty_like(x)
    Kp = np.empty((B, N, H, dh))
    Vp = np.empty((B, N, H, dh))
    for t, keys, queries in lowbit_blocks(N):
        j = t - 1
        s = np.einsum("bhe,bhe->bh", Q[:, j], Kt[:, j]) * scale
        m[:, j], l[:, j], o[:, j] = _fold(m[:, j], l[:, j], o[:, j],
                                          s[..., None], Vt[:, j][:, :, None])
        a = o[:, j] / l[:, j][..., None]
        u = x[:, j] + a.reshape(B, d) @ W["W_o"].T
        zt = u + mlp(u, W)
        z[:, j] = zt
        rz = rms(zt)
        Kp[:, j] = _heads(rz @ W["W_k"].T, H)
        Vp[:, j] = _heads(rz @ W["W_v"].T, H)
        ki = np.array(keys) - 1
        kb = Kp[:, ki].transpose(0, 2, 1, 3)   # [B, H, lb, dh]
        vb = Vp[:, ki].transpose(0, 2, 1, 3)
        for qj in queries:
            jj = qj - 1
            s = np.einsum("bhe,bhie->bhi", Q[:, jj], kb) * scale
            m[:, jj], l[:, jj], o[:, jj] = _fold(m[:, jj], l[:, jj], o[:, jj], s, vb)
    return z, Kp.reshape(B, N, d), Vp.reshape(B, N, d)


# --------------------------------------------------------------------------
# the fold on its own (component oracle for the block-update kernels)
# --------------------------------------------------------------------------
def block_fold(q, k, v, m, l, o, scale):
    """Fold one block: every query row of q [..., nq, dh] absorbs every key of
    k, v [..., nk, dh] into its (m, l, o) [..., nq], [..., nq], [..., nq, dh].
    Returns the updated (m, l, o). m = -inf marks an empty accumulator."""
    s = np.einsum("...qe,...ke->...qk", q, k) * scale
    vv = np.broadcast_to(v[..., None, :, :], s.shape + (v.shape[-1],))
    return _fold(m, l, o, s, vv)


# --------------------------------------------------------------------------
# stack front end and multi-layer stack
# --------------------------------------------------------------------------
def embed(ids: np.ndarray, E: np.ndarray) -> np.ndarray:
    """x = E[token] (table lookup)."""
    return E[np.asarray(ids)]


def rt_stack(ids: np.ndarray, E: np.ndarray, layers: list, H: int):
    """Token embedding, then layers applied in order, each layer's z being the
    next layer's x [RT paper §6.1: the outputs z serve as the next layer's
    input]. No final norm. Returns (z_last, [(K, V) per layer])."""
    x = embed(ids, E)
    kv = []
    for W in layers:
        x, K, V = rt_layer(x, W, H)
        kv.append((K, V))
    return x, kv
