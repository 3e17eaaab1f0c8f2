"""CPU float64 oracle for single-token incremental-decode attention over a KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
call it.  It shares no code with the CUDA path: it reads plain NumPy arrays and
writes plain NumPy arrays, and it is written straight from the definitions on
the pages, without blocking, splitting or reordering.

Sources (web pages on Multi-Query Attention; cited by title and section):

* [velog review] "[Paper review] Fast Transformer Decoding: One Write-Head is All
  You Need", §2.1 (DotProductAttention), §2.3 (Multi-head Attention (Batched):
  logits = einsum("bhnk,bhmk->bhnm"), softmax(logits + mask)), §2.4
  (MultiheadSelfAttentionIncremental) and §3 (MultiquerySelfAttentionIncremental;
  MQA drops the h axis of K/V).  These give the computation as
  einsums: logits = einsum("bhk,bmk->bhm", q, K); weights = softmax(logits);
  o = einsum("bhm,bmv->bhv", weights, V); the per-head form has K/V [b,h,m,k].
* [kuangjux notes] "Fast Transformer Decoding: One Write-Head is All You Need"
  (study notes), §1 (the scaled, masked softmax O = softmax(QKᵀ/√d_h + M)V),
  §4 (MQA drops only the head axis of K/V; worked example with two keys), §6.1
  (the decoder's local attention: the current position and the 31 before it)
  and §6.4 (local attention and MQA combined).
* [oscine blog] "GQA、MQA、MLA：当「多头」变成推理账单上最贵的一项", section
  "第三站: GQA" (H query heads split into G groups, one K/V head per group;
  GQA-1 is MQA, GQA-H is MHA).

Readings where the pages leave a step open (each listed again in the design
notes of the repository):

* Scale: the pseudocode has none, the notes divide by √d_h.  Every function here
  takes ``scale`` and multiplies the logits by it; callers pick the value.
* Mask: position t of sequence b is valid iff t < lens[b] (the query is the
  newest token, so causality is implied).  Rows at t >= lens[b] are never read,
  so their contents (NaN in the tests) cannot leak into the result.
* Grouping: query head i reads K/V head j(i) = i // (h // g), i.e. contiguous
  groups; h must be a multiple of g.
* lens[b] == 0: the output row is 0 and lse is -inf (the pages do not define it).
* Prefill: the review's batched form takes a general additive mask [b,h,n,m];
  the notes' §1 and §10 describe prefill as the whole prompt at once under a
  causal mask.  Reading: with ``causal`` query position t of a sequence sees
  the keys 0..t of the same sequence (mask 0, else -inf); without it, all keys
  of the sequence.  Sequences are packed: rows cu_seqlens[s] .. cu_seqlens[s+1]-1.
* Beam search: the notes' §6.2 and §6.4 time a beam-4 decoder but give no
  formula.  Reading: each of W beams of a sequence attends over the
  sequence's shared prefix rows followed by its own suffix rows (the tokens
  that beam generated), i.e. plain decode attention over that concatenation.
* Local window: the notes name a window of the current position plus the 31
  before it, with no formula.  With ``window`` = w > 0, position t of sequence
  b is attended iff lens[b] - w <= t < lens[b] (the newest w rows; w = 32 is the
  notes' window); w = 0 means no window.

Parity pins for every function live in ``tests/test_oracle.py``; none is
unpinned.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "dot_product_attention",
    "oracle_decode",
    "oracle_kv_append",
    "oracle_decode_step",
    "oracle_prefill",
    "oracle_decode_beam",
]


def dot_product_attention(q, K, V, scale=1.0):
    """Attention for ONE query against one K/V head, with plain Python loops.

    Follows [velog review] §2.1 DotProductAttention: q [k], K [m, k], V [m, v];
    logits_t = Σ_r q_r K_{t,r}; weights = softmax(logits); y = Σ_t w_t V_t.
    The scale multiplies the logits (the √d_h division of [kuangjux notes] §1).
    Small inputs only: this is the brute-force reference the batched oracle is
    checked against.
    """
    q = [float(x) for x in np.asarray(q, dtype=np.float64).ravel()]
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    m = K.shape[0]
    logits = []
    for t in range(m):
        acc = 0.0
        for r in range(len(q)):
            acc += q[r] * float(K[t, r])
        logits.append(acc * scale)
    top = max(logits)
    exps = [math.exp(s - top) for s in logits]
    total = math.fsum(exps)
    weights = [e / total for e in exps]
    y = []
    for c in range(V.shape[1]):
        y.append(math.fsum(weights[t] * float(V[t, c]) for t in range(m)))
    return np.array(y, dtype=np.float64), np.array(weights, dtype=np.float64)


def oracle_decode(q, k_cache, v_cache, lens, g, scale, return_weights=False, window=0):
    """One decode step of MQA / GQA / MHA attention, in float64.

    Shapes: q [b, h, d_k]; k_cache [b, m_max, g, d_k]; v_cache [b, m_max, g, d_v];
    lens int [b].  Returns o [b, h, d_v] float64 and lse [b, h] float64 (natural
    log of Σ_t exp(logit_t)), plus the weights as a list of [h, lens[b]] arrays
    when ``return_weights``.

    For each sequence b and K/V group j, the h//g query heads of that group form
    a matrix Q_j [h//g, d_k]; with L = lens[b] and K_j = k_cache[b, :L, j, :]:
        S = scale · Q_j K_jᵀ                       ([velog review] §3 logits einsum)
        w = softmax over the L valid positions      (§3 softmax; [kuangjux notes] §1)
        o = w V_j                                   (§3 weighted-V einsum)
    g = 1 is MQA, g = h is MHA, 1 < g < h is GQA ([oscine blog] "第三站: GQA").
    With ``window`` = w > 0 only positions L-w <= t < L take part (local
    attention, [kuangjux notes] §6.1 and §6.4); the weights of the others are 0.
    Inputs are used at whatever precision they hold (the tests hand in values
    already rounded to the kernel's input type) and widened to float64 here.
    """
    q = np.asarray(q)
    k_cache = np.asarray(k_cache)
    v_cache = np.asarray(v_cache)
    lens = np.asarray(lens).astype(np.int64)
    b, h, d_k = q.shape
    _, m_max, g_cache, _ = k_cache.shape
    d_v = v_cache.shape[3]
    if g_cache != g or h % g != 0:
        raise ValueError("k_cache must have g heads and h must be a multiple of g")
    hq = h // g
    window = int(window)
    if window < 0:
        raise ValueError("window must be >= 0")
    o = np.zeros((b, h, d_v), dtype=np.float64)
    lse = np.full((b, h), -np.inf, dtype=np.float64)
    weights = [] if return_weights else None
    for bi in range(b):
        L = int(lens[bi])
        if L > m_max:
            raise ValueError("lens[b] exceeds m_max")
        w_b = np.zeros((h, max(L, 0)), dtype=np.float64)
        if L <= 0:
            if return_weights:
                weights.append(w_b)
            continue
        L0 = max(0, L - window) if window > 0 else 0                        # first attended row
        for j in range(g):
            Qj = q[bi, j * hq:(j + 1) * hq, :].astype(np.float64)          # [hq, d_k]
            Kj = k_cache[bi, L0:L, j, :].astype(np.float64)                 # [L-L0, d_k]
            Vj = v_cache[bi, L0:L, j, :].astype(np.float64)                 # [L-L0, d_v]
            S = scale * (Qj @ Kj.T)                                         # [hq, L]
            mu = S.max(axis=1, keepdims=True)
            E = np.exp(S - mu)
            denom = E.sum(axis=1, keepdims=True)
            W = E / denom
            o[bi, j * hq:(j + 1) * hq, :] = W @ Vj
            lse[bi, j * hq:(j + 1) * hq] = (mu + np.log(denom))[:, 0]
            w_b[j * hq:(j + 1) * hq, L0:] = W
        if return_weights:
            weights.append(w_b)
    if return_weights:
        return o, lse, weights
    return o, lse


def oracle_kv_append(k_cache, v_cache, k_new, v_new, pos):
    """The step's K/V written into the cache: the "one write-head".

    [velog review] §3 builds new_K = concat([prev_K, k_new], axis=1) (and the same
    for V).  With a fixed-size cache [b, m_max, g, d] the concat becomes a write
    of k_new[b] at row pos[b] of sequence b; every other element is unchanged.
    Returns new arrays (the inputs are not modified).  Works on any dtype,
    including the raw bf16 bit patterns (uint16), so the comparison is bitwise.
    """
    k_out = np.array(k_cache, copy=True)
    v_out = np.array(v_cache, copy=True)
    pos = np.asarray(pos).astype(np.int64)
    for bi in range(k_out.shape[0]):
        p = int(pos[bi])
        if 0 <= p < k_out.shape[1]:
            k_out[bi, p] = k_new[bi]
            v_out[bi, p] = v_new[bi]
    return k_out, v_out


def oracle_decode_step(q, k_cache, v_cache, k_new, v_new, lens_before, g, scale, window=0):
    """One whole incremental step in the order of [velog review] §3: append the
    new K/V at row lens_before[b], then attend over lens_before[b] + 1 rows (the
    newest ``window`` of them when window > 0)."""
    k2, v2 = oracle_kv_append(k_cache, v_cache, k_new, v_new, lens_before)
    lens_after = np.asarray(lens_before).astype(np.int64) + 1
    o, lse = oracle_decode(q, k2, v2, lens_after, g, scale, window=window)
    return o, lse, k2, v2


def oracle_prefill(q, k, v, cu_seqlens, g, scale, causal=True):
    """Attention of every position of every sequence over the same sequence's
    keys, in float64: the batched form of [velog review] §2.3 with the K/V head
    axis removed as in §3 (h // g query heads per K/V head, [oscine blog]
    "第三站: GQA"), under a causal mask for prefill ([kuangjux notes] §1, §10).

    Shapes (packed sequences): q [T, h, d_k]; k [T, g, d_k]; v [T, g, d_v];
    cu_seqlens int [b+1], sequence s holding rows cu_seqlens[s] .. cu_seqlens[s+1]-1.
    Returns o [T, h, d_v] and lse [T, h] (natural log of the softmax denominator).

    For each sequence and K/V group j, with Q_j [n, h//g, d_k] and K_j, V_j [n, d]:
        S[t, i, u] = scale · Q_j[t, i] · K_j[u]          (§2.3 logits einsum)
        S[t, i, u] = -inf for u > t when causal           (the mask)
        W = softmax over u;  O[t, i] = Σ_u W[t, i, u] V_j[u]
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    cu = np.asarray(cu_seqlens).astype(np.int64)
    T, h, d_k = q.shape
    d_v = v.shape[2]
    if k.shape[:2] != (T, g) or v.shape[:2] != (T, g) or h % g != 0:
        raise ValueError("k/v must be [T, g, d] and h a multiple of g")
    hq = h // g
    o = np.zeros((T, h, d_v), dtype=np.float64)
    lse = np.full((T, h), -np.inf, dtype=np.float64)
    for si in range(len(cu) - 1):
        a, e = int(cu[si]), int(cu[si + 1])
        n = e - a
        if n <= 0:
            continue
        allowed = np.tril(np.ones((n, n), dtype=bool)) if causal else np.ones((n, n), dtype=bool)   # [query, key]
        for j in range(g):
            Qj = q[a:e, j * hq:(j + 1) * hq, :].astype(np.float64)            # [n, hq, d_k]
            Kj = k[a:e, j, :].astype(np.float64)                               # [n, d_k]
            Vj = v[a:e, j, :].astype(np.float64)                               # [n, d_v]
            S = scale * np.einsum("tik,uk->tiu", Qj, Kj)                       # [n, hq, n]
            S = np.where(allowed[:, None, :], S, -np.inf)
            mu = S.max(axis=2, keepdims=True)
            E = np.exp(S - mu)
            denom = E.sum(axis=2, keepdims=True)
            o[a:e, j * hq:(j + 1) * hq, :] = np.einsum("tiu,uv->tiv", E / denom, Vj)
            lse[a:e, j * hq:(j + 1) * hq] = (mu + np.log(denom))[:, :, 0]
    return o, lse


def oracle_decode_beam(q, prefix_k, prefix_v, prefix_lens, suffix_k, suffix_v, suffix_lens, g, scale):
    """One decode step of W beams per sequence that share a prefix, in float64
    ([kuangjux notes] §6.2/§6.4 beam-4 decoding; reading in the header).

    Shapes: q [b, W, h, d_k]; prefix_k/v [b, m_p, g, d]; prefix_lens [b];
    suffix_k/v [b*W, m_s, g, d] (beam w of sequence s at row s*W + w);
    suffix_lens [b*W].  Beam (s, w) attends over prefix rows 0..prefix_lens[s]-1
    of sequence s followed by suffix rows 0..suffix_lens[s*W+w]-1 of its own
    cache: oracle_decode on that concatenated cache.  Returns o [b, W, h, d_v]
    and lse [b, W, h].
    """
    q = np.asarray(q)
    b, W, h, d_k = q.shape
    pk, pv = np.asarray(prefix_k), np.asarray(prefix_v)
    sk, sv = np.asarray(suffix_k), np.asarray(suffix_v)
    lp = np.asarray(prefix_lens).astype(np.int64)
    ls = np.asarray(suffix_lens).astype(np.int64)
    d_v = pv.shape[3]
    o = np.zeros((b, W, h, d_v), dtype=np.float64)
    lse = np.full((b, W, h), -np.inf, dtype=np.float64)
    for si in range(b):
        for w in range(W):
            r = si * W + w
            K = np.concatenate([pk[si, :lp[si]], sk[r, :ls[r]]], axis=0)[None]     # [1, L, g, d]
            V = np.concatenate([pv[si, :lp[si]], sv[r, :ls[r]]], axis=0)[None]
            L = K.shape[1]
            if L == 0:
                continue
            ob, lb = oracle_decode(q[si, w][None], K, V, [L], g, scale)
            o[si, w], lse[si, w] = ob[0], lb[0]
    return o, lse
