"""Plain, slow fp64 reference for Dynamic Bifocal RoPE attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline leg, never by the library.

Every function follows a passage of the paper's technical summary
("Resumo Técnico: Jet-Long", gist.science, Portuguese; the French "Résumé
Technique : Jet-Long" repeats it).  Section names below are that page's.

Readings where the pages leave a step open:

* local window: key j is local for query i iff 0 <= p_i - p_j < w0, i.e. the
  window holds w0 keys including the query's own position;
* remote relative position is f(p_i) - f(p_j) with no extra offset;
* G is computed from the sequence's total length L (prefill) or from the number
  of cached tokens including the new one (decode, query at position L-1);
* positions inside a sequence are 0 .. L-1;
* Q and K arrive already rotated by standard RoPE at their absolute position;
  V is never rotated;
* RoPE is the half-split form: pair k is (x_k, x_{k+D/2}) and is rotated by the
  angle m * theta**(-2k/D);
* scores are scaled by 1/sqrt(D); LSE is the natural log of the softmax
  normaliser of the scaled scores;
* a sliding-window layer of a hybrid model (the pages: the method carries over
  to hybrid attention stacks unchanged) masks keys with p_i - p_j >= window
  (window keys including the query's own position, as for w0); the visible
  keys follow the bifocal rule and G still follows the sequence length.

Parity: pinned.  tests/test_oracle.py checks these functions against closed
forms, invariants, the worked G examples, special cases that reduce to textbook
causal RoPE attention, and pure-Python brute force on tiny inputs.
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# Position policy ("Metodologia", §1 "RoPE Bifocal Dinâmico")
# ---------------------------------------------------------------------------


def group_size(L: int, w_pretrained: int) -> int:
    """Dynamic group size G = max(1, ceil(L / w_pretrained)).

    "Agrupamento Dinâmico" bullet of §1 "RoPE Bifocal Dinâmico": G follows the
    current sequence length L and the pretrained window.  Integer ceiling, so
    it is exact for every L.  L = 0 gives G = 1.
    """
    L = int(L)
    w = int(w_pretrained)
    if w < 1:
        raise ValueError("w_pretrained must be >= 1")
    if L < 0:
        raise ValueError("L must be >= 0")
    return max(1, (L + w - 1) // w)


def position_map(x, G: int):
    """Remote position map f(x) = floor(x / G) (integer floor division).

    "Janela Remota" and "Agrupamento Dinâmico" bullets of §1: positions beyond
    the local window are aliased onto the pretrained grid by discrete floor
    division, not by interpolating frequencies.
    """
    return np.floor_divide(np.asarray(x, dtype=np.int64), int(G))


def correction_shift(p, G: int):
    """delta(p) = f(p) - p: the rotation that moves a vector stored with
    standard RoPE at position p to the grouped position f(p).

    §2 "Rotação de Correção On-the-Fly": RoPE rotations compose additively, so
    R(delta(p)) R(p) = R(f(p)).
    """
    p = np.asarray(p, dtype=np.int64)
    return position_map(p, G) - p


# ---------------------------------------------------------------------------
# RoPE (half-split pairs)
# ---------------------------------------------------------------------------


def rope_inv_freq(D: int, theta: float) -> np.ndarray:
    """inv_freq_k = theta ** (-2k / D), k = 0 .. D/2 - 1, in fp64."""
    k = np.arange(D // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * k / D)


def rope_rotate(x: np.ndarray, m, theta: float) -> np.ndarray:
    """R(m) x for the half-split RoPE: pair k = (x_k, x_{k+D/2}) is rotated by
    angle m * inv_freq_k, i.e. (a, b) -> (a cos - b sin, a sin + b cos).

    ``x`` has shape [..., D]; ``m`` (integer positions or shifts) broadcasts
    against x.shape[:-1].  Angles are formed in fp64 from exact integers.
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    h = D // 2
    ang = np.asarray(m, dtype=np.float64)[..., None] * rope_inv_freq(D, theta)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


# ---------------------------------------------------------------------------
# Shared softmax helper (plain, full-row)
# ---------------------------------------------------------------------------


def _softmax_rows(S: np.ndarray, V: np.ndarray):
    """Row softmax of scores S [R, N] (-inf = excluded) applied to V [N, D].

    Returns (O [R, D], lse [R]).  A row with no admitted key returns O = 0 and
    lse = -inf.
    """
    m = S.max(axis=1)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    P = np.exp(S - m_safe[:, None])
    l = P.sum(axis=1)
    O = np.zeros((S.shape[0], V.shape[1]), dtype=np.float64)
    O[finite] = (P[finite] @ V) / l[finite, None]
    lse = np.full(S.shape[0], -np.inf)
    lse[finite] = m_safe[finite] + np.log(l[finite])
    return O, lse


def _as64(t) -> np.ndarray:
    if hasattr(t, "detach"):
        t = t.detach().to("cpu")
        import torch

        t = t.to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def _seq_bounds(cu_seqlens):
    cu = np.asarray(cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens,
                    dtype=np.int64)
    return [(int(cu[s]), int(cu[s + 1])) for s in range(len(cu) - 1)]


# ---------------------------------------------------------------------------
# Route A: the direct definition (primary oracle)
# ---------------------------------------------------------------------------


def _attend_rows_direct(q_rows, pos_i, K, K_g, V, G, w0, theta, plain, window=0):
    """Scores of query rows against keys 0..L-1 of one sequence and one head.

    q_rows [R, D] standard-RoPE queries at positions pos_i; K [L, D]
    standard-RoPE keys at positions 0..L-1; K_g [L, D] the same keys rotated
    by R(delta(p_j)) (None when ``plain``); V [L, D].

    For each pair with 0 <= d = p_i - p_j:
      d <  w0  ->  s = <Q~_i, K~_j> / sqrt(D)                       (local, base RoPE)
      d >= w0  ->  s = <R(delta_i) Q~_i, R(delta_j) K~_j> / sqrt(D)  (remote, grouped)
    "Janela Local" / "Janela Remota" bullets of §1 and the correction rotation
    of §2.  ``plain`` scores every pair with the base RoPE (G irrelevant).
    ``window`` > 0 is a sliding-window layer of a hybrid model ("Principais
    Contribuições" 4 and the hybrid-architecture results): only keys with
    d < window are visible, and the visible ones follow the rule above.
    """
    L, D = K.shape
    scale = 1.0 / math.sqrt(D)
    pos_j = np.arange(L, dtype=np.int64)
    dist = pos_i[:, None] - pos_j[None, :]
    S_std = (q_rows @ K.T) * scale
    if plain:
        S = S_std
    else:
        q_g = rope_rotate(q_rows, correction_shift(pos_i, G), theta)
        S_grp = (q_g @ K_g.T) * scale
        S = np.where(dist < w0, S_std, S_grp)
    visible = dist >= 0
    if window > 0:
        visible &= dist < window
    S = np.where(visible, S, -np.inf)
    return _softmax_rows(S, V)


def _take64(t, idx, h):
    """fp64 copy of t[idx, h] for a torch tensor or a numpy array."""
    if hasattr(t, "detach"):
        import torch

        return _as64(t[torch.as_tensor(np.asarray(idx, dtype=np.int64)), h])
    return np.asarray(t[np.asarray(idx), h], dtype=np.float64)


def bifocal_attention(q, k, v, cu_seqlens, w_pretrained, w0, theta, rows=None, plain=False,
                      row_batch=64, window=0):
    """Dynamic Bifocal RoPE causal GQA prefill attention, route A (direct).

    q [T, Hq, D], k/v [T, Hkv, D] (any float type, torch or numpy; computed in
    fp64), packed by ``cu_seqlens`` [B+1]; query head h reads kv head
    h // (Hq / Hkv).

    ``rows``: optional sorted global token indices to evaluate (default: all).
    ``window`` > 0: sliding-window layer (keys with p_i - p_j >= window are
    masked; G still follows the sequence length).
    Returns (out [len(rows), Hq, D], lse [Hq, len(rows)]) in fp64.
    """
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    group = Hq // Hkv
    rows = np.arange(T, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((len(rows), Hq, D))
    lse = np.full((Hq, len(rows)), -np.inf)
    for a, b in _seq_bounds(cu_seqlens):
        L = b - a
        sel = np.nonzero((rows >= a) & (rows < b))[0]
        if L == 0 or len(sel) == 0:
            continue
        G = group_size(L, w_pretrained)
        pos_j = np.arange(L, dtype=np.int64)
        for kv in range(Hkv):
            K = _take64(k, np.arange(a, b), kv)
            V = _take64(v, np.arange(a, b), kv)
            K_g = None if plain else rope_rotate(K, correction_shift(pos_j, G), theta)
            for h in range(kv * group, (kv + 1) * group):
                for c in range(0, len(sel), row_batch):
                    idx = sel[c:c + row_batch]
                    pos_i = rows[idx] - a
                    o, l_ = _attend_rows_direct(_take64(q, rows[idx], h), pos_i, K, K_g, V, G, w0,
                                                theta, plain, window)
                    out[idx, h] = o
                    lse[h, idx] = l_
    return out, lse


def bifocal_attention_kv(q, k, v, cu_seqlens_q, cu_seqlens_k, w_pretrained, w0, theta, rows=None,
                         plain=False, row_batch=64, window=0):
    """Prefill of new tokens against keys that include an existing cache.

    Sequence s has keys/values k, v[cu_k[s] : cu_k[s+1]] at positions
    0 .. Lk-1 (standard RoPE, never rewritten) and Lq <= Lk queries
    q[cu_q[s] : cu_q[s+1]] at the last positions Lk-Lq .. Lk-1.  G follows
    the current length Lk (§1 "Agrupamento Dinâmico"; §2 "Rotação de Correção
    On-the-Fly": generation streams across length boundaries without
    rewriting the cache).  With Lq = Lk this is ``bifocal_attention``; with
    Lq = 1 it is one ``bifocal_decode`` step.  ``window`` as in
    ``bifocal_attention``.

    Returns (out [len(rows), Hq, D], lse [Hq, len(rows)]) for the query rows
    ``rows`` (global indices into q; default all).
    """
    Tq, Hq, D = q.shape
    Hkv = k.shape[1]
    group = Hq // Hkv
    rows = np.arange(Tq, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((len(rows), Hq, D))
    lse = np.full((Hq, len(rows)), -np.inf)
    for (aq, bq), (ak, bk) in zip(_seq_bounds(cu_seqlens_q), _seq_bounds(cu_seqlens_k)):
        Lq, Lk = bq - aq, bk - ak
        if Lq > Lk:
            raise ValueError("a sequence has more queries than keys")
        sel = np.nonzero((rows >= aq) & (rows < bq))[0]
        if Lq == 0 or len(sel) == 0:
            continue
        G = group_size(Lk, w_pretrained)
        offset = Lk - Lq
        pos_j = np.arange(Lk, dtype=np.int64)
        for kv in range(Hkv):
            K = _take64(k, np.arange(ak, bk), kv)
            V = _take64(v, np.arange(ak, bk), kv)
            K_g = None if plain else rope_rotate(K, correction_shift(pos_j, G), theta)
            for h in range(kv * group, (kv + 1) * group):
                for c in range(0, len(sel), row_batch):
                    idx = sel[c:c + row_batch]
                    pos_i = offset + (rows[idx] - aq)
                    o, l_ = _attend_rows_direct(_take64(q, rows[idx], h), pos_i, K, K_g, V, G, w0,
                                                theta, plain, window)
                    out[idx, h] = o
                    lse[h, idx] = l_
    return out, lse


def bifocal_decode(q, k_cache, v_cache, seqlens, w_pretrained, w0, theta, plain=False, window=0):
    """One decode step, route A: the new query of sequence b sits at position
    L_b - 1 and attends to cache rows 0 .. L_b - 1 with G = G(L_b).

    §2 "Rotação de Correção On-the-Fly": the cache keeps standard-RoPE keys and
    G is recomputed from the current length at every step.

    q [B, Hq, D]; k_cache, v_cache [B, Lcap, Hkv, D]; seqlens [B].
    ``window`` as in ``bifocal_attention``.
    Returns (out [B, Hq, D], lse [B, Hq]).
    """
    q = _as64(q)
    B, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    group = Hq // Hkv
    seqlens = [int(x) for x in (seqlens.tolist() if hasattr(seqlens, "tolist") else seqlens)]
    out = np.zeros((B, Hq, D))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        L = seqlens[b]
        if L == 0:
            continue
        G = group_size(L, w_pretrained)
        pos_i = np.array([L - 1], dtype=np.int64)
        pos_j = np.arange(L, dtype=np.int64)
        for kv in range(Hkv):
            K = _as64(k_cache[b, :L, kv])
            V = _as64(v_cache[b, :L, kv])
            K_g = None if plain else rope_rotate(K, correction_shift(pos_j, G), theta)
            for h in range(kv * group, (kv + 1) * group):
                o, l_ = _attend_rows_direct(q[b, h][None, :], pos_i, K, K_g, V, G, w0, theta, plain,
                                            window)
                out[b, h] = o[0]
                lse[b, h] = l_[0]
    return out, lse


# ---------------------------------------------------------------------------
# Route B: three softmax passes merged by inclusion-exclusion
# ---------------------------------------------------------------------------


def _masked_pass(q_row, K, V, keep):
    """One standard softmax-attention pass of a single query over the keys
    where ``keep`` is True.  Returns (o [D], lse) or (None, -inf) if empty."""
    if not np.any(keep):
        return None, -np.inf
    D = K.shape[1]
    s = (K[keep] @ q_row) / math.sqrt(D)
    m = s.max()
    e = np.exp(s - m)
    return (e @ V[keep]) / e.sum(), m + math.log(e.sum())


def bifocal_attention_ie_merge(q, k, v, cu_seqlens, w_pretrained, w0, theta, rows=None):
    """Route B: §2 "Mesclagem de Atenção Inclusão–Exclusão".

    Three ordinary attention passes per query row,
      (1) local window, base queries/keys     -> (o1, lse1)
      (2) full causal, grouped queries/keys   -> (o2, lse2)
      (3) local window, grouped queries/keys  -> (o3, lse3)
    merged with LSE weights so the window is not counted twice:
      O = (e^lse1 o1 + e^lse2 o2 - e^lse3 o3) / (e^lse1 + e^lse2 - e^lse3),
    stabilised by subtracting max(lse1, lse2) inside the exponentials.  When
    the row has no remote key, sets (2) and (3) are the same keys and the
    remote term is taken as exactly zero.
    Returns (out, lse) shaped like ``bifocal_attention``.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    T, Hq, D = q.shape
    group = Hq // k.shape[1]
    rows = np.arange(T, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((len(rows), Hq, D))
    lse = np.full((Hq, len(rows)), -np.inf)
    for a, b in _seq_bounds(cu_seqlens):
        L = b - a
        if L == 0:
            continue
        G = group_size(L, w_pretrained)
        pos = np.arange(L, dtype=np.int64)
        for h in range(Hq):
            kv = h // group
            K, V = k[a:b, kv], v[a:b, kv]
            Kg = rope_rotate(K, correction_shift(pos, G), theta)
            for r in np.nonzero((rows >= a) & (rows < b))[0]:
                i = int(rows[r] - a)
                qi = q[rows[r], h]
                qg = rope_rotate(qi, correction_shift(i, G), theta)
                d = i - pos
                window = (d >= 0) & (d < w0)
                causal = d >= 0
                o1, l1 = _masked_pass(qi, K, V, window)
                o2, l2 = _masked_pass(qg, Kg, V, causal)
                o3, l3 = _masked_pass(qg, Kg, V, window)
                has_remote = bool(np.any(causal & ~window))
                mx = max(l1, l2)
                a1 = math.exp(l1 - mx) if o1 is not None else 0.0
                num = a1 * (o1 if o1 is not None else 0.0)
                den = a1
                if has_remote:
                    a2 = math.exp(l2 - mx)
                    a3 = math.exp(l3 - mx) if o3 is not None else 0.0
                    num = num + a2 * o2 - (a3 * o3 if o3 is not None else 0.0)
                    den = den + a2 - a3
                out[r, h] = num / den
                lse[h, r] = mx + math.log(den)
    return out, lse


# ---------------------------------------------------------------------------
# Route C: the method stated on raw (unrotated) vectors
# ---------------------------------------------------------------------------


def bifocal_attention_from_raw(q_raw, k_raw, v, L, w_pretrained, w0, theta):
    """Route C, single sequence, every head: the bifocal definition applied to
    raw (not yet rotated) projections, without any correction rotation.

    Local pairs (0 <= i - j < w0) score <R(i) q_i, R(j) k_j>; remote pairs score
    <R(f(i)) q_i, R(f(j)) k_j> ("Janela Local" / "Janela Remota" of §1).
    q_raw [L, Hq, D], k_raw/v [L, Hkv, D].  Returns (out [L, Hq, D], lse [Hq, L]).
    """
    q_raw, k_raw, v = _as64(q_raw), _as64(k_raw), _as64(v)
    _, Hq, D = q_raw.shape
    group = Hq // k_raw.shape[1]
    G = group_size(L, w_pretrained)
    pos = np.arange(L, dtype=np.int64)
    f = position_map(pos, G)
    scale = 1.0 / math.sqrt(D)
    dist = pos[:, None] - pos[None, :]
    out = np.zeros((L, Hq, D))
    lse = np.zeros((Hq, L))
    for h in range(Hq):
        kv = h // group
        q_loc = rope_rotate(q_raw[:, h], pos, theta)
        k_loc = rope_rotate(k_raw[:, kv], pos, theta)
        q_far = rope_rotate(q_raw[:, h], f, theta)
        k_far = rope_rotate(k_raw[:, kv], f, theta)
        S = np.where(dist < w0, (q_loc @ k_loc.T) * scale, (q_far @ k_far.T) * scale)
        S = np.where(dist >= 0, S, -np.inf)
        out[:, h], lse[h] = _softmax_rows(S, v[:, kv])
    return out, lse


# ---------------------------------------------------------------------------
# Textbook causal RoPE attention (for the reduction pins)
# ---------------------------------------------------------------------------


def causal_rope_attention(q, k, v, window=0):
    """Ordinary causal softmax attention of one sequence over already-rotated
    q [L, Hq, D], k/v [L, Hkv, D], scale 1/sqrt(D).  ``window`` > 0 is the
    textbook sliding window: query i sees keys i - window + 1 .. i.
    Returns (out, lse)."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    L, Hq, D = q.shape
    group = Hq // k.shape[1]
    out = np.zeros((L, Hq, D))
    lse = np.zeros((Hq, L))
    for h in range(Hq):
        kv = h // group
        S = (q[:, h] @ k[:, kv].T) / math.sqrt(D)
        S[np.triu_indices(L, 1)] = -np.inf
        if window > 0:
            S[np.tril_indices(L, -window)] = -np.inf
        out[:, h], lse[h] = _softmax_rows(S, v[:, kv])
    return out, lse


# ---------------------------------------------------------------------------
# Brute force with pure-Python loops (tiny inputs only)
# ---------------------------------------------------------------------------


def brute_force_tiny(q_raw, k_raw, v, w_pretrained, w0, theta, window=0):
    """Pure-Python double loop over (i, j) for one sequence and one head pair:
    q_raw [L][D], k_raw [L][D], v [L][D] as nested lists of floats.

    Each score rotates the raw vectors explicitly with math.cos / math.sin at
    the position the definition names (absolute inside the window, f(.)
    outside), builds the full L x L score table and normalises each row.
    ``window`` > 0 keeps only the keys j > i - window.
    Returns (out [L][D], lse [L]).
    """
    L = len(q_raw)
    D = len(q_raw[0])
    h = D // 2
    G = max(1, -(-L // w_pretrained))

    def rot(x, m):
        y = [0.0] * D
        for kk in range(h):
            ang = m * theta ** (-2.0 * kk / D)
            c, s = math.cos(ang), math.sin(ang)
            y[kk] = x[kk] * c - x[kk + h] * s
            y[kk + h] = x[kk] * s + x[kk + h] * c
        return y

    out, lse = [], []
    for i in range(L):
        j_first = max(0, i - window + 1) if window > 0 else 0
        scores = []
        for j in range(j_first, i + 1):
            if i - j < w0:
                a, b = rot(q_raw[i], i), rot(k_raw[j], j)
            else:
                a, b = rot(q_raw[i], i // G), rot(k_raw[j], j // G)
            scores.append(sum(x * y for x, y in zip(a, b)) / math.sqrt(D))
        m = max(scores)
        e = [math.exp(s - m) for s in scores]
        z = sum(e)
        out.append([sum(e[j - j_first] * v[j][c] for j in range(j_first, i + 1)) / z for c in range(D)])
        lse.append(m + math.log(z))
    return out, lse
