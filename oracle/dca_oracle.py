"""fp64 CPU oracle for Dual Chunk Attention (DCA) prefill, decode and RoPE.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  It shares no code, table or constant with
the CUDA library under ``long_context_attention_dca_b200/`` and imports nothing
from it.

What it computes is the plain definition, written out without blocking,
fusion or reordering:

* RoPE (Dual-Chunk Attention: Training-Free 100k+ Context Guide, section
  "The Problem"): the score between a query rotated at position p_q and a key
  rotated at p_k depends only on p_q - p_k.  Half-split pairing: element k is
  paired with element k + D/2 and turned by the angle p * theta_k,
  theta_k = base^(-2k/D).
* DCA (Training-Free Long-Context Scaling of Large Language Models, Abstract:
  attention decomposed into chunk-based intra-chunk and inter-chunk pieces; the
  Guide's "Architectural Taxonomy": regions by chunk difference 0, 1 and >= 2).
  The sequence is cut into chunks of s tokens starting at token 0; c is the
  pretraining length and w = c - s.  A key j is rotated at j mod s.  A query
  i is rotated, per key, at
      i mod s                                  same chunk        (intra)
      s + (i mod s) for the first w queries
      of its chunk, c - 1 for the others       previous chunk    (successive)
      c - 1                                    any earlier chunk (inter)
  and all causal keys j <= i share one softmax.
* Attention: z_j = scale * <R(p_q) q_i, R(p_k) k_j>,  m = max z,
  l = sum exp(z - m),  O_i = sum exp(z_j - m) v_j / l,  LSE_i = m + ln l.
* Chunked prefill (dca_prefill_chunk): rows t0 .. t0+Lq-1 of the same
  definition with keys 0 .. t0-1 read, already rotated, from a cache.
* Variable-length batch (dca_prefill_varlen_rows): sequences packed one after
  another, each its own prefill (chunks from its first token, own keys only);
  with a cache per sequence (dca_prefill_varlen_chunk_rows) each packed
  sequence is the chunked prefill of its own cache at its own offset.
* SelfExtend (prior art; LLM Maybe LongLM: Self-Extend LLM Context Window
  Without Tuning, abstract): neighbour pairs (i - j < W) at positions (i, j),
  grouped pairs at (floor(i/G) + W - floor(W/G), floor(j/G)), one softmax.

Inputs are bf16 values upcast exactly to float64 (any float array works).
Every function is fp64 end to end; nothing is rounded to bf16.

Pins that hold this module to something other than itself live in
``tests/test_oracle_pins.py`` (worked index table, closed-form piece counts,
reduction to plain RoPE attention, Q = 0 and constant-V closed forms, RoPE
relativity, decode = prefill row, chunk = whole-sequence rows, packed batch =
padded batch and its Q = 0 closed form, hand-worked
SelfExtend distance tables and its reductions to plain RoPE attention, whole
DCA and SelfExtend rows rebuilt from the hand-worked distance tables, the
tensor rotation under every rule and offset against positions listed row by
row) and
``tests/test_oracle_mutations.py``
(plausible mistakes planted here must each fail a pin).
"""

from __future__ import annotations

import numpy as np

# Piece codes used by index_map(); the same numbering is the library's
# documented contract for its debug index map.
PIECE_MASKED = -1
PIECE_INTRA = 0
PIECE_SUCC = 1
PIECE_INTER = 2

# Position rules for rope_rotate(); numbering matches the library's contract.
POS_KEY = 0
POS_Q_INTRA = 1
POS_Q_SUCC = 2
POS_Q_INTER = 3
POS_ABSOLUTE = 4


def check_chunking(s: int, c: int) -> None:
    """Reject chunkings the definition does not cover.

    Every DCA position must stay inside the pretrained window [0, c-1]
    (Guide, "Architectural Taxonomy": the effective distance never exceeds the
    pretrained window).  The intra position i mod s reaches s - 1, so s <= c.
    """
    if not (1 <= s <= c):
        raise ValueError(f"DCA needs 1 <= s <= c, got s={s}, c={c}")


# --------------------------------------------------------------------------
# Index rules
# --------------------------------------------------------------------------

def piece(i, j, s):
    """Chunk relation of query i and key j (arrays broadcast).

    Chunks start at token 0, chunk(x) = floor(x / s).  Same chunk -> intra,
    previous chunk -> successive, earlier -> inter, j > i -> masked (causal).
    Citation: arXiv Abstract (intra/inter chunk); Guide "Architectural
    Taxonomy" (c_i == c_j, c_i == c_j + 1, c_i >= c_j + 2).
    """
    i = np.asarray(i, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    diff = i // s - j // s
    out = np.where(diff == 0, PIECE_INTRA,
                   np.where(diff == 1, PIECE_SUCC, PIECE_INTER))
    return np.where(j > i, PIECE_MASKED, out).astype(np.int8)


def key_position(j, s):
    """Keys are rotated once, at j mod s."""
    return np.asarray(j, dtype=np.int64) % s


def query_position(i, j, s, c):
    """Position at which query i is rotated when it meets key j (-1 if masked).

    intra: i mod s.  successive: s + (i mod s) when i mod s < w (the first w
    queries of the chunk), else c - 1.  inter: c - 1.  w = c - s.
    """
    check_chunking(s, c)
    i = np.asarray(i, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    w = c - s
    im = i % s
    p = piece(i, j, s)
    succ_pos = np.where(im < w, s + im, c - 1)
    out = np.where(p == PIECE_INTRA, im,
                   np.where(p == PIECE_SUCC, succ_pos, c - 1))
    return np.where(p == PIECE_MASKED, -1, out).astype(np.int64)


def index_map(L: int, s: int, c: int):
    """Dense L x L tables (qpos, kpos, piece) for tiny L.

    qpos[i, j] and kpos[i, j] are the rotation positions of the pair, piece is
    the chunk relation; masked pairs (j > i) hold -1 in all three.
    """
    check_chunking(s, c)
    i = np.arange(L, dtype=np.int64)[:, None]
    j = np.arange(L, dtype=np.int64)[None, :]
    pc = piece(i, j, s)
    qpos = query_position(i, j, s, c)
    kpos = np.where(pc == PIECE_MASKED, -1, key_position(j, s) + 0 * i)
    return qpos.astype(np.int32), kpos.astype(np.int32), pc


# --------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------

def inv_freq(D: int, base: float):
    """theta_k = base^(-2k/D), k = 0 .. D/2 - 1 (float64)."""
    k = np.arange(D // 2, dtype=np.float64)
    return np.power(np.float64(base), -2.0 * k / D)


def rotate(x, pos, base: float):
    """Half-split RoPE in fp64: pair (x_k, x_{k+D/2}) turned by pos * theta_k.

    x: [..., D]; pos: integer array broadcastable to x.shape[:-1].
    out_k       = x_k cos - x_{k+D/2} sin
    out_{k+D/2} = x_{k+D/2} cos + x_k sin
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    half = D // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq(D, base)
    cos, sin = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * cos - b * sin, b * cos + a * sin], axis=-1)


def rule_positions(n: int, rule: int, s: int, c: int, pos_offset: int = 0):
    """Rotation position of row r (absolute index i = pos_offset + r) under a rule.

    POS_KEY and POS_Q_INTRA: i mod s.  POS_Q_SUCC: s + (i mod s) if
    i mod s < w else c - 1.  POS_Q_INTER: c - 1.  POS_ABSOLUTE: i (plain RoPE).
    """
    i = pos_offset + np.arange(n, dtype=np.int64)
    if rule == POS_ABSOLUTE:
        return i
    check_chunking(s, c)
    im = i % s
    if rule in (POS_KEY, POS_Q_INTRA):
        return im
    if rule == POS_Q_SUCC:
        return np.where(im < c - s, s + im, c - 1)
    if rule == POS_Q_INTER:
        return np.full(n, c - 1, dtype=np.int64)
    raise ValueError(f"unknown position rule {rule}")


def rope_rotate(x, rule: int, s: int, c: int, base: float, pos_offset: int = 0):
    """Rotate x [B, L, H, D] at the positions a rule gives to each row."""
    x = np.asarray(x, dtype=np.float64)
    pos = rule_positions(x.shape[1], rule, s, c, pos_offset)
    return rotate(x, pos[None, :, None], base)


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def softmax_row(z, v):
    """Naive softmax-weighted sum of one row: returns (O, LSE), natural log."""
    m = np.max(z)
    e = np.exp(z - m)
    l = np.sum(e)
    return (e @ v) / l, m + np.log(l)


def kv_head(h: int, Hq: int, Hkv: int) -> int:
    """GQA: contiguous groups of G = Hq / Hkv query heads share kv head h // G."""
    return h // (Hq // Hkv)


def _scale(D, scale):
    return 1.0 / np.sqrt(D) if not scale else float(scale)


def dca_row(q, k_rot, v, i: int, s: int, c: int, base: float, scale: float):
    """One query row of DCA attention.

    q: [D] unrotated query at absolute index i.
    k_rot: [i+1, D] keys 0..i already rotated at j mod s.  v: [i+1, D].
    For every key the query is rotated at query_position(i, j) and the score
    is the scaled dot product; one softmax spans all three pieces.
    """
    j = np.arange(i + 1, dtype=np.int64)
    pq = query_position(i, j, s, c)
    z = np.empty(i + 1, dtype=np.float64)
    for p in np.unique(pq):
        sel = pq == p
        z[sel] = k_rot[sel] @ rotate(q, p, base)
    return softmax_row(scale * z, v)


def dca_prefill_rows(Q, K, V, s: int, c: int, base: float = 10000.0,
                     scale: float = 0.0, rows=None, heads=None, batches=None):
    """DCA prefill evaluated on selected (batch, head, row) outputs.

    Q: [B, L, Hq, D]; K, V: [B, L, Hkv, D] (unrotated).  q head h reads kv head
    h // (Hq / Hkv) (contiguous GQA groups).  Returns dict
    {(b, h, i): (O [D] fp64, LSE fp64)}.
    """
    check_chunking(s, c)
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    sc = _scale(D, scale)
    rows = range(L) if rows is None else rows
    heads = range(Hq) if heads is None else heads
    batches = range(B) if batches is None else batches
    rows = sorted(int(r) for r in rows)
    out = {}
    n = rows[-1] + 1
    for b in batches:
        for hk in sorted({kv_head(h, Hq, Hkv) for h in heads}):
            k_rot = rotate(np.asarray(K[b, :n, hk, :], np.float64),
                           key_position(np.arange(n), s), base)
            v = np.asarray(V[b, :n, hk, :], np.float64)
            for h in heads:
                if kv_head(h, Hq, Hkv) != hk:
                    continue
                for i in rows:
                    q = np.asarray(Q[b, i, h, :], np.float64)
                    out[(b, h, i)] = dca_row(q, k_rot[:i + 1], v[:i + 1], i,
                                             s, c, base, sc)
    return out


def dca_prefill(Q, K, V, s: int, c: int, base: float = 10000.0, scale: float = 0.0):
    """Full DCA prefill: O [B, L, Hq, D] and LSE [B, Hq, L], both fp64."""
    B, L, Hq, D = Q.shape
    res = dca_prefill_rows(Q, K, V, s, c, base, scale)
    O = np.zeros((B, L, Hq, D), np.float64)
    LSE = np.zeros((B, Hq, L), np.float64)
    for (b, h, i), (o, lse) in res.items():
        O[b, i, h] = o
        LSE[b, h, i] = lse
    return O, LSE


def dca_prefill_chunk(Qc, Kc, Vc, k_cache_rot, v_cache, t0: int, s: int, c: int,
                      base: float = 10000.0, scale: float = 0.0, rows=None, heads=None,
                      batches=None):
    """Rows t0 .. t0+Lq-1 of a DCA prefill whose first t0 keys come from a cache.

    Qc: [B, Lq, Hq, D], Kc, Vc: [B, Lq, Hkv, D] - the chunk's unrotated
    queries and keys and its values; chunk row r is token t0 + r.
    k_cache_rot, v_cache: [B, >= t0, Hkv, D] - keys 0 .. t0-1 ALREADY rotated
    at j mod s (taken as stored) and their values.
    The chunk's keys are rotated here at (t0 + r) mod s; chunk row r is query
    i = t0 + r over keys 0 .. i, exactly as in dca_prefill_rows (the rule
    depends only on the absolute indices).  Returns {(b, h, r): (O, LSE)}.
    """
    check_chunking(s, c)
    B, Lq, Hq, D = Qc.shape
    Hkv = Kc.shape[2]
    sc = _scale(D, scale)
    rows = range(Lq) if rows is None else rows
    heads = range(Hq) if heads is None else heads
    batches = range(B) if batches is None else batches
    rows = sorted(int(r) for r in rows)
    out = {}
    n = rows[-1] + 1
    for b in batches:
        for hk in sorted({kv_head(h, Hq, Hkv) for h in heads}):
            k_new = rotate(np.asarray(Kc[b, :n, hk, :], np.float64),
                           key_position(t0 + np.arange(n), s), base)
            k_rot = np.concatenate([np.asarray(k_cache_rot[b, :t0, hk, :], np.float64), k_new])
            v = np.concatenate([np.asarray(v_cache[b, :t0, hk, :], np.float64),
                                np.asarray(Vc[b, :n, hk, :], np.float64)])
            for h in heads:
                if kv_head(h, Hq, Hkv) != hk:
                    continue
                for r in rows:
                    i = t0 + r
                    q = np.asarray(Qc[b, r, h, :], np.float64)
                    out[(b, h, r)] = dca_row(q, k_rot[:i + 1], v[:i + 1], i, s, c, base, sc)
    return out


def dca_prefill_varlen_rows(Q, K, V, cu_seqlens, s: int, c: int, base: float = 10000.0,
                            scale: float = 0.0, rows=None, heads=None):
    """Packed variable-length batch of independent DCA prefills.

    Q: [T, Hq, D]; K, V: [T, Hkv, D] (unrotated).  Sequence b owns packed rows
    cu_seqlens[b] .. cu_seqlens[b+1]-1; its row at packed index t is query
    index t - cu_seqlens[b] of a prefill over that sequence alone: chunks are
    counted from the sequence's first token and only its own keys are
    attended.  rows: packed indices to evaluate (default: every row of every
    sequence).  Returns {(h, t): (O [D], LSE)} keyed by packed row.
    """
    cu = [int(x) for x in cu_seqlens]
    want = None if rows is None else {int(r) for r in rows}
    out = {}
    for b in range(len(cu) - 1):
        a, e = cu[b], cu[b + 1]
        if e <= a:
            continue
        local = [t - a for t in range(a, e) if want is None or t in want]
        if not local:
            continue
        res = dca_prefill_rows(Q[None, a:e], K[None, a:e], V[None, a:e], s, c, base, scale,
                               rows=local, heads=heads)
        for (_, h, r), val in res.items():
            out[(h, a + r)] = val
    return out


def dca_prefill_varlen_chunk_rows(Q, K, V, cu_seqlens, t0, k_cache_rot, v_cache, s: int,
                                  c: int, base: float = 10000.0, scale: float = 0.0,
                                  rows=None, heads=None):
    """Packed chunks, one per sequence, each against that sequence's cache.

    Q: [T, Hq, D]; K, V: [T, Hkv, D] (unrotated new tokens, packed as for
    dca_prefill_varlen_rows).  Sequence b's packed row cu_seqlens[b] + r is
    token t0[b] + r of sequence b, evaluated as in dca_prefill_chunk with
    keys 0 .. t0[b]-1 taken, as stored, from k_cache_rot[b] (already rotated
    at j mod s) and values from v_cache[b].  rows: packed indices (default
    all).  Returns {(h, t): (O [D], LSE)} keyed by packed row.
    """
    cu = [int(x) for x in cu_seqlens]
    want = None if rows is None else {int(r) for r in rows}
    out = {}
    for b in range(len(cu) - 1):
        a, e, tb = cu[b], cu[b + 1], int(t0[b])
        if e <= a:
            continue
        local = [t - a for t in range(a, e) if want is None or t in want]
        if not local:
            continue
        res = dca_prefill_chunk(Q[None, a:e], K[None, a:e], V[None, a:e],
                                k_cache_rot[b:b + 1], v_cache[b:b + 1], tb, s, c, base, scale,
                                rows=local, heads=heads)
        for (_, h, r), val in res.items():
            out[(h, a + r)] = val
    return out


def dca_decode(q, k_cache_rot, v_cache, t, s: int, c: int,
               base: float = 10000.0, scale: float = 0.0, batches=None,
               heads=None):
    """DCA decode for one new query per sequence.

    q: [B, Hq, D] unrotated, the query at absolute index t[b].
    k_cache_rot: [B, Tcap, Hkv, D] keys ALREADY rotated at j mod s.
    v_cache: [B, Tcap, Hkv, D].  Valid keys are 0 .. t[b] (the new token's own
    key and value are in the cache).  Returns O [B, Hq, D], LSE [B, Hq].
    """
    check_chunking(s, c)
    B, Hq, D = q.shape
    Hkv = k_cache_rot.shape[2]
    sc = _scale(D, scale)
    O = np.zeros((B, Hq, D), np.float64)
    LSE = np.zeros((B, Hq), np.float64)
    batches = range(B) if batches is None else batches
    heads = range(Hq) if heads is None else heads
    for b in batches:
        i = int(t[b])
        for hk in sorted({kv_head(h, Hq, Hkv) for h in heads}):
            k = np.asarray(k_cache_rot[b, :i + 1, hk, :], np.float64)
            v = np.asarray(v_cache[b, :i + 1, hk, :], np.float64)
            for h in heads:
                if kv_head(h, Hq, Hkv) != hk:
                    continue
                O[b, h], LSE[b, h] = dca_row(np.asarray(q[b, h], np.float64),
                                             k, v, i, s, c, base, sc)
    return O, LSE


def plain_rope_attention(Q, K, V, base: float = 10000.0, scale: float = 0.0):
    """Ordinary causal RoPE attention at absolute positions (no chunking).

    The textbook routine that DCA reduces to when the whole sequence fits in
    one chunk.  Q: [B, L, Hq, D]; K, V: [B, L, Hkv, D].
    """
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    sc = _scale(D, scale)
    pos = np.arange(L)
    qr = rotate(np.asarray(Q, np.float64), pos[None, :, None], base)
    kr = rotate(np.asarray(K, np.float64), pos[None, :, None], base)
    V = np.asarray(V, np.float64)
    O = np.zeros((B, L, Hq, D), np.float64)
    LSE = np.zeros((B, Hq, L), np.float64)
    for b in range(B):
        for h in range(Hq):
            for i in range(L):
                hk = kv_head(h, Hq, Hkv)
                z = sc * (kr[b, :i + 1, hk] @ qr[b, i, h])
                O[b, i, h], LSE[b, h, i] = softmax_row(z, V[b, :i + 1, hk])
    return O, LSE


def merge_partials(o_parts, lse_parts):
    """Combine attention over disjoint key sets given per-part (O, LSE).

    O = sum_p exp(LSE_p - LSE*) O_p with LSE* = ln sum_p exp(LSE_p); the
    identity follows from splitting the softmax denominator over the parts.
    o_parts: [P, D], lse_parts: [P].  Returns (O [D], LSE).
    """
    lse_parts = np.asarray(lse_parts, np.float64)
    m = np.max(lse_parts)
    wts = np.exp(lse_parts - m)
    tot = np.sum(wts)
    return (wts @ np.asarray(o_parts, np.float64)) / tot, m + np.log(tot)


# ---------------------------------------------------------------------------
# SelfExtend (prior art: "LLM Maybe LongLM: Self-Extend LLM Context Window
# Without Tuning", abstract): bi-level attention over the original model's
# RoPE attention.  Neighbour attention keeps the original positions for keys
# within a window of W tokens; grouped attention maps far keys and the query to
# floor-divided positions (group size G).  The abstract leaves the join of the
# two levels open; the reading taken here shifts the grouped query position by
# W - floor(W / G), so a grouped pair is never closer than W (the neighbour
# distances are 0 .. W-1) and one softmax spans both levels.
# ---------------------------------------------------------------------------

def selfextend_positions(i, j, G: int, W: int):
    """(query position, key position) of query i meeting key j (j <= i).

    Neighbour (i - j < W): (i, j).  Grouped (i - j >= W):
    (floor(i / G) + W - floor(W / G), floor(j / G)).
    """
    if G < 1 or W < 1:
        raise ValueError(f"SelfExtend needs G >= 1 and W >= 1, got G={G}, W={W}")
    i = np.asarray(i, np.int64)
    j = np.asarray(j, np.int64)
    near = (i - j) < W
    qpos = np.where(near, i, i // G + W - W // G)
    kpos = np.where(near, j, j // G)
    return qpos, kpos


def selfextend_row(q, k, v, i: int, G: int, W: int, base: float, scale: float):
    """One query row: q [D] unrotated at index i; k, v [i+1, D] unrotated keys
    0..i and values.  Each (query, key) pair is rotated at its own positions."""
    j = np.arange(i + 1, dtype=np.int64)
    qpos, kpos = selfextend_positions(i, j, G, W)
    k_rot = rotate(k, kpos, base)
    z = np.empty(i + 1, dtype=np.float64)
    for p in np.unique(qpos):
        sel = qpos == p
        z[sel] = k_rot[sel] @ rotate(q, p, base)
    return softmax_row(scale * z, v)


def selfextend_prefill_rows(Q, K, V, G: int, W: int, base: float = 10000.0,
                            scale: float = 0.0, rows=None, heads=None, batches=None):
    """SelfExtend prefill on selected (batch, head, row) outputs; Q [B, L, Hq, D],
    K, V [B, L, Hkv, D] unrotated.  Returns {(b, h, i): (O, LSE)}."""
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    sc = _scale(D, scale)
    rows = range(L) if rows is None else rows
    heads = range(Hq) if heads is None else heads
    batches = range(B) if batches is None else batches
    out = {}
    for b in batches:
        for h in heads:
            hk = kv_head(h, Hq, Hkv)
            for i in sorted(int(r) for r in rows):
                k = np.asarray(K[b, :i + 1, hk, :], np.float64)
                v = np.asarray(V[b, :i + 1, hk, :], np.float64)
                q = np.asarray(Q[b, i, h, :], np.float64)
                out[(b, h, i)] = selfextend_row(q, k, v, i, G, W, base, sc)
    return out
