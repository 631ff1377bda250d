"""Pins that hold the fp64 oracle to facts fixed outside itself.

Each pin is a module-level function ``pin_*`` so that the mutation tests can
re-run them against a deliberately broken oracle; the ``test_*`` wrappers run
them against the oracle as committed.  Sources of each fact:

* hand-worked index tables under ``tests/golden/`` (the DCA rule applied by
  hand; no code wrote them);
* the bound "effective distance never exceeds the pretrained window" and
  "intra-chunk distance is the exact, unscaled i - j" (Dual-Chunk Attention:
  Training-Free 100k+ Context Guide, "Architectural Taxonomy" and
  "Intra-Chunk Attention");
* closed-form piece counts (pure counting over chunk sizes);
* reduction to ordinary causal RoPE attention when the whole sequence fits
  in one chunk, checked against torch's scaled_dot_product_attention with the
  rotation done by complex multiplication;
* closed forms for Q = 0 and constant V, RoPE relativity (Guide, "The
  Problem": the score depends only on the position difference), literal
  rotation values, and the split-softmax identity;
* a chunk at t0 over a cache of the earlier keys equals the whole-sequence
  rows (the rule depends only on absolute indices);
* SelfExtend (LLM Maybe LongLM, abstract): hand-worked neighbour / grouped
  distance tables under ``tests/golden/``, its reduction to plain RoPE
  attention for G = 1 or W >= L (torch SDPA), and distance bounds;
* whole attention rows (DCA and SelfExtend) rebuilt from the hand-worked
  distance tables alone, through RoPE relativity;
* the rotation of a whole tensor under each position rule and offset,
  against positions listed row by row and a few literal values.
"""

import math
import pathlib

import numpy as np
import pytest
import torch

from oracle import dca_oracle as orc

GOLDEN = pathlib.Path(__file__).parent / "golden"
TABLES = [("dca_index_s4_c6_L12.txt", 4, 6), ("dca_index_s3_c5_L9.txt", 3, 5),
          ("dca_index_s3_c3_L7.txt", 3, 3), ("dca_index_s2_c5_L7.txt", 2, 5)]


SE_TABLES = [("selfextend_G2_W3_L10.txt", 2, 3), ("selfextend_G3_W4_L12.txt", 3, 4)]


def parse_table(name, letters=None):
    letters = letters or {"A": 0, "S": 1, "I": 2}
    lines = [ln for ln in (GOLDEN / name).read_text().splitlines()
             if ln.strip() and not ln.startswith("#")]
    rows = lines[1:]
    L = len(rows)
    pc = np.full((L, L), -1, np.int8)
    dist = np.full((L, L), -1, np.int64)
    for r, line in enumerate(rows):
        toks = line.split()
        assert int(toks[0]) == r
        assert len(toks) == L + 1
        for j, tok in enumerate(toks[1:]):
            if tok == ".":
                continue
            pc[r, j] = letters[tok[0]]
            dist[r, j] = int(tok[1:])
    return pc, dist


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _complex_rotate(x, pos, base):
    """RoPE as complex multiplication: (x_k + i x_{k+D/2}) * e^{i pos theta_k}."""
    D = x.shape[-1]
    half = D // 2
    theta = np.array([base ** (-(2.0 * k) / D) for k in range(half)])
    z = (x[..., :half] + 1j * x[..., half:]) * np.exp(1j * np.asarray(pos)[..., None] * theta)
    return np.concatenate([z.real, z.imag], axis=-1)


# --------------------------------------------------------------------------
# pins
# --------------------------------------------------------------------------

def pin_worked_tables():
    for name, s, c in TABLES:
        want_pc, want_d = parse_table(name)
        L = want_pc.shape[0]
        qpos, kpos, pc = orc.index_map(L, s, c)
        assert (pc == want_pc).all(), name
        d = np.where(pc >= 0, qpos - kpos, -1)
        assert (d == want_d).all(), name
        jj = np.broadcast_to(np.arange(L), (L, L))
        assert (kpos[pc >= 0] == (jj % s)[pc >= 0]).all(), name


def pin_distance_bounds():
    for s, c in [(4, 6), (3, 5), (5, 8), (8, 8), (2, 5), (7, 9), (192, 256), (1, 1)]:
        for L in list(range(1, 41)) + [3 * c + 7]:
            qpos, kpos, pc = orc.index_map(L, s, c)
            i = np.arange(L)[:, None] + 0 * np.arange(L)[None, :]
            j = np.arange(L)[None, :] + 0 * np.arange(L)[:, None]
            causal = j <= i
            assert ((pc >= 0) == causal).all()
            d = qpos - kpos
            assert d[causal].min() >= 0 and d[causal].max() <= c - 1
            intra = pc == orc.PIECE_INTRA
            assert (d[intra] == (i - j)[intra]).all()
            near = (pc == orc.PIECE_SUCC) & ((i % s) < c - s)
            assert (d[near] == (i - j)[near]).all()
            far = ((pc == orc.PIECE_SUCC) & ((i % s) >= c - s)) | (pc == orc.PIECE_INTER)
            assert (d[far] >= c - s).all() and (d[far] <= c - 1).all()


def closed_form_counts(L, s):
    n = [min(s, L - k * s) for k in range(-(-L // s))]
    intra = sum(nk * (nk + 1) // 2 for nk in n)
    succ = sum(nk * s for nk in n[1:])
    inter = sum(nk * (k - 1) * s for k, nk in enumerate(n) if k >= 2)
    return intra, succ, inter


def pin_piece_counts():
    # tiny prefill workload: L=1024, s=192 (c=256); sums to L(L+1)/2
    qpos, kpos, pc = orc.index_map(1024, 192, 256)
    got = tuple(int((pc == p).sum()) for p in (0, 1, 2))
    assert got == (94720, 159744, 270336)
    assert sum(got) == 1024 * 1025 // 2
    for L, s, c in [(1, 3, 5), (17, 4, 6), (40, 5, 8), (100, 7, 9), (64, 16, 16)]:
        qpos, kpos, pc = orc.index_map(L, s, c)
        got = tuple(int((pc == p).sum()) for p in (0, 1, 2))
        assert got == closed_form_counts(L, s)


def pin_rotation_literals():
    # D=4, base 10000: theta = (1, 0.01); half-split pairs (0,2) and (1,3)
    e0, e1 = np.array([1.0, 0, 0, 0]), np.array([0, 1.0, 0, 0])
    e2 = np.array([0, 0, 1.0, 0])
    np.testing.assert_allclose(orc.rotate(e0, 1, 10000.0),
                               [math.cos(1), 0, math.sin(1), 0], atol=1e-15)
    np.testing.assert_allclose(orc.rotate(e1, 1, 10000.0),
                               [0, math.cos(0.01), 0, math.sin(0.01)], atol=1e-15)
    np.testing.assert_allclose(orc.rotate(e2, 3, 10000.0),
                               [-math.sin(3), 0, math.cos(3), 0], atol=1e-15)
    x = _rand((5, 7, 3, 16), 1)
    pos = np.arange(7)[None, :, None] * 37
    np.testing.assert_allclose(orc.rotate(x, pos, 500.0),
                               _complex_rotate(x, pos, 500.0), atol=1e-12)


def pin_rope_relativity():
    q, k = _rand(16, 2), _rand(16, 3)
    for p, r in [(0, 0), (5, 2), (255, 0), (4095, 3071)]:
        ref = orc.rotate(q, p, 10000.0) @ orc.rotate(k, r, 10000.0)
        for delta in (1, 17, 1000):
            got = orc.rotate(q, p + delta, 10000.0) @ orc.rotate(k, r + delta, 10000.0)
            assert abs(got - ref) < 1e-12


def _sdpa_reference(Q, K, V, base):
    """Causal RoPE attention via torch SDPA (fp64 CPU), complex-rotated inputs."""
    B, L, Hq, D = Q.shape
    G = Hq // K.shape[2]
    pos = np.arange(L)[None, :, None]
    qr = torch.from_numpy(_complex_rotate(Q, pos, base)).permute(0, 2, 1, 3)
    kr = torch.from_numpy(_complex_rotate(K, pos, base)).permute(0, 2, 1, 3)
    v = torch.from_numpy(np.asarray(V, np.float64)).permute(0, 2, 1, 3)
    kr, v = kr.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1)
    O = torch.nn.functional.scaled_dot_product_attention(qr, kr, v, is_causal=True)
    z = (qr @ kr.transpose(-1, -2)) / math.sqrt(D)
    z = z.masked_fill(torch.ones(L, L, dtype=torch.bool).triu(1), -math.inf)
    lse = torch.logsumexp(z, dim=-1)
    return O.permute(0, 2, 1, 3).numpy(), lse.numpy()


def pin_plain_rope_matches_sdpa():
    Q, K, V = _rand((2, 13, 4, 8), 4), _rand((2, 13, 2, 8), 5), _rand((2, 13, 2, 8), 6)
    O, LSE = orc.plain_rope_attention(Q, K, V, base=100.0)
    O_ref, LSE_ref = _sdpa_reference(Q, K, V, 100.0)
    np.testing.assert_allclose(O, O_ref, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_ref, atol=1e-12)


def pin_single_chunk_is_plain_rope():
    # L <= s: every pair is intra and both positions are absolute
    Q, K, V = _rand((1, 11, 4, 8), 7), _rand((1, 11, 2, 8), 8), _rand((1, 11, 2, 8), 9)
    O, LSE = orc.dca_prefill(Q, K, V, s=12, c=16, base=100.0)
    O_ref, LSE_ref = _sdpa_reference(Q, K, V, 100.0)
    np.testing.assert_allclose(O, O_ref, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_ref, atol=1e-12)
    # L <= c with w <= s: chunk-1 queries all have i mod s < w, so the
    # successive piece sees i - j and DCA is again plain RoPE attention
    Q, K, V = _rand((1, 16, 2, 8), 10), _rand((1, 16, 2, 8), 11), _rand((1, 16, 2, 8), 12)
    O, LSE = orc.dca_prefill(Q, K, V, s=10, c=16, base=100.0)
    O_ref, LSE_ref = _sdpa_reference(Q, K, V, 100.0)
    np.testing.assert_allclose(O, O_ref, atol=1e-10)
    np.testing.assert_allclose(LSE, LSE_ref, atol=1e-10)


def pin_long_sequence_differs_from_plain():
    # beyond c the remapping must change the result (guards a no-op oracle)
    Q, K, V = _rand((1, 24, 1, 8), 13), _rand((1, 24, 1, 8), 14), _rand((1, 24, 1, 8), 15)
    O, _ = orc.dca_prefill(Q, K, V, s=4, c=6, base=2.0)
    O_ref, _ = _sdpa_reference(Q, K, V, 2.0)
    assert np.abs(O - O_ref)[0, 6:].max() > 1e-3
    np.testing.assert_allclose(O[0, :4], O_ref[0, :4], atol=1e-12)


def pin_q_zero_closed_form():
    L = 40
    K, V = _rand((1, L, 2, 8), 16), _rand((1, L, 2, 8), 17)
    Q = np.zeros((1, L, 4, 8))
    O, LSE = orc.dca_prefill(Q, K, V, s=6, c=10)
    for i in range(L):
        for h in range(4):
            np.testing.assert_allclose(LSE[0, h, i], math.log(i + 1), atol=1e-13)
            np.testing.assert_allclose(O[0, i, h], V[0, :i + 1, h // 2].mean(0), atol=1e-13)


def pin_constant_v():
    L = 30
    Q, K = _rand((1, L, 2, 8), 18), _rand((1, L, 1, 8), 19)
    v = _rand(8, 20)
    V = np.broadcast_to(v, (1, L, 1, 8)).copy()
    O, _ = orc.dca_prefill(Q, K, V, s=5, c=8)
    np.testing.assert_allclose(O[0], np.broadcast_to(v, (L, 2, 8)), atol=1e-13)


def pin_gqa_mapping():
    # q head h reads kv head h // G: same as expanding K, V by repeat_interleave
    Q, K, V = _rand((1, 20, 6, 8), 21), _rand((1, 20, 2, 8), 22), _rand((1, 20, 2, 8), 23)
    O, LSE = orc.dca_prefill(Q, K, V, s=4, c=7)
    Ke, Ve = np.repeat(K, 3, axis=2), np.repeat(V, 3, axis=2)
    O2, LSE2 = orc.dca_prefill(Q, Ke, Ve, s=4, c=7)
    np.testing.assert_allclose(O, O2, atol=1e-14)
    np.testing.assert_allclose(LSE, LSE2, atol=1e-14)


def pin_decode_equals_prefill_row():
    B, L, s, c = 2, 30, 6, 10
    Q, K, V = _rand((B, L, 4, 8), 24), _rand((B, L, 2, 8), 25), _rand((B, L, 2, 8), 26)
    k_rot = _complex_rotate(K, (np.arange(L) % s)[None, :, None], 10000.0)
    t = np.array([29, 17])
    q = np.stack([Q[b, t[b]] for b in range(B)])
    O, LSE = orc.dca_decode(q, k_rot, V, t, s, c)
    for b in range(B):
        ref = orc.dca_prefill_rows(Q[b:b + 1], K[b:b + 1], V[b:b + 1], s, c,
                                   rows=[int(t[b])])
        for h in range(4):
            o, lse = ref[(0, h, int(t[b]))]
            np.testing.assert_allclose(O[b, h], o, atol=1e-12)
            np.testing.assert_allclose(LSE[b, h], lse, atol=1e-12)


def pin_chunk_equals_prefill_rows():
    # a chunk at t0 over a cache holding the earlier keys (rotated here by the
    # independent complex-number RoPE at j mod s) gives rows t0 + r of the
    # whole-sequence prefill, for chunk starts inside and at chunk boundaries
    B, L, s, c = 2, 31, 6, 10
    Q, K, V = _rand((B, L, 4, 8), 40), _rand((B, L, 2, 8), 41), _rand((B, L, 2, 8), 42)
    k_rot = _complex_rotate(K, (np.arange(L) % s)[None, :, None], 10000.0)
    full = orc.dca_prefill_rows(Q, K, V, s, c)
    for t0, e in [(0, 9), (6, 13), (13, 31), (30, 31)]:
        got = orc.dca_prefill_chunk(Q[:, t0:e], K[:, t0:e], V[:, t0:e], k_rot[:, :t0],
                                    V[:, :t0], t0, s, c)
        assert len(got) == B * 4 * (e - t0)
        for (b, h, r), (o, lse) in got.items():
            o_ref, lse_ref = full[(b, h, t0 + r)]
            np.testing.assert_allclose(o, o_ref, atol=1e-12)
            np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


def pin_varlen_equals_padded_batch():
    # equal-length sequences packed back to back give the rows of the padded
    # batch [B, n]; n is not a multiple of s, so counting chunks from the
    # packed start (or attending an earlier sequence) moves them
    B, n, s, c = 3, 17, 5, 8
    Q, K, V = _rand((B, n, 4, 8), 43), _rand((B, n, 2, 8), 44), _rand((B, n, 2, 8), 45)
    cu = [b * n for b in range(B + 1)]
    got = orc.dca_prefill_varlen_rows(Q.reshape(B * n, 4, 8), K.reshape(B * n, 2, 8),
                                      V.reshape(B * n, 2, 8), cu, s, c)
    assert set(got) == {(h, t) for h in range(4) for t in range(B * n)}
    full = orc.dca_prefill_rows(Q, K, V, s, c)
    for (h, t), (o, lse) in got.items():
        o_ref, lse_ref = full[(t // n, h, t % n)]
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


def pin_varlen_q_zero_closed_form():
    # Q = 0: every score is 0, so LSE = ln(r + 1) and O is the mean of the
    # sequence's own values 0 .. r (local row r); rows before the first
    # sequence, after the last one and empty sequences produce nothing
    lens = [7, 1, 12, 0, 9]
    cu = [2]
    for n in lens:
        cu.append(cu[-1] + n)
    T = cu[-1] + 3
    K, V = _rand((T, 2, 8), 46), _rand((T, 2, 8), 47)
    Q = np.zeros((T, 4, 8))
    got = orc.dca_prefill_varlen_rows(Q, K, V, cu, s=4, c=6)
    assert set(got) == {(h, t) for h in range(4) for t in range(cu[0], cu[-1])}
    for b in range(len(lens)):
        for t in range(cu[b], cu[b + 1]):
            r = t - cu[b]
            for h in range(4):
                o, lse = got[(h, t)]
                np.testing.assert_allclose(lse, math.log(r + 1), atol=1e-13)
                np.testing.assert_allclose(o, V[cu[b]:t + 1, h // 2].mean(0), atol=1e-13)


def pin_varlen_chunk_equals_whole_sequences():
    # next chunks of three sequences at offsets 7, 0 and 12, packed: each
    # packed row equals row t0[b] + r of sequence b's whole-sequence prefill,
    # with the cached keys rotated by the independent complex-number RoPE
    s, c = 5, 8
    t0, n = [7, 0, 12], [6, 4, 9]
    B, Lmax = 3, max(a + m for a, m in zip(t0, n))
    Q, K, V = _rand((B, Lmax, 2, 8), 48), _rand((B, Lmax, 1, 8), 49), _rand((B, Lmax, 1, 8), 50)
    k_rot = _complex_rotate(K, (np.arange(Lmax) % s)[None, :, None], 10000.0)
    cu = [0]
    for m in n:
        cu.append(cu[-1] + m)
    pack = lambda X: np.concatenate([X[b, t0[b]:t0[b] + n[b]] for b in range(B)])
    got = orc.dca_prefill_varlen_chunk_rows(pack(Q), pack(K), pack(V), cu, t0, k_rot, V, s, c)
    assert set(got) == {(h, t) for h in range(2) for t in range(cu[-1])}
    for b in range(B):
        full = orc.dca_prefill_rows(Q[b:b + 1, :t0[b] + n[b]], K[b:b + 1, :t0[b] + n[b]],
                                    V[b:b + 1, :t0[b] + n[b]], s, c)
        for r in range(n[b]):
            for h in range(2):
                o, lse = got[(h, cu[b] + r)]
                np.testing.assert_allclose(o, full[(0, h, t0[b] + r)][0], atol=1e-12)
                np.testing.assert_allclose(lse, full[(0, h, t0[b] + r)][1], atol=1e-12)


def pin_varlen_chunk_q_zero_closed_form():
    # Q = 0: LSE = ln(t0[b] + r + 1), O = mean of the cached values and the new
    # values up to the row
    t0, n = [3, 0, 10], [5, 2, 4]
    cu = [0, 5, 7, 11]
    Kc, Vc = _rand((3, 16, 2, 8), 51), _rand((3, 16, 2, 8), 52)
    K, V = _rand((11, 2, 8), 53), _rand((11, 2, 8), 54)
    Q = np.zeros((11, 4, 8))
    got = orc.dca_prefill_varlen_chunk_rows(Q, K, V, cu, t0, Kc, Vc, s=4, c=6)
    for b in range(3):
        for r in range(n[b]):
            t = cu[b] + r
            for h in range(4):
                o, lse = got[(h, t)]
                vals = np.concatenate([Vc[b, :t0[b], h // 2], V[cu[b]:t + 1, h // 2]])
                np.testing.assert_allclose(lse, math.log(t0[b] + r + 1), atol=1e-13)
                np.testing.assert_allclose(o, vals.mean(0), atol=1e-13)


def pin_merge_partials():
    z, v = _rand(50, 27) * 3, _rand((50, 8), 28)
    o_full, lse_full = orc.softmax_row(z, v)
    cuts = [0, 7, 31, 50]
    parts = [orc.softmax_row(z[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
    o, lse = orc.merge_partials([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(o, o_full, atol=1e-13)
    np.testing.assert_allclose(lse, lse_full, atol=1e-13)
    # LSE is the natural-log normaliser of the scaled scores
    np.testing.assert_allclose(lse_full, math.log(np.exp(z).sum()), atol=1e-12)


def pin_rule_positions():
    s, c = 5, 8
    n = 23
    i = np.arange(n)
    assert (orc.rule_positions(n, orc.POS_KEY, s, c) == i % s).all()
    assert (orc.rule_positions(n, orc.POS_Q_INTRA, s, c) == i % s).all()
    assert (orc.rule_positions(n, orc.POS_Q_INTER, s, c) == c - 1).all()
    assert (orc.rule_positions(n, orc.POS_ABSOLUTE, s, c, 9) == i + 9).all()
    # derived closed form of the successive rule: min(s + i mod s, c - 1)
    for s2, c2 in [(5, 8), (3, 3), (2, 5), (3072, 4096)]:
        m = 3 * s2 + 1
        got = orc.rule_positions(m, orc.POS_Q_SUCC, s2, c2)
        assert (got == np.minimum(s2 + np.arange(m) % s2, c2 - 1)).all()
    # the successive rule agrees with the index map's previous-chunk column
    qpos, _, pc = orc.index_map(n, s, c)
    succ = orc.rule_positions(n, orc.POS_Q_SUCC, s, c)
    for r in range(s, n):
        assert qpos[r, (r // s - 1) * s] == succ[r]


def pin_selfextend_worked_tables():
    # hand-worked neighbour / grouped distance tables
    for name, G, W in SE_TABLES:
        want_lv, want_d = parse_table(name, {"N": 0, "G": 1})
        L = want_lv.shape[0]
        for i in range(L):
            j = np.arange(i + 1)
            qpos, kpos = orc.selfextend_positions(i, j, G, W)
            assert (qpos - kpos == want_d[i, :i + 1]).all(), (name, i)
            grouped = (i - j) >= W
            assert (grouped.astype(np.int8) == want_lv[i, :i + 1]).all(), (name, i)
            # neighbours keep the original absolute positions
            assert (qpos[~grouped] == i).all() and (kpos[~grouped] == j[~grouped]).all()


def pin_selfextend_reduces_to_plain_rope():
    # G = 1 (no grouping) and W >= L (every key a neighbour) are plain RoPE
    # attention, checked against torch SDPA over complex-rotated inputs
    Q, K, V = _rand((1, 17, 4, 8), 50), _rand((1, 17, 2, 8), 51), _rand((1, 17, 2, 8), 52)
    O_ref, LSE_ref = _sdpa_reference(Q, K, V, 100.0)
    for G, W in [(1, 1), (1, 5), (4, 17), (3, 40)]:
        got = orc.selfextend_prefill_rows(Q, K, V, G, W, base=100.0)
        for (b, h, i), (o, lse) in got.items():
            np.testing.assert_allclose(o, O_ref[b, i, h], atol=1e-12)
            np.testing.assert_allclose(lse, LSE_ref[b, h, i], atol=1e-12)
    # with grouping active beyond W the result must differ from plain RoPE
    got = orc.selfextend_prefill_rows(Q, K, V, 2, 3, base=2.0, rows=[16])
    O2, _ = _sdpa_reference(Q, K, V, 2.0)
    assert np.abs(got[(0, 0, 16)][0] - O2[0, 16, 0]).max() > 1e-3


def pin_selfextend_distance_bounds():
    # grouped pairs are never closer than the window; the largest distance is
    # floor((L-1)/G) + W - floor(W/G); distances never decrease as j moves away
    for G, W, L in [(2, 3, 40), (4, 16, 200), (8, 5, 120), (3, 1, 50)]:
        for i in range(L):
            j = np.arange(i + 1)
            qpos, kpos = orc.selfextend_positions(i, j, G, W)
            d = qpos - kpos
            assert (d[(i - j) >= W] >= W).all()
            assert d.max() <= (L - 1) // G + W - W // G
            assert (np.diff(d[::-1]) >= 0).all()


def pin_rope_rotate():
    # rope_rotate on [B, L, H, D] with L != H: row r of every batch entry and
    # head is turned to the rule's position of absolute index pos_offset + r.
    # The positions are listed per row here from the rule as the pages state
    # it; the rotation is the complex-number RoPE.
    s, c = 5, 8
    x = _rand((2, 11, 3, 8), 60)
    for off in (0, 17, s - 1, 3 * s + 2):
        for rule in (orc.POS_KEY, orc.POS_Q_INTRA, orc.POS_Q_SUCC, orc.POS_Q_INTER,
                     orc.POS_ABSOLUTE):
            want_pos = []
            for r in range(x.shape[1]):
                i = off + r
                if rule == orc.POS_ABSOLUTE:
                    want_pos.append(i)
                elif rule in (orc.POS_KEY, orc.POS_Q_INTRA):
                    want_pos.append(i % s)
                elif rule == orc.POS_Q_SUCC:
                    want_pos.append(s + i % s if i % s < c - s else c - 1)
                else:
                    want_pos.append(c - 1)
            want = _complex_rotate(x, np.array(want_pos)[None, :, None], 100.0)
            got = orc.rope_rotate(x, rule, s, c, 100.0, pos_offset=off)
            assert got.shape == x.shape
            np.testing.assert_allclose(got, want, atol=1e-12, err_msg=f"rule {rule} off {off}")
    # literal values, D = 2 (one pair, theta_0 = 1): x = (1, 0) turned by the
    # angle p gives (cos p, sin p).  s = 3, c = 5 (w = 2): index 4 has
    # 4 mod 3 = 1 < w, so the successive position is 3 + 1 = 4; index 5 has
    # 5 mod 3 = 2 >= w, so it is c - 1 = 4 as well; index 3 has intra 0.
    e = np.zeros((1, 3, 1, 2))
    e[..., 0] = 1.0
    got = orc.rope_rotate(e, orc.POS_Q_SUCC, 3, 5, 10000.0, pos_offset=3)
    np.testing.assert_allclose(got[0, :, 0], [[math.cos(3), math.sin(3)],
                                              [math.cos(4), math.sin(4)],
                                              [math.cos(4), math.sin(4)]], atol=1e-15)
    got = orc.rope_rotate(e, orc.POS_Q_INTRA, 3, 5, 10000.0, pos_offset=3)
    np.testing.assert_allclose(got[0, :, 0], [[1, 0], [math.cos(1), math.sin(1)],
                                              [math.cos(2), math.sin(2)]], atol=1e-15)


def _softmax_from_distances(q, k, v, dist, base, sc):
    """Row outputs from an explicit distance per key: by RoPE relativity the
    score of the pair is <R(d) q, k>, so only the distance is needed."""
    z = np.array([_complex_rotate(q, d, base) @ k[n] for n, d in enumerate(dist)]) * sc
    m = z.max()
    e = np.exp(z - m)
    return (e @ v) / e.sum(), m + math.log(e.sum())


def pin_dca_rows_from_worked_tables():
    # every row of a DCA prefill rebuilt from the hand-worked distance tables
    # alone: score = scale * <R(d_ij) q_i, k_j>, one naive softmax per row
    for name, s, c in TABLES:
        _, want_d = parse_table(name)
        L = want_d.shape[0]
        Q, K, V = _rand((1, L, 2, 8), 61), _rand((1, L, 1, 8), 62), _rand((1, L, 1, 8), 63)
        O, LSE = orc.dca_prefill(Q, K, V, s, c, base=100.0)
        for h in range(2):
            for i in range(L):
                o, lse = _softmax_from_distances(Q[0, i, h], K[0, :i + 1, 0], V[0, :i + 1, 0],
                                                 want_d[i, :i + 1], 100.0, 1 / math.sqrt(8))
                np.testing.assert_allclose(O[0, i, h], o, atol=1e-12, err_msg=name)
                np.testing.assert_allclose(LSE[0, h, i], lse, atol=1e-12, err_msg=name)


def pin_selfextend_rows_from_worked_tables():
    # every SelfExtend row rebuilt from the hand-worked neighbour / grouped
    # distance tables alone, as for the DCA rows above
    for name, G, W in SE_TABLES:
        _, want_d = parse_table(name, {"N": 0, "G": 1})
        L = want_d.shape[0]
        Q, K, V = _rand((1, L, 2, 8), 64), _rand((1, L, 1, 8), 65), _rand((1, L, 1, 8), 66)
        got = orc.selfextend_prefill_rows(Q, K, V, G, W, base=100.0)
        assert len(got) == 2 * L
        for (b, h, i), (o, lse) in got.items():
            o_ref, lse_ref = _softmax_from_distances(Q[0, i, h], K[0, :i + 1, 0],
                                                     V[0, :i + 1, 0], want_d[i, :i + 1],
                                                     100.0, 1 / math.sqrt(8))
            np.testing.assert_allclose(o, o_ref, atol=1e-12, err_msg=name)
            np.testing.assert_allclose(lse, lse_ref, atol=1e-12, err_msg=name)


PINS = [pin_worked_tables, pin_distance_bounds, pin_piece_counts,
        pin_rotation_literals, pin_rope_relativity, pin_plain_rope_matches_sdpa,
        pin_single_chunk_is_plain_rope, pin_long_sequence_differs_from_plain,
        pin_q_zero_closed_form, pin_constant_v, pin_gqa_mapping,
        pin_decode_equals_prefill_row, pin_chunk_equals_prefill_rows,
        pin_varlen_equals_padded_batch, pin_varlen_q_zero_closed_form,
        pin_varlen_chunk_equals_whole_sequences, pin_varlen_chunk_q_zero_closed_form,
        pin_merge_partials,
        pin_rule_positions, pin_rope_rotate, pin_dca_rows_from_worked_tables,
        pin_selfextend_worked_tables, pin_selfextend_reduces_to_plain_rope,
        pin_selfextend_distance_bounds, pin_selfextend_rows_from_worked_tables]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


def test_rejects_bad_chunking():
    with pytest.raises(ValueError):
        orc.index_map(8, 5, 4)
    with pytest.raises(ValueError):
        orc.index_map(8, 0, 4)
