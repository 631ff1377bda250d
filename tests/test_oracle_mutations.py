"""Plausible mistakes planted in the oracle must each fail at least one pin.

Every mutant replaces one oracle function (on the CPU, through monkeypatch)
with a version carrying a typical slip: an off-by-one in the successive rule,
a dropped modulo, interleaved instead of half-split RoPE pairing, a flipped
sign, a wrong frequency exponent, a missing softmax scale, a log2 LSE, a
causal off-by-one, a wrong GQA mapping, a shifted chunk origin, a broken
partial merge, a decode that reads one key too few, a chunked prefill
that ignores or misaligns its cache, or a packed variable-length batch that
leaks across sequences, counts positions from the packed start or reports
local rows, packed chunks that ignore their cache offsets or read
another sequence's cache, a tensor rotation that drops its position offset
or lays positions along the head axis, a SelfExtend row that rotates a
grouped query at its own index, and a DCA row that rotates its query once
for all keys.  The pins of
``test_oracle_pins`` must reject each one.
"""

import numpy as np
import pytest

from oracle import dca_oracle as orc
from tests import test_oracle_pins as pins

_orig_query_position = orc.query_position
_orig_rotate = orc.rotate
_orig_piece = orc.piece
_orig_softmax_row = orc.softmax_row


def _qpos_succ_le(i, j, s, c):
    i = np.asarray(i, np.int64)
    j = np.asarray(j, np.int64)
    im = i % s
    p = orc.piece(i, j, s)
    succ = np.where(im <= c - s, s + im, c - 1)
    out = np.where(p == 0, im, np.where(p == 1, succ, c - 1))
    return np.where(p < 0, -1, out)


def _qpos_succ_c(i, j, s, c):
    out = _orig_query_position(i, j, s, c)
    i = np.asarray(i, np.int64)
    p = orc.piece(i, j, s)
    return np.where((p == 1) & (i % s >= c - s), c, out)


def _qpos_inter_succ(i, j, s, c):
    # inter piece wrongly treated like the successive piece
    i = np.asarray(i, np.int64)
    j = np.asarray(j, np.int64)
    im = i % s
    p = orc.piece(i, j, s)
    succ = np.where(im < c - s, s + im, c - 1)
    out = np.where(p == 0, im, succ)
    return np.where(p < 0, -1, out)


def _qpos_succ_as_intra(i, j, s, c):
    out = _orig_query_position(i, j, s, c)
    p = orc.piece(i, j, s)
    return np.where(p == 1, np.asarray(i) % s, out)


def _key_abs(j, s):
    return np.asarray(j, np.int64)


def _rotate_interleaved(x, pos, base):
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    ang = np.asarray(pos, np.float64)[..., None] * orc.inv_freq(D, base)
    cos, sin = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * cos - b * sin
    out[..., 1::2] = b * cos + a * sin
    return out


def _rotate_sign(x, pos, base):
    return _orig_rotate(x, -np.asarray(pos), base)


def _inv_freq_half(D, base):
    k = np.arange(D // 2, dtype=np.float64)
    return np.power(np.float64(base), -k / D)


def _scale_one(D, scale):
    return 1.0


def _softmax_log2(z, v):
    o, lse = _orig_softmax_row(z, v)
    return o, lse / np.log(2.0)


def _softmax_drop_last(z, v):
    # causal off-by-one: the diagonal key is left out of the row
    if len(z) == 1:
        return _orig_softmax_row(z, v)
    return _orig_softmax_row(z[:-1], v[:-1])


def _kv_head_mod(h, Hq, Hkv):
    return h % Hkv


def _piece_shift(i, j, s):
    i = np.asarray(i, np.int64)
    j = np.asarray(j, np.int64)
    diff = (i + 1) // s - (j + 1) // s
    out = np.where(diff == 0, 0, np.where(diff == 1, 1, 2))
    return np.where(j > i, -1, out).astype(np.int8)


def _merge_mean(o_parts, lse_parts):
    return np.mean(np.asarray(o_parts), axis=0), np.max(lse_parts)


def _decode_short(q, k_cache_rot, v_cache, t, s, c, base=10000.0, scale=0.0,
                  batches=None, heads=None):
    return _ORIG_DECODE(q, k_cache_rot, v_cache, np.asarray(t) - 1, s, c, base,
                        scale, batches, heads)


_ORIG_DECODE = orc.dca_decode
_ORIG_CHUNK = orc.dca_prefill_chunk
_ORIG_SE_POS = orc.selfextend_positions


def _se_no_shift(i, j, G, W):
    # grouped query at floor(i/G) without the W - floor(W/G) shift
    q, k = _ORIG_SE_POS(i, j, G, W)
    far = (np.asarray(i) - np.asarray(j)) >= W
    return np.where(far, np.asarray(i) // G, q), k


def _se_window_le(i, j, G, W):
    # neighbour window one too wide (i - j <= W)
    q, k = _ORIG_SE_POS(i, j, G, W)
    at = (np.asarray(i) - np.asarray(j)) == W
    return np.where(at, np.asarray(i), q), np.where(at, np.asarray(j), k)


def _se_key_not_grouped(i, j, G, W):
    q, k = _ORIG_SE_POS(i, j, G, W)
    far = (np.asarray(i) - np.asarray(j)) >= W
    return q, np.where(far, np.asarray(j), k)


def _chunk_ignores_cache(Qc, Kc, Vc, k_cache_rot, v_cache, t0, s, c, *args, **kw):
    # the chunk attends to its own keys only, as if it started the sequence
    return _ORIG_CHUNK(Qc, Kc, Vc, k_cache_rot[:, :0], v_cache[:, :0], 0, s, c, *args, **kw)


def _chunk_start_early(Qc, Kc, Vc, k_cache_rot, v_cache, t0, s, c, *args, **kw):
    # off-by-one chunk start: one cached key too few, the chunk placed at t0 - 1
    t = max(t0 - 1, 0)
    return _ORIG_CHUNK(Qc, Kc, Vc, k_cache_rot[:, :t], v_cache[:, :t], t, s, c, *args, **kw)

_ORIG_VARLEN = orc.dca_prefill_varlen_rows


def _varlen_whole_pack(Q, K, V, cu_seqlens, s, c, base=10000.0, scale=0.0, rows=None,
                       heads=None):
    # the packed tensor treated as one sequence: earlier sequences attended,
    # chunks counted from the packed start
    cu = [int(x) for x in cu_seqlens]
    want = [t for t in range(cu[0], cu[-1]) if rows is None or t in set(rows)]
    res = orc.dca_prefill_rows(Q[None], K[None], V[None], s, c, base, scale, rows=want,
                               heads=heads)
    return {(h, t): val for (_, h, t), val in res.items()}


def _varlen_global_positions(Q, K, V, cu_seqlens, s, c, base=10000.0, scale=0.0, rows=None,
                             heads=None):
    # own keys only, but query and key positions taken from the packed index
    cu = [int(x) for x in cu_seqlens]
    T, Hq, D = Q.shape
    G = Hq // K.shape[1]
    sc = 1.0 / np.sqrt(D) if not scale else scale
    out = {}
    for b in range(len(cu) - 1):
        a = cu[b]
        for t in range(a, cu[b + 1]):
            if rows is not None and t not in set(rows):
                continue
            j = np.arange(a, t + 1)
            pq = orc.query_position(t, j, s, c)
            for h in range(Hq) if heads is None else heads:
                k_rot = orc.rotate(K[a:t + 1, h // G], orc.key_position(j, s), base)
                z = np.array([k_rot[n] @ orc.rotate(Q[t, h], pq[n], base)
                              for n in range(len(j))])
                out[(h, t)] = orc.softmax_row(sc * z, V[a:t + 1, h // G])
    return out


def _varlen_local_keys(*args, **kw):
    # results keyed from the first sequence's start instead of packed row 0
    return {(h, t - min(tt for _, tt in _ORIG_VARLEN(*args, **kw))): v
            for (h, t), v in _ORIG_VARLEN(*args, **kw).items()}


_ORIG_VARLEN_CHUNK = orc.dca_prefill_varlen_chunk_rows


def _varlen_chunk_no_offset(Q, K, V, cu_seqlens, t0, k_cache_rot, v_cache, *args, **kw):
    # every sequence's chunk taken as its first tokens (cache offsets ignored)
    return _ORIG_VARLEN_CHUNK(Q, K, V, cu_seqlens, [0] * len(t0), k_cache_rot, v_cache, *args,
                              **kw)


def _varlen_chunk_first_cache(Q, K, V, cu_seqlens, t0, k_cache_rot, v_cache, *args, **kw):
    # every sequence reads batch entry 0 of the caches
    B = len(t0)
    return _ORIG_VARLEN_CHUNK(Q, K, V, cu_seqlens, t0, np.repeat(k_cache_rot[:1], B, axis=0),
                              np.repeat(v_cache[:1], B, axis=0), *args, **kw)


_ORIG_RULE_POS = orc.rule_positions
_ORIG_SE_ROW = orc.selfextend_row
_ORIG_DCA_ROW = orc.dca_row


def _rope_rotate_no_offset(x, rule, s, c, base, pos_offset=0):
    # pos_offset dropped: every call rotates as if the rows started at index 0
    x = np.asarray(x, np.float64)
    pos = _ORIG_RULE_POS(x.shape[1], rule, s, c, 0)
    return orc.rotate(x, pos[None, :, None], base)


def _rope_rotate_head_axis(x, rule, s, c, base, pos_offset=0):
    # positions laid along the head axis instead of the row axis
    x = np.asarray(x, np.float64)
    pos = _ORIG_RULE_POS(x.shape[2], rule, s, c, pos_offset)
    return orc.rotate(x, pos[None, None, :], base)


def _se_row_query_at_i(q, k, v, i, G, W, base, scale):
    # grouped pairs rotate the query at its own index i instead of the
    # shifted grouped position
    j = np.arange(i + 1, dtype=np.int64)
    _, kpos = orc.selfextend_positions(i, j, G, W)
    z = orc.rotate(k, kpos, base) @ orc.rotate(q, i, base)
    return orc.softmax_row(scale * z, v)


def _dca_row_one_rotation(q, k_rot, v, i, s, c, base, scale):
    # the query rotated once, at the position its first key asks for, and
    # used for every key
    pq = orc.query_position(i, np.arange(i + 1), s, c)
    z = k_rot @ orc.rotate(q, pq[0], base)
    return orc.softmax_row(scale * z, v)


MUTANTS = {
    "succ_rule_le": ("query_position", _qpos_succ_le),
    "succ_far_pos_c": ("query_position", _qpos_succ_c),
    "inter_as_succ": ("query_position", _qpos_inter_succ),
    "succ_as_intra": ("query_position", _qpos_succ_as_intra),
    "key_not_mod_s": ("key_position", _key_abs),
    "rope_interleaved": ("rotate", _rotate_interleaved),
    "rope_sign": ("rotate", _rotate_sign),
    "theta_exponent": ("inv_freq", _inv_freq_half),
    "no_softmax_scale": ("_scale", _scale_one),
    "lse_log2": ("softmax_row", _softmax_log2),
    "causal_off_by_one": ("softmax_row", _softmax_drop_last),
    "gqa_modulo": ("kv_head", _kv_head_mod),
    "chunk_origin_shift": ("piece", _piece_shift),
    "merge_mean": ("merge_partials", _merge_mean),
    "decode_short": ("dca_decode", _decode_short),
    "chunk_ignores_cache": ("dca_prefill_chunk", _chunk_ignores_cache),
    "chunk_start_early": ("dca_prefill_chunk", _chunk_start_early),
    "selfextend_no_shift": ("selfextend_positions", _se_no_shift),
    "selfextend_window_le": ("selfextend_positions", _se_window_le),
    "selfextend_key_not_grouped": ("selfextend_positions", _se_key_not_grouped),
    "varlen_whole_pack": ("dca_prefill_varlen_rows", _varlen_whole_pack),
    "varlen_global_positions": ("dca_prefill_varlen_rows", _varlen_global_positions),
    "varlen_local_keys": ("dca_prefill_varlen_rows", _varlen_local_keys),
    "varlen_chunk_no_offset": ("dca_prefill_varlen_chunk_rows", _varlen_chunk_no_offset),
    "varlen_chunk_first_cache": ("dca_prefill_varlen_chunk_rows", _varlen_chunk_first_cache),
    "rope_rotate_no_offset": ("rope_rotate", _rope_rotate_no_offset),
    "rope_rotate_head_axis": ("rope_rotate", _rope_rotate_head_axis),
    "selfextend_query_at_i": ("selfextend_row", _se_row_query_at_i),
    "dca_row_one_rotation": ("dca_row", _dca_row_one_rotation),
}


def _some_pin_fails():
    for pin in pins.PINS:
        try:
            pin()
        except AssertionError:
            return True
    return False


def test_unmutated_oracle_passes_every_pin():
    assert not _some_pin_fails()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(orc, attr, fn)
    assert _some_pin_fails(), f"mutant {name} passed every pin"
