"""GPU parity: the CUDA library (called through its C ABI) against the fp64
oracle on the same seeded inputs.

Index maps are compared bit-exactly; RoPE outputs within bf16 rounding of the
fp64 rotation; attention outputs within max-abs 2e-2 / mean-abs 2e-3 on O and
1e-3 relative on LSE (see parity_util).  Small cases compare every output;
the full-size workloads compare sampled rows (every chunk's first and last
row, rows around i mod s = w, the ragged tail, seeded random rows) on a few
heads per GQA group.  Inputs are drawn on the CPU and copied to the GPU.
"""

import math

import numpy as np
import pytest
import torch

import long_context_attention_dca_b200 as dca
from long_context_attention_dca_b200 import workloads as W
from oracle import dca_oracle as orc
from tests import parity_util as pu
from tests.test_oracle_pins import TABLES, parse_table

pytestmark = pytest.mark.gpu

PATHS = [dca.DCA_PATH_GENERAL, dca.DCA_PATH_TCGEN05]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from long_context_attention_dca_b200 import build
    build.build()
    dca.lib()
    yield
    dca.dca_sync_status()


def _prefill_gpu(Q, K, V, s, c, path, base=10000.0):
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    ws = dca.dca_prefill_rope(Qd, Kd, s, c, base)
    O, LSE = dca.dca_prefill_attention(Vd, ws, Q.shape[2], s, c, path=path)
    dca.dca_sync_status()
    return O.cpu(), LSE.cpu()


# ---------------------------------------------------------------------------
# index rule
# ---------------------------------------------------------------------------

def test_index_map_bit_exact_small_grid():
    for s, c in [(4, 6), (3, 5), (5, 8), (8, 8), (2, 5), (1, 1), (7, 9)]:
        for L in range(1, 41):
            qpos, kpos, piece = dca.dca_debug_index_map(L, s, c)
            rq, rk, rp = orc.index_map(L, s, c)
            assert (qpos.cpu().numpy() == rq).all(), (s, c, L)
            assert (kpos.cpu().numpy() == rk).all(), (s, c, L)
            assert (piece.cpu().numpy() == rp).all(), (s, c, L)


def test_index_map_matches_hand_tables():
    for name, s, c in TABLES:
        want_pc, want_d = parse_table(name)
        L = want_pc.shape[0]
        qpos, kpos, piece = (x.cpu().numpy() for x in dca.dca_debug_index_map(L, s, c))
        assert (piece == want_pc).all(), name
        assert (np.where(piece >= 0, qpos - kpos, -1) == want_d).all(), name


def test_index_map_tiny_workload():
    cfg = W.CONFIGS["tiny"]
    qpos, kpos, piece = (x.cpu().numpy() for x in dca.dca_debug_index_map(cfg["L"], cfg["s"],
                                                                          cfg["c"]))
    rq, rk, rp = orc.index_map(cfg["L"], cfg["s"], cfg["c"])
    assert (qpos == rq).all() and (kpos == rk).all() and (piece == rp).all()


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("rule", range(5))
def test_rope_rotate_all_rules(D, rule):
    gen = torch.Generator().manual_seed(1)
    x = torch.randn(2, 333, 3, D, generator=gen).to(torch.bfloat16)
    s, c, off = 100, 160, 17
    got = dca.dca_rope_rotate(x.cuda(), rule, s, c, 10000.0, pos_offset=off).cpu()
    ref = orc.rope_rotate(x.float().numpy(), rule, s, c, 10000.0, pos_offset=off)
    err = np.abs(got.double().numpy() - ref)
    # fp32 rotation then one bf16 rounding: within 2^-8 relative (+ fp32 slack)
    assert (err <= np.abs(ref) * 2.0 ** -8 + 1e-5).all(), err.max()


def test_prefill_rope_workspace_planes():
    cfg = W.scaled(W.CONFIGS["llama2_70b_32k"], L=4000, Hq=16, Hkv=2)
    Q, K, V = W.make_prefill_inputs(cfg)
    s, c = cfg["s"], cfg["c"]
    ws = dca.dca_prefill_rope(Q.cuda(), K.cuda(), s, c).cpu()
    B, L, Hq, D = Q.shape
    n_q = 3 * B * L * Hq * D
    # the workspace planes are fp16 (operands of S = Q K^T): one fp16 rounding
    qr = ws[: n_q * 2].view(torch.float16).view(3, B, L, Hq, D)
    q_off = (n_q * 2 + 255) // 256 * 256
    kr = ws[q_off: q_off + B * L * 2 * D * 2].view(torch.float16).view(B, L, 2, D)
    tol = lambda ref: np.abs(ref) * 2.0 ** -11 + 1e-6
    for v, rule in enumerate((orc.POS_Q_INTRA, orc.POS_Q_SUCC, orc.POS_Q_INTER)):
        ref = orc.rope_rotate(Q.float().numpy(), rule, s, c, 10000.0)
        assert (np.abs(qr[v].double().numpy() - ref) <= tol(ref)).all()
    ref = orc.rope_rotate(K.float().numpy(), orc.POS_KEY, s, c, 10000.0)
    assert (np.abs(kr.double().numpy() - ref) <= tol(ref)).all()


# ---------------------------------------------------------------------------
# prefill, small cases, every output
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", PATHS)
def test_prefill_tiny_workload_full(path):
    cfg = W.CONFIGS["tiny"]
    Q, K, V = W.make_prefill_inputs(cfg)
    O, LSE = _prefill_gpu(Q, K, V, cfg["s"], cfg["c"], path)
    O_ref, LSE_ref = orc.dca_prefill(Q.float().numpy(), K.float().numpy(), V.float().numpy(),
                                     cfg["s"], cfg["c"], cfg["base"])
    err = np.abs(O.double().numpy() - O_ref)
    lse_rel = np.abs(LSE.double().numpy() - LSE_ref) / np.maximum(np.abs(LSE_ref), 1.0)
    print(f"tiny path {path}: O max {err.max():.3e} mean {err.mean():.3e} "
          f"LSE rel {lse_rel.max():.3e}")
    pu.assert_close(err.max(), err.mean(), lse_rel.max(), "tiny")


SMALL = [  # (B, L, Hq, Hkv, D, s, c)
    (1, 1, 1, 1, 128, 128, 256),
    (1, 2, 2, 1, 64, 1, 1),
    (2, 300, 4, 2, 128, 64, 96),
    (1, 777, 2, 1, 64, 100, 150),
    (1, 513, 4, 4, 128, 128, 256),
    (1, 700, 8, 1, 128, 128, 128),     # w = 0: successive piece always at c-1
    (1, 900, 2, 2, 128, 256, 384),
    (1, 640, 2, 1, 128, 128, 1000),    # w > s
    (1, 129, 3, 3, 64, 16, 20),
    # s % 256 == 0: the two-tile (ping-pong) tensor-core kernel
    (1, 1, 1, 1, 128, 256, 256),
    (2, 1000, 4, 2, 128, 256, 256),    # w = 0
    (1, 1500, 2, 1, 128, 512, 768),
    (1, 1300, 2, 2, 128, 256, 4096),   # w > s
    (1, 129, 2, 2, 128, 256, 300),
    (1, 2200, 4, 1, 128, 512, 640),
    (1, 2600, 4, 2, 128, 512, 768),    # pairs at i mod s = 256 >= w: inter + successive in one walk
    # D = 128, s not a multiple of 128: tiles straddle chunk boundaries
    (1, 1000, 2, 1, 128, 192, 256),
    (2, 777, 4, 2, 128, 100, 150),
    (1, 600, 2, 2, 128, 3, 5),         # many chunks per tile
    (1, 1500, 4, 4, 128, 300, 400),
    (1, 900, 2, 1, 128, 160, 1000),    # w > s
    (1, 1100, 2, 1, 128, 1000, 1000),  # w = 0
]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("case", SMALL, ids=[str(c) for c in SMALL])
def test_prefill_small_full(case, path):
    B, L, Hq, Hkv, D, s, c = case
    cfg = dict(B=B, L=L, Hq=Hq, Hkv=Hkv, D=D)
    Q, K, V = W.make_prefill_inputs(cfg, seed=L)
    O, LSE = _prefill_gpu(Q, K, V, s, c, path)
    O_ref, LSE_ref = orc.dca_prefill(Q.float().numpy(), K.float().numpy(), V.float().numpy(),
                                     s, c)
    err = np.abs(O.double().numpy() - O_ref)
    lse_rel = np.abs(LSE.double().numpy() - LSE_ref) / np.maximum(np.abs(LSE_ref), 1.0)
    print(f"{case} path {path}: O max {err.max():.3e} mean {err.mean():.3e} "
          f"LSE rel {lse_rel.max():.3e}")
    pu.assert_close(err.max(), err.mean(), lse_rel.max(), str(case))


def test_prefill_closed_forms_on_gpu():
    # Q = 0: LSE_i = ln(i + 1), O_i = mean of V[0..i]; constant V: O = v
    L, s, c = 300, 64, 96
    gen = torch.Generator().manual_seed(3)
    K = torch.randn(1, L, 2, 128, generator=gen).to(torch.bfloat16)
    V = torch.randn(1, L, 2, 128, generator=gen).to(torch.bfloat16)
    Q = torch.zeros(1, L, 4, 128, dtype=torch.bfloat16)
    O, LSE = _prefill_gpu(Q, K, V, s, c, dca.DCA_PATH_GENERAL)
    ln = np.log(np.arange(1, L + 1))
    assert np.abs(LSE[0].double().numpy() - ln[None]).max() < 1e-4
    mean = np.cumsum(V[0].double().numpy(), axis=0) / np.arange(1, L + 1)[:, None, None]
    assert np.abs(O[0].double().numpy() - np.repeat(mean, 2, axis=1)).max() < 1e-2
    v = torch.randn(128, generator=gen).to(torch.bfloat16)
    Vc = v.expand(1, L, 2, 128).contiguous()
    Q = torch.randn(1, L, 4, 128, generator=gen).to(torch.bfloat16)
    O, _ = _prefill_gpu(Q, K, Vc, s, c, dca.DCA_PATH_GENERAL)
    assert (O[0].double() - v.double()).abs().max() < 1e-2


# ---------------------------------------------------------------------------
# prefill, full-size workloads, sampled rows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name", ["llama2_7b_16k", "llama2_70b_32k", "prefill_100k"])
def test_prefill_workload_sampled(name, path):
    cfg = W.CONFIGS[name]
    Q, K, V = W.make_prefill_inputs(cfg)
    O, LSE = _prefill_gpu(Q, K, V, cfg["s"], cfg["c"], path)
    rows = pu.sample_rows(cfg["L"], cfg["s"], cfg["c"])
    heads = pu.sample_heads(cfg["Hq"], cfg["Hkv"])
    ref = orc.dca_prefill_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V), cfg["s"], cfg["c"],
                               cfg["base"], rows=rows, heads=heads)
    mx, mean, lse = pu.compare_rows(O, LSE, ref)
    print(f"{name} path {path}: {len(rows)} rows x {len(heads)} heads: O max {mx:.3e} "
          f"mean {mean:.3e} LSE rel {lse:.3e}")
    pu.assert_close(mx, mean, lse, name)
    assert torch.isfinite(O.float()).all() and torch.isfinite(LSE).all()


def test_tcgen05_matches_general_path():
    cfg = W.scaled(W.CONFIGS["llama2_70b_32k"], L=8192 + 96, Hq=16, Hkv=2)
    if dca.dca_prefill_path(cfg["L"], 128, cfg["s"], cfg["c"]) != dca.DCA_PATH_TCGEN05:
        pytest.skip("tcgen05 path not built")
    Q, K, V = W.make_prefill_inputs(cfg)
    O1, L1 = _prefill_gpu(Q, K, V, cfg["s"], cfg["c"], dca.DCA_PATH_GENERAL)
    O2, L2 = _prefill_gpu(Q, K, V, cfg["s"], cfg["c"], dca.DCA_PATH_TCGEN05)
    d = (O1.float() - O2.float()).abs()
    print(f"tcgen05 vs general: O max {d.max():.3e} mean {d.mean():.3e} "
          f"LSE max {(L1 - L2).abs().max():.3e}")
    assert d.max() < 2e-2 and d.mean() < 1e-3
    assert (L1 - L2).abs().max() < 1e-3


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

def _decode_gpu(t, q, Kc, Vc, s, c):
    O, LSE = dca.dca_attn_decode(q.cuda(), Kc.cuda(), Vc.cuda(), t.cuda(), s, c)
    dca.dca_sync_status()
    return O.cpu(), LSE.cpu()


def _decode_compare(O, LSE, t, q, Kc, Vc, s, c, batches=None, heads=None):
    O_ref, LSE_ref = orc.dca_decode(pu.F64View(q), pu.F64View(Kc), pu.F64View(Vc),
                                    t.numpy(), s, c, batches=batches, heads=heads)
    B, Hq = q.shape[:2]
    bs = range(B) if batches is None else batches
    hs = range(Hq) if heads is None else heads
    sel = np.ix_(list(bs), list(hs))
    err = np.abs(O.double().numpy()[sel] - O_ref[sel])
    lse_rel = np.abs(LSE.double().numpy()[sel] - LSE_ref[sel]) / np.maximum(
        np.abs(LSE_ref[sel]), 1.0)
    return err.max(), err.mean(), lse_rel.max()


DEC_SMALL = [  # (B, Hq, Hkv, D, Tcap, s, c, t values)
    (3, 8, 1, 128, 3000, 96, 128, [0, 1500, 2999]),
    (2, 4, 2, 64, 2100, 100, 150, [1023, 2047]),
    (2, 16, 1, 128, 5000, 3072, 4096, [4999, 3072]),   # two groups of 8 heads
    (2, 6, 2, 128, 4096, 512, 512, [1024, 4000]),      # G = 3 (padded), w = 0
]


@pytest.mark.parametrize("case", DEC_SMALL, ids=[str(c[:7]) for c in DEC_SMALL])
def test_decode_small_full(case):
    B, Hq, Hkv, D, T, s, c, tv = case
    cfg = dict(B=B, Hq=Hq, Hkv=Hkv, D=D, Tcap=T, t_lo=0, t_hi=T)
    t, q, Kc, Vc = W.make_decode_inputs(cfg, seed=T)
    t = torch.tensor(tv, dtype=torch.int32)
    O, LSE = _decode_gpu(t, q, Kc, Vc, s, c)
    mx, mean, lse = _decode_compare(O, LSE, t, q, Kc, Vc, s, c)
    print(f"decode {case[:7]}: O max {mx:.3e} mean {mean:.3e} LSE rel {lse:.3e}")
    pu.assert_close(mx, mean, lse, str(case))


def test_decode_workload():
    cfg = W.CONFIGS["decode_b16"]
    t, q, Kc, Vc = W.make_decode_inputs(cfg)
    O, LSE = _decode_gpu(t, q, Kc, Vc, cfg["s"], cfg["c"])
    heads = pu.sample_heads(cfg["Hq"], cfg["Hkv"]) + [21, 42]
    mx, mean, lse = _decode_compare(O, LSE, t, q, Kc, Vc, cfg["s"], cfg["c"], heads=heads)
    print(f"decode_b16 ({len(heads)} heads x 16 seqs): O max {mx:.3e} mean {mean:.3e} "
          f"LSE rel {lse:.3e}")
    pu.assert_close(mx, mean, lse, "decode_b16")
    assert torch.isfinite(O.float()).all()


def test_decode_long_splits_with_short_sequences():
    # 8 sequences x 8 head groups x 19 splits = 1216 CTAs: the launch takes
    # 2048-key splits; positions on both sides of split and tile edges, the
    # first key alone and the last cache row
    cfg = dict(B=8, Hq=64, Hkv=8, D=128, Tcap=19 * 2048, t_lo=0, t_hi=1)
    _, q, Kc, Vc = W.make_decode_inputs(cfg, seed=9)
    t = torch.tensor([0, 1, 63, 2047, 2048, 2049, 20000, 19 * 2048 - 1], dtype=torch.int32)
    s, c = 3072, 4096
    O, LSE = _decode_gpu(t, q, Kc, Vc, s, c)
    heads = pu.sample_heads(cfg["Hq"], cfg["Hkv"])
    mx, mean, lse = _decode_compare(O, LSE, t, q, Kc, Vc, s, c, heads=heads)
    print(f"decode, 2048-key splits: O max {mx:.3e} mean {mean:.3e} LSE rel {lse:.3e}")
    pu.assert_close(mx, mean, lse, "decode 2048-key splits")
    # t = 0: every head returns its kv head's only value
    assert (O[0].float() - Vc[0, 0].float().repeat_interleave(8, dim=0)).abs().max() <= 2e-2


def test_decode_independent_of_split_size():
    # the same four sequences decoded alone (4 x 8 x 19 = 608 CTAs: 1024-key
    # splits) and inside a batch of eight (1216 CTAs: 2048-key splits) agree
    # to fp32 reordering: the LSE merge of partial softmaxes is exact
    cfg = dict(B=8, Hq=64, Hkv=8, D=128, Tcap=19 * 2048, t_lo=30000, t_hi=19 * 2048)
    t, q, Kc, Vc = W.make_decode_inputs(cfg, seed=10)
    s, c = 3072, 4096
    O8, L8 = _decode_gpu(t, q, Kc, Vc, s, c)
    O4, L4 = _decode_gpu(t[:4].contiguous(), q[:4].contiguous(), Kc[:4].contiguous(),
                         Vc[:4].contiguous(), s, c)
    assert (L8[:4] - L4).abs().max() <= 5e-5
    # bf16 outputs: at most one rounding step apart
    assert (O8[:4].float() - O4.float()).abs().max() <= 8e-3


def test_decode_equals_prefill_row_on_gpu():
    # Same K/V: the decode of token t (cache rotated by the library's RoPE at
    # j mod s) must equal row t of prefill, and both must match the oracle.
    L, Hq, Hkv, D, s, c = 2600, 8, 2, 128, 512, 768
    cfg = dict(B=1, L=L, Hq=Hq, Hkv=Hkv, D=D)
    Q, K, V = W.make_prefill_inputs(cfg, seed=5)
    O_p, LSE_p = _prefill_gpu(Q, K, V, s, c, dca.DCA_PATH_GENERAL)
    Kc = dca.dca_rope_rotate(K.cuda(), dca.DCA_POS_KEY, s, c)
    for tt in (0, 511, 512, 1279, 1280, 2599):
        t = torch.tensor([tt], dtype=torch.int32)
        O_d, LSE_d = dca.dca_attn_decode(Q[:, tt].contiguous().cuda(), Kc, V.cuda(), t.cuda(),
                                         s, c)
        dca.dca_sync_status()
        assert (O_d.cpu().float() - O_p[:, tt].float()).abs().max() < 2e-2
        assert (LSE_d.cpu() - LSE_p[:, :, tt]).abs().max() < 2e-3
        ref = orc.dca_prefill_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V), s, c,
                                   rows=[tt])
        for h in range(Hq):
            assert np.abs(O_d[0, h].cpu().double().numpy() - ref[(0, h, tt)][0]).max() < 2e-2


def test_decode_rejects_position_outside_cache():
    B, Hq, Hkv, D, T = 2, 8, 1, 128, 1000
    t = torch.tensor([5, T], dtype=torch.int32).cuda()   # second one is out of range
    q = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device="cuda")
    Kc = torch.zeros(B, T, Hkv, D, dtype=torch.bfloat16, device="cuda")
    O, LSE = dca.dca_attn_decode(q, Kc, Kc, t, 256, 384)
    with pytest.raises(dca.DcaError) as ei:
        dca.dca_sync_status()
    assert ei.value.status == 1
    assert torch.isnan(LSE[1]).all() and torch.isfinite(LSE[0]).all()
    dca.dca_sync_status()  # the error word was cleared


def test_empty_and_degenerate_sizes():
    x = torch.empty(0, 5, 2, 128, dtype=torch.bfloat16, device="cuda")
    assert dca.dca_rope_rotate(x, dca.DCA_POS_KEY, 4, 6).numel() == 0
    Q = torch.empty(1, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    O, LSE = dca.dca_attn_prefill(Q, Q[:, :, :1], Q[:, :, :1], 3072, 4096)
    assert O.numel() == 0 and LSE.numel() == 0
    dca.dca_sync_status()


# ---------------------------------------------------------------------------
# fp16 range of the rotated score operands
# ---------------------------------------------------------------------------
def _expect_fp16_range_error():
    with pytest.raises(dca.DcaError) as ei:
        dca.dca_sync_status()
    assert ei.value.status == 1 and "fp16" in str(ei.value)
    dca.dca_sync_status()  # the error word was cleared


@pytest.mark.parametrize("where", ["q", "k"])
def test_prefill_reports_rotated_value_beyond_fp16(where):
    # one input element of 1e5 rotates (at the intra position 123 mod 192 and
    # at the others) into a value fp16 cannot hold: reported as a bad
    # argument, and the context keeps working for the next call
    cfg = W.scaled(W.CONFIGS["tiny"], L=300, Hq=2, Hkv=1)
    s, c = cfg["s"], cfg["c"]
    Q, K, V = W.make_prefill_inputs(cfg, seed=9)
    X = Q if where == "q" else K
    X[0, 123, 0, 5] = 1e5
    dca.dca_attn_prefill(Q.cuda(), K.cuda(), V.cuda(), s, c)
    _expect_fp16_range_error()
    X[0, 123, 0, 5] = 0.5
    O, LSE = dca.dca_attn_prefill(Q.cuda(), K.cuda(), V.cuda(), s, c)
    dca.dca_sync_status()
    rows = [0, 123, 191, 192, 299]
    ref = orc.dca_prefill_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V), s, c, rows=rows)
    pu.assert_close(*pu.compare_rows(O.cpu(), LSE.cpu(), ref), what=f"after {where} overflow")


def test_prefill_accepts_pairs_inside_fp16_range():
    # a pair of norm below 65504 stays finite under every rotation: no report
    cfg = W.scaled(W.CONFIGS["tiny"], L=300, Hq=2, Hkv=1)
    Q, K, V = W.make_prefill_inputs(cfg, seed=10)
    Q[0, 200, 1, 3] = 60000.0
    K[0, 17, 0, 40] = -60000.0
    dca.dca_attn_prefill(Q.cuda(), K.cuda(), V.cuda(), cfg["s"], cfg["c"])
    dca.dca_sync_status()


def test_selfextend_reports_rotated_value_beyond_fp16():
    cfg = W.scaled(W.CONFIGS["tiny"], L=200, Hq=2, Hkv=1)
    Q, K, V = W.make_prefill_inputs(cfg, seed=11)
    K[0, 150, 0, 0] = -1e5
    dca.dca_attn_prefill_selfextend(Q.cuda(), K.cuda(), V.cuda(), 4, 32)
    _expect_fp16_range_error()


def test_chunk_reports_cached_key_beyond_fp16():
    # a cached bf16 key of 1e5 cannot be converted to the fp16 score operand
    B, Lq, Hq, Hkv, D, t0, s, c = 1, 64, 2, 1, 64, 256, 192, 256
    g = torch.Generator().manual_seed(12)
    mk = lambda *sh: torch.randn(*sh, generator=g).to(torch.bfloat16)
    Q, K, V = mk(B, Lq, Hq, D), mk(B, Lq, Hkv, D), mk(B, Lq, Hkv, D)
    Kc, Vc = mk(B, 512, Hkv, D), mk(B, 512, Hkv, D)
    Kc[0, 100, 0, 7] = 1e5
    dca.dca_attn_prefill_chunk(Q.cuda(), K.cuda(), V.cuda(), Kc.cuda(), Vc.cuda(), t0, s, c)
    _expect_fp16_range_error()
