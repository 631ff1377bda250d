"""GPU parity for the packed variable-length prefill (dca_attn_prefill_varlen).

Sequences of different lengths sit back to back in one [T, H, D] tensor; each
is its own DCA prefill.  Checked against the oracle's packed-batch function
on every row (small cases, both tcgen05 kernels, D = 64 and 128, straddling
chunks, empty and one-row sequences, rows before and after the sequences), bit
for bit against one dca_attn_prefill call per sequence (the same kernels on
the same numbers), on sampled rows of a Llama-2 7B-shaped mix of prompt
lengths, and for offsets the kernels must refuse.
"""

import numpy as np
import pytest
import torch

import long_context_attention_dca_b200 as dca
from long_context_attention_dca_b200 import workloads as W
from oracle import dca_oracle as orc
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

O_FILL, LSE_FILL = 3.0, -7.0


@pytest.fixture(scope="module", autouse=True)
def _built():
    from long_context_attention_dca_b200 import build
    build.build()
    dca.lib()
    yield
    dca.dca_sync_status()


def _packed(lens, lead, tail, Hq, Hkv, D, seed):
    """Packed inputs with `lead` rows before the first sequence and `tail`
    rows after the last one (rows of no sequence)."""
    cfg = dict(Hq=Hq, Hkv=Hkv, D=D)
    Q, K, V, cu, _ = W.make_varlen_inputs(cfg, seed=seed, lens=[lead] + list(lens) + [tail])
    return Q, K, V, cu[1:-1].contiguous()


def _run(Q, K, V, cu, s, c):
    T, Hq, _ = Q.shape
    O = torch.full(Q.shape, O_FILL, dtype=torch.bfloat16, device="cuda")
    LSE = torch.full((Hq, T), LSE_FILL, dtype=torch.float32, device="cuda")
    max_len = int((cu[1:] - cu[:-1]).max())
    dca.dca_attn_prefill_varlen(Q.cuda(), K.cuda(), V.cuda(), cu.cuda(), max_len, s, c,
                                O=O, LSE=LSE)
    dca.dca_sync_status()
    return O.cpu(), LSE.cpu()


def _compare(O, LSE, ref, what):
    keys = sorted(ref)
    o_ref = np.stack([ref[k][0] for k in keys])
    l_ref = np.array([ref[k][1] for k in keys])
    o_got = np.stack([O[t, h].double().numpy() for h, t in keys])
    l_got = np.array([float(LSE[h, t]) for h, t in keys])
    err = np.abs(o_got - o_ref)
    lse_rel = float(np.max(np.abs(l_got - l_ref) / np.maximum(np.abs(l_ref), 1.0)))
    print(f"{what}: O max {err.max():.3e} mean {err.mean():.3e} LSE rel {lse_rel:.3e}")
    pu.assert_close(float(err.max()), float(err.mean()), lse_rel, what)


VARLEN_CASES = [
    # lens, lead rows, tail rows, Hq, Hkv, D, s, c
    ([300, 1, 700, 0, 513], 0, 0, 4, 2, 128, 256, 400),    # two-tile kernel
    ([300, 1, 700, 0, 513], 5, 7, 4, 2, 128, 100, 150),    # interval kernel, straddling
    ([129, 1000, 64, 257], 3, 0, 2, 1, 64, 192, 256),      # D = 64
    ([2000, 37], 0, 9, 8, 1, 128, 512, 640),               # GQA 8, long + short
]


@pytest.mark.parametrize("case", VARLEN_CASES, ids=str)
def test_varlen_matches_oracle(case):
    lens, lead, tail, Hq, Hkv, D, s, c = case
    Q, K, V, cu = _packed(lens, lead, tail, Hq, Hkv, D, seed=51)
    O, LSE = _run(Q, K, V, cu, s, c)
    ref = orc.dca_prefill_varlen_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V),
                                      cu.tolist(), s, c)
    assert len(ref) == Hq * sum(lens)
    _compare(O, LSE, ref, f"varlen {case}")
    # rows that belong to no sequence are left as they were
    outside = list(range(0, int(cu[0]))) + list(range(int(cu[-1]), Q.shape[0]))
    assert (O[outside].float() == O_FILL).all() and (LSE[:, outside] == LSE_FILL).all()


@pytest.mark.parametrize("case", VARLEN_CASES, ids=str)
def test_varlen_equals_one_call_per_sequence(case):
    lens, lead, tail, Hq, Hkv, D, s, c = case
    Q, K, V, cu = _packed(lens, lead, tail, Hq, Hkv, D, seed=52)
    O, LSE = _run(Q, K, V, cu, s, c)
    for b, n in enumerate(lens):
        if n == 0:
            continue
        a = int(cu[b])
        Ob, Lb = dca.dca_attn_prefill(Q[None, a:a + n].cuda(), K[None, a:a + n].cuda(),
                                      V[None, a:a + n].cuda(), s, c)
        dca.dca_sync_status()
        assert torch.equal(O[a:a + n], Ob[0].cpu()), (case, b)
        assert torch.equal(LSE[:, a:a + n], Lb[0].cpu()), (case, b)


def test_varlen_workload_sampled():
    cfg = W.CONFIGS["varlen_7b_mix"]
    s, c = cfg["s"], cfg["c"]
    Q, K, V, cu, lens = W.make_varlen_inputs(cfg)
    O, LSE = _run(Q, K, V, cu, s, c)
    assert torch.isfinite(O.float()).all() and torch.isfinite(LSE).all()
    heads = pu.sample_heads(cfg["Hq"], cfg["Hkv"])
    longest = int(np.argmax(lens))
    for b in sorted({0, longest, len(lens) - 1}):
        a, n = int(cu[b]), lens[b]
        rows = [a + r for r in pu.sample_rows(n, s, c, n_random=24, seed=b)]
        ref = orc.dca_prefill_varlen_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V),
                                          cu.tolist(), s, c, rows=rows, heads=heads)
        _compare(O, LSE, ref, f"varlen_7b_mix sequence {b} (n={n})")
    # the longest prompt alone through the one-sequence API: the same bits
    a, n = int(cu[longest]), lens[longest]
    Ob, Lb = dca.dca_attn_prefill(Q[None, a:a + n].cuda(), K[None, a:a + n].cuda(),
                                  V[None, a:a + n].cuda(), s, c)
    dca.dca_sync_status()
    assert torch.equal(O[a:a + n], Ob[0].cpu()) and torch.equal(LSE[:, a:a + n], Lb[0].cpu())


@pytest.mark.parametrize("bad", ["longer_than_max", "decreasing", "past_T"])
def test_varlen_bad_offsets_are_reported(bad):
    Hq, Hkv, D, s, c = 2, 1, 128, 256, 384
    T = 600
    Q = torch.zeros(T, Hq, D, dtype=torch.bfloat16, device="cuda")
    K, V = torch.zeros(T, Hkv, D, dtype=torch.bfloat16, device="cuda"), \
        torch.ones(T, Hkv, D, dtype=torch.bfloat16, device="cuda")
    # sequence 0 (rows 0 .. 99) is valid in every case; sequence 1 is not
    cu, max_len = {"longer_than_max": ([0, 100, 400], 200),
                   "decreasing": ([0, 100, 50], 100),
                   "past_T": ([0, 100, 700], 600)}[bad]
    O = torch.full(Q.shape, O_FILL, dtype=torch.bfloat16, device="cuda")
    LSE = torch.full((Hq, T), LSE_FILL, dtype=torch.float32, device="cuda")
    dca.dca_attn_prefill_varlen(Q, K, V, torch.tensor(cu, dtype=torch.int32, device="cuda"),
                                max_len, s, c, O=O, LSE=LSE)
    with pytest.raises(dca.DcaError) as ei:
        dca.dca_sync_status()
    assert ei.value.status == 1
    # the valid first sequence was computed (Q = 0, V = 1: O = 1, LSE = ln(r+1)),
    # the refused one was not written
    O, LSE = O.cpu(), LSE.cpu()
    assert (O[:100].float() == 1.0).all()
    np.testing.assert_allclose(LSE[:, :100].numpy(),
                               np.log(np.arange(1, 101))[None, :].repeat(Hq, 0), atol=1e-5)
    assert (O[100:].float() == O_FILL).all() and (LSE[:, 100:] == LSE_FILL).all()
    dca.dca_sync_status()  # cleared; the context keeps working


# ---------------------------------------------------------------------------
# packed chunks over per-sequence caches (dca_attn_prefill_varlen_chunk)
# ---------------------------------------------------------------------------

def _chunk_inputs(lens, t0, Hq, Hkv, D, Tcap, seed):
    """Packed new tokens and caches whose rows 0 .. t0[b]-1 hold random bf16
    keys (standing for keys already rotated at j mod s: a rotation of i.i.d.
    N(0, 1) pairs is again i.i.d. N(0, 1)) and values; every later cache row
    holds NaN, so a row read or written by mistake shows."""
    gen = torch.Generator().manual_seed(seed)
    T, B = sum(lens), len(lens)
    Q = torch.randn(T, Hq, D, generator=gen).to(torch.bfloat16)
    K = torch.randn(T, Hkv, D, generator=gen).to(torch.bfloat16)
    V = torch.randn(T, Hkv, D, generator=gen).to(torch.bfloat16)
    Kc = torch.full((B, Tcap, Hkv, D), float("nan"), dtype=torch.bfloat16)
    Vc = torch.full((B, Tcap, Hkv, D), float("nan"), dtype=torch.bfloat16)
    for b in range(B):
        Kc[b, :t0[b]] = torch.randn(t0[b], Hkv, D, generator=gen).to(torch.bfloat16)
        Vc[b, :t0[b]] = torch.randn(t0[b], Hkv, D, generator=gen).to(torch.bfloat16)
    cu = torch.zeros(B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens), 0).to(torch.int32)
    return Q, K, V, Kc, Vc, cu


def _run_chunk(Q, K, V, Kc, Vc, cu, t0, s, c, max_kv):
    T, Hq, _ = Q.shape
    O = torch.full(Q.shape, O_FILL, dtype=torch.bfloat16, device="cuda")
    LSE = torch.full((Hq, T), LSE_FILL, dtype=torch.float32, device="cuda")
    Kd, Vd = Kc.cuda(), Vc.cuda()
    max_len = max(1, int((cu[1:] - cu[:-1]).max()))
    dca.dca_attn_prefill_varlen_chunk(Q.cuda(), K.cuda(), V.cuda(), Kd, Vd, cu.cuda(),
                                      torch.tensor(t0, dtype=torch.int32, device="cuda"),
                                      max_len, max_kv, s, c, O=O, LSE=LSE)
    return O, LSE, Kd, Vd


VARLEN_CHUNK_CASES = [
    # lens, t0, Hq, Hkv, D, s, c, Tcap
    ([300, 1, 700, 0, 513], [0, 256, 77, 5, 1000], 4, 2, 128, 256, 400, 1600),
    ([129, 400, 64], [511, 3, 0], 2, 1, 64, 192, 256, 700),
    ([2000, 37], [300, 4000], 8, 1, 128, 512, 640, 4100),
    ([90, 260], [1, 129], 2, 2, 128, 100, 150, 420),
]


@pytest.mark.parametrize("case", VARLEN_CHUNK_CASES, ids=str)
def test_varlen_chunk_matches_oracle(case):
    lens, t0, Hq, Hkv, D, s, c, Tcap = case
    Q, K, V, Kc, Vc, cu = _chunk_inputs(lens, t0, Hq, Hkv, D, Tcap, seed=61)
    max_kv = max(a + n for a, n in zip(t0, lens))
    O, LSE, Kd, Vd = _run_chunk(Q, K, V, Kc, Vc, cu, t0, s, c, max_kv)
    dca.dca_sync_status()
    O, LSE, Kg, Vg = O.cpu(), LSE.cpu(), Kd.cpu(), Vd.cpu()
    assert torch.isfinite(O.float()).all() and torch.isfinite(LSE).all()
    ref = orc.dca_prefill_varlen_chunk_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V),
                                            cu.tolist(), t0, pu.F64View(Kc), pu.F64View(Vc),
                                            s, c)
    assert len(ref) == Hq * sum(lens)
    _compare(O, LSE, ref, f"varlen chunk {case}")
    for b, (a, n) in enumerate(zip(t0, lens)):
        r0 = int(cu[b])
        # cached rows unchanged, new rows written, the tail zeroed, the rest as it was
        assert torch.equal(Kg[b, :a], Kc[b, :a]) and torch.equal(Vg[b, :a], Vc[b, :a])
        assert torch.equal(Vg[b, a:a + n], V[r0:r0 + n])
        ref_k = orc.rotate(K[r0:r0 + n].double().numpy().transpose(1, 0, 2),
                           orc.key_position(a + np.arange(n), s), 10000.0).transpose(1, 0, 2)
        err = np.abs(Kg[b, a:a + n].double().numpy() - ref_k)
        assert (err <= np.abs(ref_k) * 2.0 ** -8 + 1e-5).all(), (case, b)
        tail = min((a + n + 127) // 128 * 128, max_kv)
        assert (Vg[b, a + n:tail].float() == 0).all()
        assert torch.isnan(Vg[b, max(tail, a + n):].float()).all()
        assert torch.isnan(Kg[b, a + n:].float()).all()


def test_varlen_chunk_continues_a_packed_prefill():
    # two calls (first chunks at t0 = 0, then the rest) give what one packed
    # prefill of the whole sequences gives, up to the bf16 rounding of the
    # cached keys (the second call reads them as stored)
    Hq, Hkv, D, s, c = 4, 2, 128, 256, 384
    first, rest = [300, 513, 64], [400, 1, 700]
    full = [a + b for a, b in zip(first, rest)]
    cfg = dict(Hq=Hq, Hkv=Hkv, D=D)
    Q, K, V, cu_full, _ = W.make_varlen_inputs(cfg, seed=62, lens=full)
    Tcap = max(full) + 100
    pick = lambda X, lo, hi: torch.cat([X[int(cu_full[b]) + lo[b]:int(cu_full[b]) + hi[b]]
                                        for b in range(3)])
    zeros = [0, 0, 0]
    Kd = torch.zeros(3, Tcap, Hkv, D, dtype=torch.bfloat16, device="cuda")
    Vd = torch.zeros_like(Kd)
    outs = []
    for lo, hi in ((zeros, first), (first, full)):
        n = [h - l for l, h in zip(lo, hi)]
        cu = torch.zeros(4, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(n), 0).to(torch.int32)
        O, LSE = dca.dca_attn_prefill_varlen_chunk(
            pick(Q, lo, hi).cuda(), pick(K, lo, hi).cuda(), pick(V, lo, hi).cuda(), Kd, Vd,
            cu.cuda(), torch.tensor(lo, dtype=torch.int32, device="cuda"), max(n), Tcap, s, c)
        outs.append((O.cpu(), LSE.cpu(), cu))
    dca.dca_sync_status()
    Of, Lf = dca.dca_attn_prefill_varlen(Q.cuda(), K.cuda(), V.cuda(), cu_full.cuda(), max(full),
                                         s, c)
    Of, Lf = Of.cpu(), Lf.cpu()
    for b in range(3):
        a = int(cu_full[b])
        for (O, LSE, cu), lo in zip(outs, (zeros, first)):
            r0, n = int(cu[b]), int(cu[b + 1] - cu[b])
            d_o = (O[r0:r0 + n].float() - Of[a + lo[b]:a + lo[b] + n].float()).abs().max()
            d_l = (LSE[:, r0:r0 + n] - Lf[:, a + lo[b]:a + lo[b] + n]).abs().max()
            assert d_o <= 2e-2 and d_l <= 3e-3, (b, lo, float(d_o), float(d_l))


def test_varlen_chunk_workload_sampled():
    # Llama-2 7B heads: eight sequences with 0 .. 14000 cached tokens and new
    # chunks of 256 .. 2048 tokens, packed
    rng = np.random.default_rng(7)
    B, Hq, Hkv, D, s, c = 8, 32, 32, 128, 3072, 4096
    t0 = [int(x) for x in rng.integers(0, 14001, B)]
    lens = [int(x) for x in rng.integers(256, 2049, B)]
    Tcap = 16384
    Q, K, V, Kc, Vc, cu = _chunk_inputs(lens, t0, Hq, Hkv, D, Tcap, seed=63)
    max_kv = max(a + n for a, n in zip(t0, lens))
    O, LSE, _, _ = _run_chunk(Q, K, V, Kc, Vc, cu, t0, s, c, max_kv)
    dca.dca_sync_status()
    O, LSE = O.cpu(), LSE.cpu()
    heads = pu.sample_heads(Hq, Hkv)
    for b in (0, 3, 7):
        a = int(cu[b])
        rows = [a + r for r in pu.sample_rows(lens[b], s, c, n_random=16, seed=b)]
        ref = orc.dca_prefill_varlen_chunk_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V),
                                                cu.tolist(), t0, pu.F64View(Kc),
                                                pu.F64View(Vc), s, c, rows=rows, heads=heads)
        _compare(O, LSE, ref, f"varlen chunk 7B sequence {b} (t0={t0[b]}, n={lens[b]})")


@pytest.mark.parametrize("bad", ["past_max_kv", "negative_t0"])
def test_varlen_chunk_bad_offsets_are_reported(bad):
    Hq, Hkv, D, s, c, Tcap = 2, 1, 128, 256, 384, 600
    lens, t0 = [100, 200], {"past_max_kv": [0, 450], "negative_t0": [0, -3]}[bad]
    Q, K, V, Kc, Vc, cu = _chunk_inputs(lens, [max(a, 0) for a in t0], Hq, Hkv, D, Tcap, seed=64)
    O, LSE, Kd, Vd = _run_chunk(Q, K, V, Kc, Vc, cu, t0, s, c, max_kv=600 if bad == "negative_t0"
                                else 500)
    with pytest.raises(dca.DcaError) as ei:
        dca.dca_sync_status()
    assert ei.value.status == 1
    O, LSE, Kg, Vg = O.cpu(), LSE.cpu(), Kd.cpu(), Vd.cpu()
    # sequence 0 computed and cached; sequence 1 neither computed nor cached
    assert torch.isfinite(O[:100].float()).all()
    assert (O[100:].float() == O_FILL).all() and (LSE[:, 100:] == LSE_FILL).all()
    assert torch.equal(Vg[0, :100], V[:100])
    assert torch.equal(Kg[1].view(torch.int16), Kc[1].view(torch.int16))
    assert torch.equal(Vg[1].view(torch.int16), Vc[1].view(torch.int16))
    dca.dca_sync_status()


def _to_pool(cache, block_rows, perm, num_blocks):
    """Scatter a contiguous cache [B][Tcap][H][D] into a pool of num_blocks
    blocks; block j of sequence b goes to pool block perm[b * max_blocks + j]."""
    B, Tcap, H, D = cache.shape
    nb = Tcap // block_rows
    pool = torch.full((num_blocks, block_rows, H, D), float("nan"), dtype=cache.dtype)
    pool[perm] = cache.reshape(B * nb, block_rows, H, D)
    return pool


def _from_pool(pool, perm, B):
    nb = len(perm) // B
    blocks = pool[perm]
    return blocks.reshape(B, nb * pool.shape[1], *pool.shape[2:])


@pytest.mark.parametrize("block_rows", [128, 256])
@pytest.mark.parametrize("case", VARLEN_CHUNK_CASES[:3], ids=str)
def test_varlen_chunk_paged_equals_contiguous(case, block_rows):
    lens, t0, Hq, Hkv, D, s, c, _ = case
    max_kv = max(a + n for a, n in zip(t0, lens))
    Tcap = (max_kv + block_rows - 1) // block_rows * block_rows + block_rows
    Q, K, V, Kc, Vc, cu = _chunk_inputs(lens, t0, Hq, Hkv, D, Tcap, seed=65)
    O1, L1, Kd, Vd = _run_chunk(Q, K, V, Kc, Vc, cu, t0, s, c, max_kv)
    dca.dca_sync_status()
    B, nb = len(lens), Tcap // block_rows
    num_blocks = B * nb + 3
    perm = torch.randperm(num_blocks, generator=torch.Generator().manual_seed(66))[:B * nb]
    Kp, Vp = _to_pool(Kc, block_rows, perm, num_blocks), _to_pool(Vc, block_rows, perm,
                                                                   num_blocks)
    Kpd, Vpd = Kp.cuda(), Vp.cuda()
    table = perm.view(B, nb).to(torch.int32).cuda()
    O2, L2 = dca.dca_attn_prefill_varlen_chunk_paged(
        Q.cuda(), K.cuda(), V.cuda(), Kpd, Vpd, table, cu.cuda(),
        torch.tensor(t0, dtype=torch.int32, device="cuda"), max(lens), max_kv, s, c)
    dca.dca_sync_status()
    # same bits out, same cache rows written; the value tail zeroed to the
    # 128-row tile edge (the contiguous call stops at max_kv, which its value
    # map does not read past); the pool's unused blocks untouched
    assert torch.equal(O1.cpu(), O2.cpu()) and torch.equal(L1.cpu(), L2.cpu())
    Kp2, Vp2 = Kpd.cpu(), Vpd.cpu()
    assert torch.equal(_from_pool(Kp2, perm, B).view(torch.int16), Kd.cpu().view(torch.int16))
    want_v = Vd.cpu().clone()
    for b, (a, n) in enumerate(zip(t0, lens)):
        want_v[b, a + n:min((a + n + 127) // 128 * 128, Tcap)] = 0
    assert torch.equal(_from_pool(Vp2, perm, B).view(torch.int16), want_v.view(torch.int16))
    unused = sorted(set(range(num_blocks)) - set(perm.tolist()))
    assert torch.isnan(Kp2[unused].float()).all() and torch.isnan(Vp2[unused].float()).all()



@pytest.mark.parametrize("case", VARLEN_CHUNK_CASES[:2], ids=str)
def test_varlen_chunk_paged_matches_oracle(case):
    # the paged call against the oracle directly; the oracle reads each
    # sequence's cached rows from the pool as stored, through its table row
    lens, t0, Hq, Hkv, D, s, c, _ = case
    block_rows = 128
    max_kv = max(a + n for a, n in zip(t0, lens))
    Tcap = (max_kv + block_rows - 1) // block_rows * block_rows
    Q, K, V, Kc, Vc, cu = _chunk_inputs(lens, t0, Hq, Hkv, D, Tcap, seed=68)
    B, nb = len(lens), Tcap // block_rows
    num_blocks = B * nb + 2
    perm = torch.randperm(num_blocks, generator=torch.Generator().manual_seed(69))[:B * nb]
    Kp, Vp = _to_pool(Kc, block_rows, perm, num_blocks), _to_pool(Vc, block_rows, perm,
                                                                   num_blocks)
    table = perm.view(B, nb).to(torch.int32)
    O, LSE = dca.dca_attn_prefill_varlen_chunk_paged(
        Q.cuda(), K.cuda(), V.cuda(), Kp.cuda(), Vp.cuda(), table.cuda(), cu.cuda(),
        torch.tensor(t0, dtype=torch.int32, device="cuda"), max(1, max(lens)), max_kv, s, c)
    dca.dca_sync_status()
    Kg = Kp[table.long()].reshape(B, Tcap, Hkv, D)
    Vg = Vp[table.long()].reshape(B, Tcap, Hkv, D)
    ref = orc.dca_prefill_varlen_chunk_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V),
                                            cu.tolist(), t0, pu.F64View(Kg), pu.F64View(Vg),
                                            s, c)
    assert len(ref) == Hq * sum(lens)
    _compare(O.cpu(), LSE.cpu(), ref, f"paged varlen chunk {case}")

def test_varlen_chunk_paged_table_out_of_range_is_reported():
    lens, t0, Hq, Hkv, D, s, c = [100, 200], [300, 0], 2, 1, 128, 256, 384
    block_rows, Tcap = 128, 512
    Q, K, V, Kc, Vc, cu = _chunk_inputs(lens, t0, Hq, Hkv, D, Tcap, seed=67)
    B, nb = 2, Tcap // block_rows
    perm = torch.arange(B * nb)
    Kpd, Vpd = _to_pool(Kc, block_rows, perm, B * nb).cuda(), \
        _to_pool(Vc, block_rows, perm, B * nb).cuda()
    table = perm.view(B, nb).to(torch.int32)
    table[0, 1] = B * nb  # sequence 0's cached rows 128 .. 255: a block past the pool
    dca.dca_attn_prefill_varlen_chunk_paged(
        Q.cuda(), K.cuda(), V.cuda(), Kpd, Vpd, table.cuda(), cu.cuda(),
        torch.tensor(t0, dtype=torch.int32, device="cuda"), max(lens), 400, s, c)
    with pytest.raises(dca.DcaError) as ei:
        dca.dca_sync_status()
    assert ei.value.status == 1
    dca.dca_sync_status()  # cleared; the context keeps working


# ---------------------------------------------------------------------------
# packed chunks with a caller-owned fp16 key mirror (no per-call conversion)
# ---------------------------------------------------------------------------

MIRROR_CASES = [
    # full lengths, chunk boundaries per sequence (cumulative), Hq, Hkv, D, s, c
    ([700, 1300, 257], [[0, 300, 301, 700], [0, 512, 1000, 1300], [0, 0, 256, 257]],
     4, 2, 128, 256, 400),
    ([900, 450], [[0, 100, 777, 900], [0, 449, 450, 450]], 2, 1, 64, 192, 256),
]


@pytest.mark.parametrize("case", MIRROR_CASES, ids=str)
def test_varlen_chunk_mirror_chunks_equal_whole_prefill(case):
    # each sequence is fed in three packed calls from an empty cache; every
    # row must equal the row of a one-shot prefill over the whole sequence
    # (the keys read back from the mirror were rounded once, to fp16, like a
    # one-shot prefill's); caches start as NaN, so a row read before it is
    # written shows
    lens, bounds, Hq, Hkv, D, s, c = case
    B, Tcap = len(lens), max(lens) + 128
    gen = torch.Generator().manual_seed(70)
    Qs = [torch.randn(n, Hq, D, generator=gen).to(torch.bfloat16) for n in lens]
    Ks = [torch.randn(n, Hkv, D, generator=gen).to(torch.bfloat16) for n in lens]
    Vs = [torch.randn(n, Hkv, D, generator=gen).to(torch.bfloat16) for n in lens]
    Kc = torch.full((B, Tcap, Hkv, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    Vc = torch.full_like(Kc, float("nan"))
    Kf = torch.full((B, Tcap, Hkv, D), float("nan"), dtype=torch.float16, device="cuda")
    ref = [orc.dca_prefill_rows(pu.F64View(Qs[b][None]), pu.F64View(Ks[b][None]),
                                pu.F64View(Vs[b][None]), s, c) for b in range(B)]
    for k in range(3):
        t0 = [bounds[b][k] for b in range(B)]
        ends = [bounds[b][k + 1] for b in range(B)]
        n = [e - a for a, e in zip(t0, ends)]
        cu = torch.zeros(B + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(n), 0).to(torch.int32)
        pack = lambda X: torch.cat([X[b][t0[b]:ends[b]] for b in range(B)])
        Q, K, V = pack(Qs), pack(Ks), pack(Vs)
        if Q.shape[0] == 0:
            continue
        max_kv = max(ends)
        O, LSE = dca.dca_attn_prefill_varlen_chunk_mirror(
            Q.cuda(), K.cuda(), V.cuda(), Kc, Vc, Kf, cu.cuda(),
            torch.tensor(t0, dtype=torch.int32, device="cuda"), max(1, max(n)), max_kv, s, c)
        dca.dca_sync_status()
        want = {}
        for b in range(B):
            for r in range(n[b]):
                for h in range(Hq):
                    want[(h, int(cu[b]) + r)] = ref[b][(0, h, t0[b] + r)]
        _compare(O.cpu(), LSE.cpu(), want, f"mirror {case} call {k}")
    # the caches hold every sequence's rows: values as given, keys rotated at
    # j mod s (bf16 in the cache, fp16 in the mirror)
    for b in range(B):
        n = lens[b]
        assert torch.equal(Vc[b, :n].cpu(), Vs[b])
        ref_k = orc.rotate(Ks[b].double().numpy().transpose(1, 0, 2),
                           orc.key_position(np.arange(n), s), 10000.0).transpose(1, 0, 2)
        for cache, ulp in ((Kc, 2.0 ** -8), (Kf, 2.0 ** -11)):
            err = np.abs(cache[b, :n].cpu().double().numpy() - ref_k)
            assert (err <= np.abs(ref_k) * ulp + 1e-5).all(), (case, b)
