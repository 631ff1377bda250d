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
