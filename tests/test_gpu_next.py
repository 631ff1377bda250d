"""GPU parity for the rows beyond the core path: decode-time KV append.

dca_kv_append rotates each sequence's new key at t mod s and writes key and
value to cache row t.  Checked against the oracle's rotation (within one bf16
rounding), with every other cache row bit-for-bit untouched; and end to end:
a cache built token by token with dca_kv_append, then decoded, reproduces the
prefill rows and the oracle.
"""

import numpy as np
import pytest
import torch

import long_context_attention_dca_b200 as dca
from long_context_attention_dca_b200 import workloads as W
from oracle import dca_oracle as orc
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from long_context_attention_dca_b200 import build
    build.build()
    dca.lib()
    yield
    dca.dca_sync_status()


@pytest.mark.parametrize("D", [64, 128])
def test_kv_append_writes_one_rotated_row(D):
    B, Hkv, T, s, c = 3, 2, 100, 24, 40
    gen = torch.Generator().manual_seed(11)
    Kc = torch.randn(B, T, Hkv, D, generator=gen).to(torch.bfloat16)
    Vc = torch.randn(B, T, Hkv, D, generator=gen).to(torch.bfloat16)
    k_new = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
    v_new = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
    t = torch.tensor([0, 57, 99], dtype=torch.int32)
    Kd, Vd = Kc.cuda(), Vc.cuda()
    dca.dca_kv_append(k_new.cuda(), v_new.cuda(), Kd, Vd, t.cuda(), s, c)
    dca.dca_sync_status()
    Kg, Vg = Kd.cpu(), Vd.cpu()
    for b in range(B):
        tb = int(t[b])
        ref = orc.rotate(k_new[b].float().numpy(), tb % s, 10000.0)
        got = Kg[b, tb].double().numpy()
        assert (np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-5).all()
        assert torch.equal(Vg[b, tb], v_new[b])
        keep = [r for r in range(T) if r != tb]
        assert torch.equal(Kg[b, keep], Kc[b, keep]) and torch.equal(Vg[b, keep], Vc[b, keep])


def test_cache_built_by_append_decodes_like_prefill():
    L, Hq, Hkv, D, s, c = 700, 8, 2, 128, 256, 384
    cfg = dict(B=1, L=L, Hq=Hq, Hkv=Hkv, D=D)
    Q, K, V = W.make_prefill_inputs(cfg, seed=21)
    O_p, LSE_p = dca.dca_attn_prefill(Q.cuda(), K.cuda(), V.cuda(), s, c)
    Kc = torch.zeros(1, L, Hkv, D, dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    Kd, Vd = K.cuda(), V.cuda()
    checkpoints = {0, 255, 256, 383, 384, 511, 512, 699}
    for tt in range(L):
        t = torch.tensor([tt], dtype=torch.int32, device="cuda")
        dca.dca_kv_append(Kd[:, tt].contiguous(), Vd[:, tt].contiguous(), Kc, Vc, t, s, c)
        if tt in checkpoints:
            O_d, LSE_d = dca.dca_attn_decode(Q[:, tt].contiguous().cuda(), Kc, Vc, t, s, c)
            dca.dca_sync_status()
            assert (O_d.cpu().float() - O_p[:, tt].cpu().float()).abs().max() < 2e-2, tt
            assert (LSE_d.cpu() - LSE_p[:, :, tt].cpu()).abs().max() < 2e-3, tt
            ref = orc.dca_prefill_rows(pu.F64View(Q), pu.F64View(K), pu.F64View(V), s, c,
                                       rows=[tt])
            o_ref = np.stack([ref[(0, h, tt)][0] for h in range(Hq)])
            l_ref = np.array([ref[(0, h, tt)][1] for h in range(Hq)])
            err = np.abs(O_d[0].cpu().double().numpy() - o_ref)
            lse_rel = np.abs(LSE_d[0].cpu().double().numpy() - l_ref) / np.maximum(
                np.abs(l_ref), 1.0)
            pu.assert_close(err.max(), err.mean(), lse_rel.max(), f"append+decode t={tt}")
    # the appended cache equals the library's own RoPE of the whole K at j mod s
    Kr = dca.dca_rope_rotate(Kd, dca.DCA_POS_KEY, s, c)
    assert torch.equal(Kr.cpu(), Kc.cpu()) and torch.equal(Vc.cpu(), V)


def test_kv_append_rejects_position_outside_cache():
    B, Hkv, D, T = 2, 1, 128, 16
    Kc = torch.zeros(B, T, Hkv, D, dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    new = torch.ones(B, Hkv, D, dtype=torch.bfloat16, device="cuda")
    t = torch.tensor([3, T], dtype=torch.int32, device="cuda")
    dca.dca_kv_append(new, new, Kc, Vc, t, 8, 12)
    with pytest.raises(dca.DcaError) as ei:
        dca.dca_sync_status()
    assert ei.value.status == 1
    assert Vc[0, 3].float().eq(1).all() and Vc[1].float().eq(0).all()
    dca.dca_sync_status()


def test_bounded_wait_reports_timeout_and_context_survives():
    # a wait on a barrier that nothing completes gives up after 20 ms
    dca.dca_debug_wait_timeout(20000)
    with pytest.raises(dca.DcaError) as ei:
        dca.dca_sync_status()
    assert ei.value.status == 4  # DCA_ERR_TIMEOUT
    dca.dca_sync_status()        # cleared
    # the context still runs kernels correctly afterwards
    qpos, kpos, piece = dca.dca_debug_index_map(12, 4, 6)
    dca.dca_sync_status()
    want = orc.index_map(12, 4, 6)
    assert (qpos.cpu().numpy() == want[0]).all() and (piece.cpu().numpy() == want[2]).all()
