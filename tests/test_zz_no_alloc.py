"""dca_attn_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (for example a plugin inside a serving framework whose
allocator owns all GPU memory, or a decode loop that must avoid cudaMalloc's
implicit synchronisation).  It keeps the split-KV scratch in a fixed array in
the library instead of a caller workspace.

The GPU test calls it twice in a row through the C ABI, on two different
decode problems, and checks each result against dca_attn_decode (the entry
point with a caller workspace) within the parity tolerance used by the other
tests.  This file is collected last so that a stop-at-first-failure run has
already run every other test; it also passes on its own in a fresh process.
"""

import ctypes

import pytest
import torch

import long_context_attention_dca_b200 as dca
from long_context_attention_dca_b200 import workloads as W
from tests import parity_util as pu


@pytest.fixture(scope="module")
def lib():
    from long_context_attention_dca_b200 import build
    build.build()
    return dca.lib()


def _inputs(B, Hq, Hkv, D, Tcap, t_values, seed):
    cfg = dict(B=B, Hq=Hq, Hkv=Hkv, D=D, Tcap=Tcap, t_lo=0, t_hi=Tcap)
    _, q, Kc, Vc = W.make_decode_inputs(cfg, seed=seed)
    t = torch.tensor(t_values, dtype=torch.int32)
    return [x.cuda() for x in (t, q, Kc, Vc)]


def _call_noalloc(lib, t, q, Kc, Vc, s, c):
    B, Hq, D = q.shape
    Tcap, Hkv = Kc.shape[1], Kc.shape[2]
    O = torch.empty_like(q)
    LSE = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    P = ctypes.c_void_p
    st = lib.dca_attn_decode_noalloc(P(q.data_ptr()), P(Kc.data_ptr()), P(Vc.data_ptr()),
                                     P(t.data_ptr()), P(O.data_ptr()), P(LSE.data_ptr()), B, Hq,
                                     Hkv, D, Tcap, s, c, 10000.0, 0.0,
                                     P(torch.cuda.current_stream().cuda_stream))
    assert st == 0, dca.dca_last_error_string()
    return O, LSE


def _compare(O_new, LSE_new, O_ref, LSE_ref, what):
    d = (O_new.float() - O_ref.float()).abs()
    lse_rel = ((LSE_new - LSE_ref).abs() / LSE_ref.abs().clamp_min(1.0)).max().item()
    pu.assert_close(d.max().item(), d.mean().item(), lse_rel, what)


@pytest.mark.gpu
def test_noalloc_matches_workspace_decode_two_calls(lib):
    problems = [
        # (B, Hq, Hkv, D, Tcap, t values, s, c, seed)
        (4, 16, 2, 128, 9000, [8999, 4096, 3071, 17], 3072, 4096, 1),
        (3, 8, 8, 64, 2500, [2499, 0, 1234], 256, 384, 2),
    ]
    for B, Hq, Hkv, D, Tcap, tv, s, c, seed in problems:
        t, q, Kc, Vc = _inputs(B, Hq, Hkv, D, Tcap, tv, seed)
        O_ref, LSE_ref = dca.dca_attn_decode(q, Kc, Vc, t, s, c)
        O_new, LSE_new = _call_noalloc(lib, t, q, Kc, Vc, s, c)
        dca.dca_sync_status()
        assert torch.isfinite(O_new.float()).all() and torch.isfinite(LSE_new).all()
        _compare(O_new, LSE_new, O_ref, LSE_ref, f"noalloc B={B} Tcap={Tcap}")


def test_noalloc_rejects_scratch_beyond_its_limit(lib):
    # 64 sequences x 64 heads x 64 splits x (128 + 2) floats > 48 MiB; the
    # check runs on the host before anything touches a GPU.
    fake = ctypes.c_void_p(0x10000)
    st = lib.dca_attn_decode_noalloc(fake, fake, fake, fake, fake, fake, 64, 64, 8, 128, 65536,
                                     3072, 4096, 10000.0, 0.0, None)
    assert st == 5
    assert "fixed" in dca.dca_last_error_string()
    # the decode workload itself (16 x 64 heads, Tcap 65536) fits
    assert dca.dca_attn_decode_workspace(16, 64, 128, 65536) <= 48 << 20
