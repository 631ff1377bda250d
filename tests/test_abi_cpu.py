"""Host-only checks of the C ABI: the library loads, exports every entry point
declared in include/dca.h, and rejects bad arguments before touching the GPU.

Every call here returns from the library's argument checks; none launches a
kernel, so the tests run on a machine without a GPU.
"""

import ctypes
import os
import re

import pytest

import long_context_attention_dca_b200 as dca

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dca.h")


def _header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dca_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from long_context_attention_dca_b200 import build
    build.build()
    return dca.lib()


def test_header_declares_the_binding_surface():
    assert _header_functions() == sorted(dca.EXPORTED_SYMBOLS)


def _header_prototypes():
    """{name: [parameter type strings]} for every function in the header."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(dca_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text):
        params = [p.strip() for p in m.group(2).split(",") if p.strip()]
        if params == ["void"]:
            params = []
        out[m.group(1)] = params
    return out


def _ctype_of(param):
    """The ctypes class the binding must use for a C parameter."""
    t = re.sub(r"\b[A-Za-z_][A-Za-z0-9_]*$", "", param).strip() if " " in param else param
    if "*" in t:
        return ctypes.c_void_p
    t = t.replace("const", "").strip()
    return {"int": ctypes.c_int, "float": ctypes.c_float, "size_t": ctypes.c_size_t,
            "dca_pos_rule_t": ctypes.c_int}[t]


def test_binding_signatures_match_the_header():
    # every argument the ctypes binding passes has the C type of the
    # header's parameter at that position (a count or type slip would pass
    # garbage through the ABI)
    protos = _header_prototypes()
    assert sorted(protos) == sorted(dca.EXPORTED_SYMBOLS)
    for name, params in protos.items():
        _, argtypes = dca._SIGS[name]
        assert len(argtypes) == len(params), (name, len(argtypes), len(params))
        for i, (want, got) in enumerate(zip(params, argtypes)):
            assert _ctype_of(want) is got, (name, i, want, got)


def test_library_exports_every_declared_symbol(lib):
    for name in _header_functions():
        assert hasattr(lib, name), name
    # C linkage: the dynamic symbol table has the plain names
    out = os.popen(f"nm -D --defined-only {dca.lib_path}").read()
    exported = set(re.findall(r"\bT (dca_[a-z0-9_]+)\b", out))
    assert set(_header_functions()) <= exported


def test_workspace_queries(lib):
    # Qrot (3 planes) + Krot, bf16, each rounded up to 256 bytes
    B, L, Hq, Hkv, D = 1, 1000, 4, 2, 64
    q = 3 * B * L * Hq * D * 2
    k = B * L * Hkv * D * 2
    up = lambda x: (x + 255) // 256 * 256
    assert dca.dca_attn_prefill_workspace(B, L, Hq, Hkv, D) == up(q) + up(k)
    assert dca.dca_attn_prefill_workspace(1, 10, 3, 2, 64) == 0  # Hq % Hkv
    assert dca.dca_attn_prefill_workspace(1, 10, 2, 2, 96) == 0  # D
    # decode: one fp32 row + (max, sum) per (b, head, split); splits of 2048
    # keys while B * ceil(Hq/8) * ceil(Tcap/2048) >= 1184, else of 1024
    assert dca.dca_attn_decode_workspace(16, 64, 128, 65536) == 16 * 64 * 32 * 130 * 4
    assert dca.dca_attn_decode_workspace(2, 8, 64, 1025) == 2 * 8 * 2 * 66 * 4
    assert dca.dca_attn_decode_workspace(4, 64, 128, 65536) == 4 * 64 * 64 * 130 * 4
    assert dca.dca_attn_decode_workspace(5, 64, 128, 65536) == 5 * 64 * 32 * 130 * 4
    # chunked prefill: three fp16 query rotations of the chunk + fp16 keys 0 .. t0+Lq-1
    assert dca.dca_attn_prefill_chunk_workspace(2, 100, 8, 2, 128, 50) == (
        up(3 * 2 * 100 * 8 * 128 * 2) + up(2 * 150 * 2 * 128 * 2))
    assert dca.dca_attn_prefill_chunk_workspace(2, 100, 8, 2, 128, -1) == 0
    # host prefill: whole-sequence fp16 keys and values + two chunk-sized sets
    # of staging (Q, K), outputs (O, LSE) and three query rotations (one set
    # per compute stream)
    B, L, Hq, Hkv, D, C = 2, 1000, 8, 2, 64, 300
    want = 2 * up(B * L * Hkv * D * 2) + 2 * (up(B * C * Hq * D * 2) + up(B * C * Hkv * D * 2) +
                                              up(B * C * Hq * D * 2) + up(B * Hq * C * 4)) + \
        2 * up(3 * B * C * Hq * D * 2)
    assert dca.dca_attn_prefill_host_workspace(B, L, Hq, Hkv, D, C) == want
    assert dca.dca_attn_prefill_host_workspace(B, L, Hq, Hkv, D, 0) == 0
    # SelfExtend: neighbour + grouped rotations of Q and K, fp16
    assert dca.dca_selfextend_workspace(1, 100, 4, 2, 64) == (up(2 * 100 * 4 * 64 * 2) +
                                                              up(2 * 100 * 2 * 64 * 2))
    # packed variable-length batch: the prefill workspace of one T-row sequence
    assert dca.dca_attn_prefill_varlen_workspace(777, 8, 2, 128) == (
        up(3 * 777 * 8 * 128 * 2) + up(777 * 2 * 128 * 2))
    assert dca.dca_attn_prefill_varlen_workspace(777, 8, 3, 128) == 0
    # packed chunks over caches: query rotations of the T rows + fp16 keys of
    # max_kv rows per sequence
    assert dca.dca_attn_prefill_varlen_chunk_workspace(3, 100, 300, 4, 2, 128) == (
        up(3 * 100 * 4 * 128 * 2) + up(3 * 300 * 2 * 128 * 2) + up(3 * 1 * 4))
    assert dca.dca_attn_prefill_varlen_chunk_workspace(3, 1000, 300, 4, 2, 128) == (
        up(3 * 1000 * 4 * 128 * 2) + up(3 * 300 * 2 * 128 * 2) + up(3 * 4 * 4))
    assert dca.dca_attn_prefill_varlen_chunk_workspace(3, 100, -1, 4, 2, 128) == 0


def test_prefill_path_selection(lib):
    assert dca.dca_prefill_path(16384, 128, 3072, 4096) in (dca.DCA_PATH_GENERAL,
                                                              dca.DCA_PATH_TCGEN05)
    assert dca.dca_prefill_path(1024, 64, 192, 256) == dca.DCA_PATH_TCGEN05
    assert dca.dca_prefill_path(1024, 128, 192, 256) == dca.DCA_PATH_TCGEN05
    assert dca.dca_prefill_path(1024, 128, 300, 256) == 0  # s > c
    assert dca.dca_prefill_path(1024, 96, 128, 256) == 0


P = ctypes.c_void_p


def _code(ret):
    return int(ret)


def test_argument_errors_return_codes(lib):
    fake = P(0x10000)      # 16-byte aligned, never dereferenced on these paths
    odd = P(0x10008)       # 8-byte aligned only
    ws = P(0x20000)
    # rope: null input, misaligned output, bad D, bad rule, s > c
    assert _code(lib.dca_rope_rotate(None, fake, 1, 8, 1, 64, 0, 4, 6, 1e4, 0, None)) == 1
    assert _code(lib.dca_rope_rotate(fake, odd, 1, 8, 1, 64, 0, 4, 6, 1e4, 0, None)) == 1
    assert _code(lib.dca_rope_rotate(fake, fake, 1, 8, 1, 80, 0, 4, 6, 1e4, 0, None)) == 2
    assert _code(lib.dca_rope_rotate(fake, fake, 1, 8, 1, 64, 0, 4, 6, 1e4, 9, None)) == 2
    assert _code(lib.dca_rope_rotate(fake, fake, 1, 8, 1, 64, 0, 7, 6, 1e4, 0, None)) == 2
    assert _code(lib.dca_rope_rotate(fake, fake, 1, 8, 1, 64, -1, 4, 6, 1e4, 4, None)) == 1
    assert "offset" in dca.dca_last_error_string()
    # empty problems are no-ops even with null pointers
    assert _code(lib.dca_rope_rotate(None, None, 0, 8, 1, 64, 0, 4, 6, 1e4, 0, None)) == 0
    assert _code(lib.dca_attn_prefill(None, None, None, None, None, 1, 0, 4, 2, 128, 3072, 4096,
                                      1e4, 0.0, None, 0, None)) == 0
    # prefill: Hq % Hkv, s > c, short workspace, null workspace
    args = (fake, fake, fake, fake, fake)
    assert _code(lib.dca_attn_prefill(*args, 1, 64, 3, 2, 128, 16, 32, 1e4, 0.0, ws, 1 << 30,
                                      None)) == 2
    assert _code(lib.dca_attn_prefill(*args, 1, 64, 4, 2, 128, 64, 32, 1e4, 0.0, ws, 1 << 30,
                                      None)) == 2
    assert _code(lib.dca_attn_prefill(*args, 1, 64, 4, 2, 128, 16, 32, 1e4, 0.0, ws, 100,
                                      None)) == 5
    assert "workspace" in dca.dca_last_error_string()
    assert _code(lib.dca_attn_prefill(*args, 1, 64, 4, 2, 128, 16, 32, 1e4, 0.0, None, 1 << 30,
                                      None)) == 1
    # a head dimension no path covers
    assert _code(lib.dca_prefill_attention(fake, fake, fake, 1, 64, 4, 2, 96, 96, 128, 0.0,
                                           2, ws, 1 << 30, None)) == 2
    assert _code(lib.dca_prefill_attention(fake, fake, fake, 1, 64, 4, 2, 128, 96, 128, 0.0,
                                           7, ws, 1 << 30, None)) == 1
    # decode: null t, Tcap < 1, short workspace
    dargs = (fake, fake, fake)
    assert _code(lib.dca_attn_decode(*dargs, None, fake, fake, 2, 8, 1, 128, 64, 16, 32, 1e4,
                                     0.0, ws, 1 << 30, None)) == 1
    assert _code(lib.dca_attn_decode(*dargs, fake, fake, fake, 2, 8, 1, 128, 0, 16, 32, 1e4,
                                     0.0, ws, 1 << 30, None)) == 1
    assert _code(lib.dca_attn_decode(*dargs, fake, fake, fake, 2, 8, 1, 128, 64, 16, 32, 1e4,
                                     0.0, ws, 8, None)) == 5
    # chunked prefill: chunk past the cache end, negative t0, short workspace
    cargs = (fake,) * 7
    assert _code(lib.dca_attn_prefill_chunk(*cargs, 1, 64, 4, 2, 128, 100, 128, 16, 32, 1e4,
                                            0.0, ws, 1 << 30, None)) == 1
    assert "outside cache" in dca.dca_last_error_string()
    assert _code(lib.dca_attn_prefill_chunk(*cargs, 1, 64, 4, 2, 128, -1, 128, 16, 32, 1e4,
                                            0.0, ws, 1 << 30, None)) == 1
    assert _code(lib.dca_attn_prefill_chunk(*cargs, 1, 64, 4, 2, 128, 64, 128, 16, 32, 1e4,
                                            0.0, ws, 64, None)) == 5
    # paged decode / append: null table, block_rows not a multiple of 64
    assert _code(lib.dca_attn_decode_paged(fake, fake, fake, None, 4, 64, 8, fake, fake, fake, 2,
                                           8, 1, 128, 64, 96, 1e4, 0.0, ws, 1 << 30, None)) == 1
    assert _code(lib.dca_attn_decode_paged(fake, fake, fake, fake, 4, 96, 8, fake, fake, fake, 2,
                                           8, 1, 128, 64, 96, 1e4, 0.0, ws, 1 << 30, None)) == 2
    assert _code(lib.dca_attn_decode_paged(fake, fake, fake, fake, 4, 64, 8, fake, fake, fake, 2,
                                           8, 1, 128, 64, 96, 1e4, 0.0, ws, 8, None)) == 5
    assert _code(lib.dca_kv_append_paged(fake, fake, fake, fake, fake, 4, 100, 8, fake, 2, 1,
                                         128, 64, 96, 1e4, None)) == 2
    # host prefill: chunk_rows < 1, null host buffer, short workspace
    hargs = (fake,) * 5
    assert _code(lib.dca_attn_prefill_host(*hargs, 1, 64, 4, 2, 128, 16, 32, 1e4, 0.0, 0, ws,
                                           1 << 30, None)) == 1
    assert _code(lib.dca_attn_prefill_host(None, fake, fake, fake, fake, 1, 64, 4, 2, 128, 16, 32,
                                           1e4, 0.0, 32, ws, 1 << 30, None)) == 1
    assert _code(lib.dca_attn_prefill_host(*hargs, 1, 64, 4, 2, 128, 16, 32, 1e4, 0.0, 32, ws, 64,
                                           None)) == 5
    # SelfExtend: G < 1, W < 1, short workspace
    sargs = (fake,) * 5
    assert _code(lib.dca_attn_prefill_selfextend(*sargs, 1, 64, 4, 2, 128, 0, 8, 1e4, 0.0, ws,
                                                 1 << 30, None)) == 1
    assert _code(lib.dca_attn_prefill_selfextend(*sargs, 1, 64, 4, 2, 128, 2, 0, 1e4, 0.0, ws,
                                                 1 << 30, None)) == 1
    assert _code(lib.dca_attn_prefill_selfextend(*sargs, 1, 64, 4, 2, 128, 2, 8, 1e4, 0.0, ws,
                                                 64, None)) == 5
    # packed batch: null or misaligned offsets, negative T, short workspace, s > c
    vargs = (fake,) * 5
    assert _code(lib.dca_attn_prefill_varlen(*vargs, None, 3, 64, 100, 4, 2, 128, 16, 32, 1e4,
                                             0.0, ws, 1 << 30, None)) == 1
    assert "cu_seqlens" in dca.dca_last_error_string()
    assert _code(lib.dca_attn_prefill_varlen(*vargs, P(0x10002), 3, 64, 100, 4, 2, 128, 16, 32,
                                             1e4, 0.0, ws, 1 << 30, None)) == 1
    assert _code(lib.dca_attn_prefill_varlen(*vargs, fake, 3, 64, -1, 4, 2, 128, 16, 32, 1e4,
                                             0.0, ws, 1 << 30, None)) == 1
    assert _code(lib.dca_attn_prefill_varlen(*vargs, fake, 3, 64, 100, 4, 2, 128, 16, 32, 1e4,
                                             0.0, ws, 64, None)) == 5
    assert _code(lib.dca_attn_prefill_varlen(*vargs, fake, 3, 64, 100, 4, 2, 128, 64, 32, 1e4,
                                             0.0, ws, 1 << 30, None)) == 2
    # empty batches are no-ops even with null pointers
    assert _code(lib.dca_attn_prefill_varlen(None, None, None, None, None, None, 0, 64, 100, 4,
                                             2, 128, 16, 32, 1e4, 0.0, None, 0, None)) == 0
    # packed chunks over caches: max_kv beyond the cache, null t0, short workspace
    cargs7 = (fake,) * 7
    assert _code(lib.dca_attn_prefill_varlen_chunk(*cargs7, fake, fake, 3, 64, 100, 500, 4, 2,
                                                   128, 400, 16, 32, 1e4, 0.0, ws, 1 << 30,
                                                   None)) == 1
    assert "max_kv" in dca.dca_last_error_string()
    assert _code(lib.dca_attn_prefill_varlen_chunk(*cargs7, fake, None, 3, 64, 100, 300, 4, 2,
                                                   128, 400, 16, 32, 1e4, 0.0, ws, 1 << 30,
                                                   None)) == 1
    assert _code(lib.dca_attn_prefill_varlen_chunk(*cargs7, fake, fake, 3, 64, 100, 300, 4, 2,
                                                   128, 400, 16, 32, 1e4, 0.0, ws, 64,
                                                   None)) == 5
    # paged: block_rows not a multiple of 128, null table, max_kv past the pool's reach
    pv = (fake,) * 5
    assert _code(lib.dca_attn_prefill_varlen_chunk_paged(*pv, fake, 4, 64, 16, fake, fake, fake,
                                                         fake, 3, 64, 100, 200, 4, 2, 128, 16,
                                                         32, 1e4, 0.0, ws, 1 << 30, None)) == 2
    assert _code(lib.dca_attn_prefill_varlen_chunk_paged(*pv, None, 4, 128, 16, fake, fake, fake,
                                                         fake, 3, 64, 100, 200, 4, 2, 128, 16,
                                                         32, 1e4, 0.0, ws, 1 << 30, None)) == 1
    assert _code(lib.dca_attn_prefill_varlen_chunk_paged(*pv, fake, 1, 128, 16, fake, fake, fake,
                                                         fake, 3, 64, 100, 200, 4, 2, 128, 16,
                                                         32, 1e4, 0.0, ws, 1 << 30, None)) == 1
    # wait self-test: deadline out of range
    assert _code(lib.dca_debug_wait_timeout(0, None)) == 1
    assert _code(lib.dca_debug_wait_timeout(5000000, None)) == 1
    # index map: L too large, s > c
    assert _code(lib.dca_debug_index_map(9000, 4, 6, fake, fake, fake, None)) == 1
    assert _code(lib.dca_debug_index_map(16, 8, 6, fake, fake, fake, None)) == 2


def test_binding_fails_loudly_without_cuda_tensors(lib):
    import torch
    x = torch.zeros(1, 4, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(dca.DcaError):
        dca.dca_rope_rotate(x, dca.DCA_POS_KEY, 4, 6)


def test_header_is_plain_c(tmp_path):
    # the boundary header must stay usable from C: compile a translation unit
    # that includes it with a strict C99 compiler (no CUDA or C++ types)
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_header.c"
    src.write_text('#include "dca.h"\n'
                   "size_t f(void) { return dca_attn_prefill_workspace(1, 1, 1, 1, 64); }\n")
    res = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                          os.path.dirname(HEADER), "-c", str(src), "-o",
                          str(tmp_path / "use_header.o")], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
