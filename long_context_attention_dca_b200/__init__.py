"""Dual Chunk Attention (DCA) for NVIDIA B200 -- thin Python binding.

Every function here marshals torch tensors into the C ABI declared in
``include/dca.h`` (data pointers, sizes, the current CUDA stream) and calls
the in-tree shared library ``libdca_b200.so``.  All arithmetic runs in the
library's sm_100a kernels; there is no CPU or PyTorch fallback: if the library
is missing or a call fails, a ``DcaError`` is raised.  PyTorch is used only
for device memory (outputs and the workspace the C ABI asks for) and streams.

Build the library with ``python -m long_context_attention_dca_b200.build``.
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "DcaError", "lib", "lib_path",
    "DCA_POS_KEY", "DCA_POS_Q_INTRA", "DCA_POS_Q_SUCC", "DCA_POS_Q_INTER", "DCA_POS_ABSOLUTE",
    "DCA_PATH_AUTO", "DCA_PATH_GENERAL", "DCA_PATH_TCGEN05",
    "dca_rope_rotate", "dca_attn_prefill_workspace", "dca_prefill_rope",
    "dca_prefill_attention", "dca_attn_prefill", "dca_prefill_path",
    "dca_attn_prefill_3pass_workspace", "dca_attn_prefill_3pass",
    "dca_attn_prefill_chunk_workspace", "dca_attn_prefill_chunk",
    "dca_attn_prefill_varlen_workspace", "dca_attn_prefill_varlen",
    "dca_attn_prefill_varlen_chunk_workspace", "dca_attn_prefill_varlen_chunk",
    "dca_attn_prefill_varlen_chunk_paged",
    "dca_attn_prefill_varlen_chunk_mirror_workspace", "dca_attn_prefill_varlen_chunk_mirror",
    "dca_selfextend_workspace", "dca_attn_prefill_selfextend",
    "dca_attn_prefill_host_workspace", "dca_attn_prefill_host",
    "dca_attn_decode_paged", "dca_kv_append_paged",
    "dca_attn_decode_workspace", "dca_attn_decode", "dca_attn_decode_noalloc", "dca_kv_append",
    "dca_debug_index_map", "dca_debug_wait_timeout",
    "dca_sync_status", "dca_last_error_string", "EXPORTED_SYMBOLS",
]

DCA_POS_KEY, DCA_POS_Q_INTRA, DCA_POS_Q_SUCC, DCA_POS_Q_INTER, DCA_POS_ABSOLUTE = range(5)
DCA_PATH_AUTO, DCA_PATH_GENERAL, DCA_PATH_TCGEN05 = range(3)
_STATUS = {0: "DCA_OK", 1: "DCA_ERR_INVALID_ARG", 2: "DCA_ERR_UNSUPPORTED",
           3: "DCA_ERR_CUDA", 4: "DCA_ERR_TIMEOUT", 5: "DCA_ERR_WORKSPACE"}

lib_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdca_b200.so")

_I, _F, _P, _Z = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
# name -> (restype, argtypes); mirrors include/dca.h
_SIGS = {
    "dca_rope_rotate": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "dca_attn_prefill_workspace": (_Z, [_I, _I, _I, _I, _I]),
    "dca_prefill_rope": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "dca_prefill_attention": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _Z, _P]),
    "dca_attn_prefill": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _P, _Z,
                              _P]),
    "dca_prefill_path": (_I, [_I, _I, _I, _I]),
    "dca_attn_prefill_3pass_workspace": (_Z, [_I, _I, _I, _I, _I]),
    "dca_attn_prefill_varlen_workspace": (_Z, [_I, _I, _I, _I]),
    "dca_attn_prefill_varlen_chunk_workspace": (_Z, [_I, _I, _I, _I, _I, _I]),
    "dca_attn_prefill_varlen_chunk": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I,
                                           _I, _I, _I, _I, _I, _I, _F, _F, _P, _Z, _P]),
    "dca_attn_prefill_varlen_chunk_mirror_workspace": (_Z, [_I, _I, _I, _I, _I]),
    "dca_attn_prefill_varlen_chunk_mirror": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I,
                                                  _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _F,
                                                  _P, _Z, _P]),
    "dca_attn_prefill_varlen_chunk_paged": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P,
                                                 _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _F,
                                                 _P, _Z, _P]),
    "dca_attn_prefill_varlen": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F,
                                     _F, _P, _Z, _P]),
    "dca_attn_prefill_chunk_workspace": (_Z, [_I, _I, _I, _I, _I, _I]),
    "dca_selfextend_workspace": (_Z, [_I, _I, _I, _I, _I]),
    "dca_attn_prefill_host_workspace": (_Z, [_I, _I, _I, _I, _I, _I]),
    "dca_attn_decode_paged": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _I, _I, _I, _I, _I,
                                   _I, _F, _F, _P, _Z, _P]),
    "dca_kv_append_paged": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _I, _I, _I, _I, _I, _F,
                                 _P]),
    "dca_attn_prefill_host": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _I,
                                   _P, _Z, _P]),
    "dca_attn_prefill_selfextend": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F,
                                         _P, _Z, _P]),
    "dca_attn_prefill_chunk": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                                    _I, _F, _F, _P, _Z, _P]),
    "dca_attn_prefill_3pass": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _P,
                                    _Z, _P]),
    "dca_attn_decode_workspace": (_Z, [_I, _I, _I, _I]),
    "dca_attn_decode": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _P,
                             _Z, _P]),
    "dca_kv_append": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "dca_attn_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F,
                                     _F, _P]),
    "dca_debug_index_map": (_I, [_I, _I, _I, _P, _P, _P, _P]),
    "dca_debug_wait_timeout": (_I, [_I, _P]),
    "dca_sync_status": (_I, [_P]),
    "dca_last_error_string": (ctypes.c_char_p, []),
}
EXPORTED_SYMBOLS = tuple(_SIGS)


class DcaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load the shared library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise DcaError(3, f"{lib_path} not built; run "
                              "python -m long_context_attention_dca_b200.build")
        handle = ctypes.CDLL(lib_path)
        for name, (res, args) in _SIGS.items():
            f = getattr(handle, name)
            f.restype, f.argtypes = res, args
        _lib = handle
    return _lib


def _check(status: int):
    if status != 0:
        raise DcaError(status, lib().dca_last_error_string().decode())


def _stream(t: torch.Tensor | None = None):
    dev = t.device if t is not None else torch.device("cuda")
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise DcaError(1, f"{name} must be a CUDA tensor")
    if t.dtype != dtype or t.dim() != ndim or not t.is_contiguous():
        raise DcaError(1, f"{name} must be a contiguous {ndim}-d {dtype} tensor, "
                          f"got {t.dtype} {tuple(t.shape)}")


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def dca_last_error_string() -> str:
    return lib().dca_last_error_string().decode()


def dca_sync_status(device=None) -> None:
    """Synchronise the current stream and raise if a kernel reported an error."""
    dev = torch.device(device) if device is not None else torch.device("cuda")
    _check(lib().dca_sync_status(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)))


def dca_debug_wait_timeout(deadline_us: int = 20000) -> None:
    """Enqueue the bounded-wait self-test (see include/dca.h)."""
    _check(lib().dca_debug_wait_timeout(deadline_us, _stream()))


def dca_rope_rotate(x: torch.Tensor, rule: int, s: int, c: int, base: float = 10000.0,
                    pos_offset: int = 0, out: torch.Tensor | None = None) -> torch.Tensor:
    """Rotate x [B, L, H, D] bf16 at the positions of a DCA rule (see dca.h)."""
    _need(x, "x", torch.bfloat16, 4)
    out = torch.empty_like(x) if out is None else out
    _need(out, "out", torch.bfloat16, 4)
    B, L, H, D = x.shape
    _check(lib().dca_rope_rotate(_ptr(x), _ptr(out), B, L, H, D, pos_offset, s, c, base, rule,
                                 _stream(x)))
    return out


def dca_attn_prefill_workspace(B: int, L: int, Hq: int, Hkv: int, D: int) -> int:
    return int(lib().dca_attn_prefill_workspace(B, L, Hq, Hkv, D))


def dca_prefill_path(L: int, D: int, s: int, c: int) -> int:
    return int(lib().dca_prefill_path(L, D, s, c))


def dca_prefill_rope(Q, K, s, c, base=10000.0, workspace=None):
    """Fused RoPE step alone; returns the filled workspace (uint8 tensor)."""
    _need(Q, "Q", torch.bfloat16, 4)
    _need(K, "K", torch.bfloat16, 4)
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    nbytes = dca_attn_prefill_workspace(B, L, Hq, Hkv, D)
    ws = _workspace(nbytes, Q.device) if workspace is None else workspace
    _check(lib().dca_prefill_rope(_ptr(Q), _ptr(K), B, L, Hq, Hkv, D, s, c, base, _ptr(ws),
                                  ws.numel(), _stream(Q)))
    return ws


def dca_prefill_attention(V, workspace, Hq, s, c, scale=0.0, path=DCA_PATH_AUTO, O=None,
                          LSE=None):
    """Attention step alone over a workspace from dca_prefill_rope."""
    _need(V, "V", torch.bfloat16, 4)
    B, L, Hkv, D = V.shape
    O = torch.empty((B, L, Hq, D), dtype=torch.bfloat16, device=V.device) if O is None else O
    LSE = torch.empty((B, Hq, L), dtype=torch.float32, device=V.device) if LSE is None else LSE
    _need(O, "O", torch.bfloat16, 4)
    _need(LSE, "LSE", torch.float32, 3)
    _check(lib().dca_prefill_attention(_ptr(V), _ptr(O), _ptr(LSE), B, L, Hq, Hkv, D, s, c,
                                       scale, path, _ptr(workspace), workspace.numel(),
                                       _stream(V)))
    return O, LSE


def dca_attn_prefill(Q, K, V, s, c, base=10000.0, scale=0.0, workspace=None, O=None,
                     LSE=None):
    """DCA prefill: returns (O [B, L, Hq, D] bf16, LSE [B, Hq, L] fp32)."""
    _need(Q, "Q", torch.bfloat16, 4)
    _need(K, "K", torch.bfloat16, 4)
    _need(V, "V", torch.bfloat16, 4)
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    nbytes = dca_attn_prefill_workspace(B, L, Hq, Hkv, D)
    ws = _workspace(nbytes, Q.device) if workspace is None else workspace
    O = torch.empty_like(Q) if O is None else O
    LSE = torch.empty((B, Hq, L), dtype=torch.float32, device=Q.device) if LSE is None else LSE
    _need(O, "O", torch.bfloat16, 4)
    _need(LSE, "LSE", torch.float32, 3)
    _check(lib().dca_attn_prefill(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, L, Hq, Hkv,
                                  D, s, c, base, scale, _ptr(ws), ws.numel(), _stream(Q)))
    return O, LSE


def dca_attn_prefill_varlen_workspace(T: int, Hq: int, Hkv: int, D: int) -> int:
    return int(lib().dca_attn_prefill_varlen_workspace(T, Hq, Hkv, D))


def dca_attn_prefill_varlen(Q, K, V, cu_seqlens, max_seqlen, s, c, base=10000.0, scale=0.0,
                            workspace=None, O=None, LSE=None):
    """Packed variable-length prefill.  Q [T, Hq, D], K, V [T, Hkv, D] bf16;
    cu_seqlens int32 [B+1] on the device (sequence b owns rows cu_seqlens[b]
    .. cu_seqlens[b+1]-1); max_seqlen (int) bounds every sequence's length.
    Returns (O [T, Hq, D] bf16, LSE [Hq, T] fp32); rows of no sequence are left
    as allocated."""
    _need(Q, "Q", torch.bfloat16, 3)
    _need(K, "K", torch.bfloat16, 3)
    _need(V, "V", torch.bfloat16, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    T, Hq, D = Q.shape
    Hkv = K.shape[1]
    B = cu_seqlens.numel() - 1
    nbytes = dca_attn_prefill_varlen_workspace(T, Hq, Hkv, D)
    ws = _workspace(nbytes, Q.device) if workspace is None else workspace
    O = torch.empty_like(Q) if O is None else O
    LSE = torch.empty((Hq, T), dtype=torch.float32, device=Q.device) if LSE is None else LSE
    _need(O, "O", torch.bfloat16, 3)
    _need(LSE, "LSE", torch.float32, 2)
    _check(lib().dca_attn_prefill_varlen(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE),
                                         _ptr(cu_seqlens), B, int(max_seqlen), T, Hq, Hkv, D, s,
                                         c, base, scale, _ptr(ws), ws.numel(), _stream(Q)))
    return O, LSE


def dca_attn_prefill_varlen_chunk_workspace(B: int, T: int, max_kv: int, Hq: int, Hkv: int,
                                            D: int) -> int:
    return int(lib().dca_attn_prefill_varlen_chunk_workspace(B, T, max_kv, Hq, Hkv, D))


def dca_attn_prefill_varlen_chunk(Q, K, V, Kcache, Vcache, cu_seqlens, t0, max_seqlen, max_kv,
                                  s, c, base=10000.0, scale=0.0, workspace=None, O=None,
                                  LSE=None):
    """Packed chunks over per-sequence caches.  Q [T, Hq, D], K, V [T, Hkv, D]
    bf16 (sequence b's new tokens at rows cu_seqlens[b] .. cu_seqlens[b+1]-1);
    Kcache, Vcache [B, Tcap, Hkv, D] bf16 holding t0[b] cached rows each;
    cu_seqlens int32 [B+1] and t0 int32 [B] on the device.  Returns
    (O [T, Hq, D] bf16, LSE [Hq, T] fp32) and extends the caches."""
    _need(Q, "Q", torch.bfloat16, 3)
    _need(K, "K", torch.bfloat16, 3)
    _need(V, "V", torch.bfloat16, 3)
    _need(Kcache, "Kcache", torch.bfloat16, 4)
    _need(Vcache, "Vcache", torch.bfloat16, 4)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    _need(t0, "t0", torch.int32, 1)
    T, Hq, D = Q.shape
    Hkv = K.shape[1]
    B, Tcap = Kcache.shape[:2]
    nbytes = dca_attn_prefill_varlen_chunk_workspace(B, T, int(max_kv), Hq, Hkv, D)
    ws = _workspace(nbytes, Q.device) if workspace is None else workspace
    O = torch.empty_like(Q) if O is None else O
    LSE = torch.empty((Hq, T), dtype=torch.float32, device=Q.device) if LSE is None else LSE
    _need(O, "O", torch.bfloat16, 3)
    _need(LSE, "LSE", torch.float32, 2)
    _check(lib().dca_attn_prefill_varlen_chunk(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(Kcache), _ptr(Vcache), _ptr(O), _ptr(LSE),
        _ptr(cu_seqlens), _ptr(t0), B, int(max_seqlen), T, int(max_kv), Hq, Hkv, D, Tcap, s, c,
        base, scale, _ptr(ws), ws.numel(), _stream(Q)))
    return O, LSE



def dca_attn_prefill_varlen_chunk_mirror_workspace(B: int, T: int, Hq: int, Hkv: int,
                                                   D: int) -> int:
    return lib().dca_attn_prefill_varlen_chunk_mirror_workspace(B, T, Hq, Hkv, D)


def dca_attn_prefill_varlen_chunk_mirror(Q, K, V, Kcache, Vcache, Kf16, cu_seqlens, t0,
                                         max_seqlen, max_kv, s, c, base=10000.0, scale=0.0,
                                         workspace=None, O=None, LSE=None):
    """As dca_attn_prefill_varlen_chunk, with Kf16 [B, Tcap, Hkv, D] fp16: the
    caller's fp16 copy of the rotated keys, read for rows 0 .. t0[b]-1 and
    extended by this call's new rows (see dca.h)."""
    _need(Q, "Q", torch.bfloat16, 3)
    _need(K, "K", torch.bfloat16, 3)
    _need(V, "V", torch.bfloat16, 3)
    _need(Kcache, "Kcache", torch.bfloat16, 4)
    _need(Vcache, "Vcache", torch.bfloat16, 4)
    _need(Kf16, "Kf16", torch.float16, 4)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    _need(t0, "t0", torch.int32, 1)
    T, Hq, D = Q.shape
    Hkv = K.shape[1]
    B, Tcap = Kcache.shape[:2]
    if tuple(Kf16.shape) != tuple(Kcache.shape):
        raise DcaError(1, "Kf16 must have the shape of Kcache")
    nbytes = dca_attn_prefill_varlen_chunk_mirror_workspace(B, T, Hq, Hkv, D)
    ws = _workspace(nbytes, Q.device) if workspace is None else workspace
    O = torch.empty_like(Q) if O is None else O
    LSE = torch.empty((Hq, T), dtype=torch.float32, device=Q.device) if LSE is None else LSE
    _need(O, "O", torch.bfloat16, 3)
    _need(LSE, "LSE", torch.float32, 2)
    _check(lib().dca_attn_prefill_varlen_chunk_mirror(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(Kcache), _ptr(Vcache), _ptr(Kf16), _ptr(O), _ptr(LSE),
        _ptr(cu_seqlens), _ptr(t0), B, int(max_seqlen), T, int(max_kv), Hq, Hkv, D, Tcap, s, c,
        base, scale, _ptr(ws), ws.numel(), _stream(Q)))
    return O, LSE

def dca_attn_prefill_varlen_chunk_paged(Q, K, V, Kpool, Vpool, block_table, cu_seqlens, t0,
                                        max_seqlen, max_kv, s, c, base=10000.0, scale=0.0,
                                        workspace=None, O=None, LSE=None):
    """dca_attn_prefill_varlen_chunk over paged pools Kpool, Vpool
    [num_blocks, block_rows, Hkv, D] bf16 and block_table int32 [B, max_blocks]
    on the device (block_rows a multiple of 128)."""
    _need(Q, "Q", torch.bfloat16, 3)
    _need(K, "K", torch.bfloat16, 3)
    _need(V, "V", torch.bfloat16, 3)
    _need(Kpool, "Kpool", torch.bfloat16, 4)
    _need(Vpool, "Vpool", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    _need(t0, "t0", torch.int32, 1)
    T, Hq, D = Q.shape
    Hkv = K.shape[1]
    num_blocks, block_rows = Kpool.shape[:2]
    B, max_blocks = block_table.shape
    nbytes = dca_attn_prefill_varlen_chunk_workspace(B, T, int(max_kv), Hq, Hkv, D)
    ws = _workspace(nbytes, Q.device) if workspace is None else workspace
    O = torch.empty_like(Q) if O is None else O
    LSE = torch.empty((Hq, T), dtype=torch.float32, device=Q.device) if LSE is None else LSE
    _need(O, "O", torch.bfloat16, 3)
    _need(LSE, "LSE", torch.float32, 2)
    _check(lib().dca_attn_prefill_varlen_chunk_paged(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(Kpool), _ptr(Vpool), _ptr(block_table), max_blocks,
        block_rows, num_blocks, _ptr(O), _ptr(LSE), _ptr(cu_seqlens), _ptr(t0), B,
        int(max_seqlen), T, int(max_kv), Hq, Hkv, D, s, c, base, scale, _ptr(ws), ws.numel(),
        _stream(Q)))
    return O, LSE


def dca_attn_prefill_3pass_workspace(B: int, L: int, Hq: int, Hkv: int, D: int) -> int:
    return int(lib().dca_attn_prefill_3pass_workspace(B, L, Hq, Hkv, D))


def dca_attn_prefill_3pass(Q, K, V, s, c, base=10000.0, scale=0.0):
    """DCA prefill as three single-piece flash passes merged by LSE."""
    _need(Q, "Q", torch.bfloat16, 4)
    _need(K, "K", torch.bfloat16, 4)
    _need(V, "V", torch.bfloat16, 4)
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    nbytes = dca_attn_prefill_3pass_workspace(B, L, Hq, Hkv, D)
    ws = _workspace(nbytes, Q.device)
    O = torch.empty_like(Q)
    LSE = torch.empty((B, Hq, L), dtype=torch.float32, device=Q.device)
    _check(lib().dca_attn_prefill_3pass(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, L, Hq,
                                        Hkv, D, s, c, base, scale, _ptr(ws), ws.numel(),
                                        _stream(Q)))
    return O, LSE


def dca_attn_prefill_chunk_workspace(B: int, Lq: int, Hq: int, Hkv: int, D: int, t0: int) -> int:
    return int(lib().dca_attn_prefill_chunk_workspace(B, Lq, Hq, Hkv, D, t0))


def dca_attn_prefill_chunk(Q, K, V, Kcache, Vcache, t0, s, c, base=10000.0, scale=0.0):
    """Prefill of the chunk Q/K/V at absolute rows t0 .. t0+Lq-1 against the
    caches (rotated keys and values of rows 0 .. t0-1); appends the chunk to
    the caches in place and returns its (O, LSE)."""
    _need(Q, "Q", torch.bfloat16, 4)
    _need(K, "K", torch.bfloat16, 4)
    _need(V, "V", torch.bfloat16, 4)
    _need(Kcache, "Kcache", torch.bfloat16, 4)
    _need(Vcache, "Vcache", torch.bfloat16, 4)
    B, Lq, Hq, D = Q.shape
    Hkv = K.shape[2]
    Tcap = Kcache.shape[1]
    nbytes = dca_attn_prefill_chunk_workspace(B, Lq, Hq, Hkv, D, int(t0))
    ws = _workspace(nbytes, Q.device)
    O = torch.empty_like(Q)
    LSE = torch.empty((B, Hq, Lq), dtype=torch.float32, device=Q.device)
    _check(lib().dca_attn_prefill_chunk(_ptr(Q), _ptr(K), _ptr(V), _ptr(Kcache), _ptr(Vcache),
                                        _ptr(O), _ptr(LSE), B, Lq, Hq, Hkv, D, int(t0), Tcap, s,
                                        c, base, scale, _ptr(ws), ws.numel(), _stream(Q)))
    return O, LSE


def dca_selfextend_workspace(B: int, L: int, Hq: int, Hkv: int, D: int) -> int:
    return int(lib().dca_selfextend_workspace(B, L, Hq, Hkv, D))


def dca_attn_prefill_selfextend(Q, K, V, G, W, base=10000.0, scale=0.0):
    """SelfExtend prefill (neighbour window W, group size G) -> (O, LSE)."""
    _need(Q, "Q", torch.bfloat16, 4)
    _need(K, "K", torch.bfloat16, 4)
    _need(V, "V", torch.bfloat16, 4)
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    ws = _workspace(dca_selfextend_workspace(B, L, Hq, Hkv, D), Q.device)
    O = torch.empty_like(Q)
    LSE = torch.empty((B, Hq, L), dtype=torch.float32, device=Q.device)
    _check(lib().dca_attn_prefill_selfextend(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, L,
                                             Hq, Hkv, D, int(G), int(W), base, scale, _ptr(ws),
                                             ws.numel(), _stream(Q)))
    return O, LSE


def dca_attn_prefill_host_workspace(B: int, L: int, Hq: int, Hkv: int, D: int,
                                    chunk_rows: int) -> int:
    return int(lib().dca_attn_prefill_host_workspace(B, L, Hq, Hkv, D, chunk_rows))


def dca_attn_prefill_host(Q, K, V, s, c, base=10000.0, scale=0.0, chunk_rows=2048,
                          workspace=None, O=None, LSE=None, device=None):
    """DCA prefill with host (CPU) tensors in and out, copies overlapped with
    the kernels.  Q, K, V: contiguous bf16 CPU tensors (pinned for overlap);
    returns CPU (O, LSE), written into O / LSE when given.  `workspace` is a
    device uint8 tensor (allocated when None) on `device`.  Asynchronous on
    the device's current stream: synchronise before reading O and LSE."""
    for t, name in ((Q, "Q"), (K, "K"), (V, "V")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.bfloat16 \
                or t.dim() != 4 or not t.is_contiguous():
            raise DcaError(1, f"{name} must be a contiguous 4-d bf16 CPU tensor")
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else \
        torch.device(device)
    if workspace is None:
        workspace = _workspace(dca_attn_prefill_host_workspace(B, L, Hq, Hkv, D, chunk_rows), dev)
    if O is None:
        O = torch.empty(Q.shape, dtype=torch.bfloat16, pin_memory=True)
    if LSE is None:
        LSE = torch.empty((B, Hq, L), dtype=torch.float32, pin_memory=True)
    with torch.cuda.device(dev):
        strm = torch.cuda.current_stream(dev).cuda_stream
        _check(lib().dca_attn_prefill_host(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, L,
                                           Hq, Hkv, D, s, c, base, scale, int(chunk_rows),
                                           _ptr(workspace), workspace.numel(), strm))
    return O, LSE


def dca_attn_decode_workspace(B: int, Hq: int, D: int, Tcap: int) -> int:
    return int(lib().dca_attn_decode_workspace(B, Hq, D, Tcap))


def dca_attn_decode(q, Kcache, Vcache, t, s, c, base=10000.0, scale=0.0, workspace=None,
                    O=None, LSE=None):
    """DCA decode: q [B, Hq, D] unrotated; caches [B, Tcap, Hkv, D] with keys
    pre-rotated at j mod s; t int32 [B] on device.  Returns (O, LSE)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(Kcache, "Kcache", torch.bfloat16, 4)
    _need(Vcache, "Vcache", torch.bfloat16, 4)
    _need(t, "t", torch.int32, 1)
    B, Hq, D = q.shape
    Tcap, Hkv = Kcache.shape[1], Kcache.shape[2]
    nbytes = dca_attn_decode_workspace(B, Hq, D, Tcap)
    ws = _workspace(nbytes, q.device) if workspace is None else workspace
    O = torch.empty_like(q) if O is None else O
    LSE = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if LSE is None else LSE
    _check(lib().dca_attn_decode(_ptr(q), _ptr(Kcache), _ptr(Vcache), _ptr(t), _ptr(O),
                                 _ptr(LSE), B, Hq, Hkv, D, Tcap, s, c, base, scale, _ptr(ws),
                                 ws.numel(), _stream(q)))
    return O, LSE


def dca_kv_append(k_new, v_new, Kcache, Vcache, t, s, c, base=10000.0):
    """Write each sequence's new token (key rotated at t mod s) to cache row t."""
    _need(k_new, "k_new", torch.bfloat16, 3)
    _need(v_new, "v_new", torch.bfloat16, 3)
    _need(Kcache, "Kcache", torch.bfloat16, 4)
    _need(Vcache, "Vcache", torch.bfloat16, 4)
    _need(t, "t", torch.int32, 1)
    B, Hkv, D = k_new.shape
    _check(lib().dca_kv_append(_ptr(k_new), _ptr(v_new), _ptr(Kcache), _ptr(Vcache), _ptr(t), B,
                               Hkv, D, Kcache.shape[1], s, c, base, _stream(k_new)))


def dca_attn_decode_paged(q, Kpool, Vpool, block_table, t, s, c, base=10000.0, scale=0.0,
                          workspace=None):
    """Decode over paged pools Kpool, Vpool [num_blocks][block_rows][Hkv][D] with
    block_table int32 [B][max_blocks] (device)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(Kpool, "Kpool", torch.bfloat16, 4)
    _need(Vpool, "Vpool", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(t, "t", torch.int32, 1)
    B, Hq, D = q.shape
    num_blocks, block_rows, Hkv = Kpool.shape[0], Kpool.shape[1], Kpool.shape[2]
    max_blocks = block_table.shape[1]
    if workspace is None:
        workspace = _workspace(dca_attn_decode_workspace(B, Hq, D, max_blocks * block_rows),
                               q.device)
    O = torch.empty_like(q)
    LSE = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check(lib().dca_attn_decode_paged(_ptr(q), _ptr(Kpool), _ptr(Vpool), _ptr(block_table),
                                       max_blocks, block_rows, num_blocks, _ptr(t), _ptr(O),
                                       _ptr(LSE), B, Hq, Hkv, D, s, c, base, scale,
                                       _ptr(workspace), workspace.numel(), _stream(q)))
    return O, LSE


def dca_kv_append_paged(k_new, v_new, Kpool, Vpool, block_table, t, s, c, base=10000.0):
    """Append one token per sequence into paged pools (in place)."""
    _need(k_new, "k_new", torch.bfloat16, 3)
    _need(v_new, "v_new", torch.bfloat16, 3)
    _need(Kpool, "Kpool", torch.bfloat16, 4)
    _need(Vpool, "Vpool", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(t, "t", torch.int32, 1)
    B, Hkv, D = k_new.shape
    _check(lib().dca_kv_append_paged(_ptr(k_new), _ptr(v_new), _ptr(Kpool), _ptr(Vpool),
                                     _ptr(block_table), block_table.shape[1], Kpool.shape[1],
                                     Kpool.shape[0], _ptr(t), B, Hkv, D, s, c, base,
                                     _stream(k_new)))


def dca_attn_decode_noalloc(q, Kcache, Vcache, t, s, c, base=10000.0, scale=0.0, O=None,
                            LSE=None):
    """dca_attn_decode without a workspace: for callers that cannot allocate
    device memory, the library uses its fixed 48 MiB scratch array (shared by
    all calls; see include/dca.h).  Outputs may be passed in preallocated."""
    _need(q, "q", torch.bfloat16, 3)
    _need(Kcache, "Kcache", torch.bfloat16, 4)
    _need(Vcache, "Vcache", torch.bfloat16, 4)
    _need(t, "t", torch.int32, 1)
    B, Hq, D = q.shape
    Tcap, Hkv = Kcache.shape[1], Kcache.shape[2]
    O = torch.empty_like(q) if O is None else O
    LSE = torch.empty((B, Hq), dtype=torch.float32, device=q.device) if LSE is None else LSE
    _check(lib().dca_attn_decode_noalloc(_ptr(q), _ptr(Kcache), _ptr(Vcache), _ptr(t), _ptr(O),
                                         _ptr(LSE), B, Hq, Hkv, D, Tcap, s, c, base, scale,
                                         _stream(q)))
    return O, LSE


def dca_debug_index_map(L: int, s: int, c: int, device="cuda"):
    """Dense (qpos, kpos, piece) tables [L, L] computed on the GPU."""
    qpos = torch.empty((L, L), dtype=torch.int32, device=device)
    kpos = torch.empty((L, L), dtype=torch.int32, device=device)
    piece = torch.empty((L, L), dtype=torch.int8, device=device)
    _check(lib().dca_debug_index_map(L, s, c, _ptr(qpos), _ptr(kpos), _ptr(piece),
                                     _stream(qpos)))
    return qpos, kpos, piece
