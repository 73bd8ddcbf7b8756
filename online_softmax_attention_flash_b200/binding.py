"""Thin ctypes binding over libattn_b200.so (argument marshalling only).

Every function here has the name of the C entry point it calls (include/attn.h),
checks that the torch tensors it is given are CUDA tensors of the right dtype,
shape and layout, passes their device pointers and the current CUDA stream,
and raises :class:`AttnError` on a non-zero status. No attention arithmetic
happens in Python, and there is no fallback: if the shared library is missing
the first call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libattn_b200.so")

STATUS = {
    0: "ATTN_OK", -1: "ATTN_ERR_NULL", -2: "ATTN_ERR_SHAPE", -3: "ATTN_ERR_UNSUPPORTED",
    -4: "ATTN_ERR_ALIGN", -5: "ATTN_ERR_WORKSPACE", -6: "ATTN_ERR_CUDA",
    -7: "ATTN_ERR_DEVICE_TIMEOUT", -8: "ATTN_ERR_BLOCK_TABLE", -9: "ATTN_ERR_SEQUENCE",
}

# (name, restype, argtypes) for every symbol declared in include/attn.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
SIGNATURES = [
    ("attn_encoder_fwd", _I, [_P, _P, _P, _P, _I, _I, _I, _I, _F, _P, _P]),
    ("attn_gqa_decode_workspace_size", _SZ, [_I, _I, _I, _I, _I]),
    ("attn_gqa_decode", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _SZ, _P]),
    ("attn_gqa_decode_noalloc", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    ("attn_paged_history", _I, [_P, _P, _P, _P, _I, _I, _I, _I, _F, _F, _F, _I, _I, _I, _I, _I,
                                _P, _P]),
    ("attn_paged_prefill", _I, [_P, _P, _P, _P, _I, _I, _I, _P, _P, _I, _I, _I, _F, _F, _F, _I, _I,
                                _I, _I, _P, _P]),
    ("attn_rope_qk", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    ("attn_qkv_rope_proj", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    ("attn_out_proj", _I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    ("attn_check", _I, [_P]),
    ("attn_status_string", ctypes.c_char_p, [_I]),
    ("attn_version", _I, []),
]


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status})")
        self.status = status


_lib = None
_lock = threading.Lock()


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and type the shared library. Raises if it is not built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is missing: build it with "
                    "`python -m online_softmax_attention_flash_b200.build` (no fallback exists)")
            lib = ctypes.CDLL(path)
            for name, res, args in SIGNATURES:
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _raise_if(status: int, where: str):
    if status != 0:
        raise AttnError(status, where)


def attn_check(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise the stream and return (and clear) the device-side status."""
    return int(load_library().attn_check(_stream_ptr(stream)))


def attn_version() -> int:
    return int(load_library().attn_version())


def attn_encoder_fwd(q, k, v, softmax_scale: float, key_bias=None, out=None, stream=None):
    """q, k, v: [B, H, S, D] bf16 CUDA tensors -> out [B, H, S, D] bf16."""
    lib = load_library()
    _need(q, "q", torch.bfloat16)
    B, H, S, D = q.shape
    _need(k, "k", torch.bfloat16, q.shape)
    _need(v, "v", torch.bfloat16, q.shape)
    if key_bias is not None:
        _need(key_bias, "key_bias", torch.float32, (B, S))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, q.shape)
    st = lib.attn_encoder_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, S, D,
                              float(softmax_scale), _ptr(key_bias), _stream_ptr(stream))
    _raise_if(st, "attn_encoder_fwd")
    return out


def attn_gqa_decode_workspace_size(B: int, Hq: int, Hkv: int, S_ctx: int, D: int) -> int:
    return int(load_library().attn_gqa_decode_workspace_size(B, Hq, Hkv, S_ctx, D))


def attn_gqa_decode(q, k, v, attn_mask, softmax_scale: float, num_kv_groups: int,
                    out=None, workspace=None, stream=None):
    """q [B, Hq, 1, D], k/v [B, Hkv, S_ctx, D] bf16, attn_mask [B, 1, 1, S_ctx] fp32 or None."""
    lib = load_library()
    _need(q, "q", torch.bfloat16)
    B, Hq, one, D = q.shape
    if one != 1:
        raise ValueError("q must be [B, Hq, 1, D] (single-token decode)")
    _need(k, "k", torch.bfloat16)
    Bk, Hkv, S_ctx, Dk = k.shape
    if Bk != B or Dk != D:
        raise ValueError("k must be [B, Hkv, S_ctx, D]")
    _need(v, "v", torch.bfloat16, k.shape)
    if attn_mask is not None:
        _need(attn_mask, "attn_mask", torch.float32, (B, 1, 1, S_ctx))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, q.shape)
    need = attn_gqa_decode_workspace_size(B, Hq, Hkv, S_ctx, D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace", torch.uint8)
    st = lib.attn_gqa_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(attn_mask), _ptr(out), B, Hq, Hkv,
                             int(num_kv_groups), S_ctx, D, float(softmax_scale), _ptr(workspace),
                             workspace.numel(), _stream_ptr(stream))
    _raise_if(st, "attn_gqa_decode")
    return out


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024  # ATTN_NOALLOC_SCRATCH_BYTES in include/attn.h


def attn_gqa_decode_noalloc(q, k, v, attn_mask, softmax_scale: float, num_kv_groups: int,
                            out=None, stream=None):
    """attn_gqa_decode without a caller workspace: the partials live in the
    library's static per-device scratch (for callers that cannot allocate).
    Calls that may overlap on the GPU share that scratch and race."""
    lib = load_library()
    _need(q, "q", torch.bfloat16)
    B, Hq, one, D = q.shape
    if one != 1:
        raise ValueError("q must be [B, Hq, 1, D] (single-token decode)")
    _need(k, "k", torch.bfloat16)
    Bk, Hkv, S_ctx, Dk = k.shape
    if Bk != B or Dk != D:
        raise ValueError("k must be [B, Hkv, S_ctx, D]")
    _need(v, "v", torch.bfloat16, k.shape)
    if attn_mask is not None:
        _need(attn_mask, "attn_mask", torch.float32, (B, 1, 1, S_ctx))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, q.shape)
    st = lib.attn_gqa_decode_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(attn_mask), _ptr(out), B,
                                     Hq, Hkv, int(num_kv_groups), S_ctx, D, float(softmax_scale),
                                     _stream_ptr(stream))
    _raise_if(st, "attn_gqa_decode_noalloc")
    return out


def attn_paged_history(q, k_cache, v_cache, block_table, block_size: int,
                       actual_history_len: int, k_scale: float, v_scale: float,
                       softmax_scale: float, num_kv_groups: int, out=None, stream=None):
    """q [Hq, Sq, D] bf16; k/v_cache [NB, Hkv, block_size, D] uint8 (E4M3FN codes);
    block_table [n_table] int32 -> out [Hq, Sq, D] bf16."""
    lib = load_library()
    _need(q, "q", torch.bfloat16)
    Hq, Sq, D = q.shape
    _need(k_cache, "k_cache", torch.uint8)
    NB, Hkv, BS, Dk = k_cache.shape
    if BS != block_size or Dk != D:
        raise ValueError("k_cache must be [num_phys_blocks, Hkv, block_size, D]")
    _need(v_cache, "v_cache", torch.uint8, k_cache.shape)
    _need(block_table, "block_table", torch.int32)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, q.shape)
    st = lib.attn_paged_history(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                block_table.numel(), NB, block_size, int(actual_history_len),
                                float(k_scale), float(v_scale), float(softmax_scale), Hq, Hkv,
                                int(num_kv_groups), Sq, D, _ptr(out), _stream_ptr(stream))
    _raise_if(st, "attn_paged_history")
    return out


def attn_paged_prefill(q, k_cache, v_cache, block_tables, q_start, hist_lens, k_scale: float,
                       v_scale: float, softmax_scale: float, num_kv_groups: int, max_q_len=None,
                       out=None, stream=None):
    """q [Hq, total_q, D] bf16 (current tokens of all sequences, packed); k/v_cache
    [NB, Hkv, block_size, D] uint8 codes holding history AND current tokens; block_tables
    [num_seqs, stride] int32; q_start [num_seqs + 1] int32; hist_lens [num_seqs] int32 (all
    CUDA). max_q_len: host bound on the sequences' current lengths (read from q_start on the
    host if None). Returns out [Hq, total_q, D] bf16."""
    lib = load_library()
    _need(q, "q", torch.bfloat16)
    Hq, total_q, D = q.shape
    _need(k_cache, "k_cache", torch.uint8)
    NB, Hkv, BS, Dk = k_cache.shape
    if Dk != D:
        raise ValueError("k_cache must be [num_phys_blocks, Hkv, block_size, D]")
    _need(v_cache, "v_cache", torch.uint8, k_cache.shape)
    _need(block_tables, "block_tables", torch.int32)
    if block_tables.dim() != 2:
        raise ValueError("block_tables must be [num_seqs, stride]")
    num_seqs, stride = block_tables.shape
    _need(q_start, "q_start", torch.int32, (num_seqs + 1,))
    _need(hist_lens, "hist_lens", torch.int32, (num_seqs,))
    if max_q_len is None:
        qs = q_start.cpu()
        max_q_len = int((qs[1:] - qs[:-1]).max()) if num_seqs > 0 else 0
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, q.shape)
    st = lib.attn_paged_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), stride, NB,
                                BS, _ptr(q_start), _ptr(hist_lens), num_seqs, total_q, int(max_q_len),
                                float(k_scale), float(v_scale), float(softmax_scale), Hq, Hkv,
                                int(num_kv_groups), D, _ptr(out), _stream_ptr(stream))
    _raise_if(st, "attn_paged_prefill")
    return out


def attn_rope_qk(q, k, cos_table, sin_table, interleaved: bool = False, q_out=None, k_out=None,
                 stream=None):
    """Rotary embedding of q and k ([B, H, S, D] bf16) with cos / sin tables [S, D/2] fp32.
    Returns (q_out, k_out); pass q_out=q, k_out=k to rotate in place."""
    lib = load_library()
    _need(q, "q", torch.bfloat16)
    B, H, S, D = q.shape
    _need(k, "k", torch.bfloat16, q.shape)
    _need(cos_table, "cos_table", torch.float32, (S, D // 2))
    _need(sin_table, "sin_table", torch.float32, (S, D // 2))
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    _need(q_out, "q_out", torch.bfloat16, q.shape)
    _need(k_out, "k_out", torch.bfloat16, q.shape)
    st = lib.attn_rope_qk(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), _ptr(cos_table),
                          _ptr(sin_table), B, H, S, D, 1 if interleaved else 0, _stream_ptr(stream))
    _raise_if(st, "attn_rope_qk")
    return q_out, k_out


def attn_qkv_rope_proj(x, w_qkv, b_qkv, H: int, D: int, cos_table=None, sin_table=None,
                       interleaved: bool = False, q=None, k=None, v=None, stream=None):
    """x [B, S, C] bf16, w_qkv [3 H D, C] bf16, b_qkv [3 H D] fp32 or None; optional RoPE
    tables [S, D/2] fp32. Returns (q, k, v), each [B, H, S, D] bf16, q and k rotated."""
    lib = load_library()
    _need(x, "x", torch.bfloat16)
    B, S, C = x.shape
    _need(w_qkv, "w_qkv", torch.bfloat16, (3 * H * D, C))
    if b_qkv is not None:
        _need(b_qkv, "b_qkv", torch.float32, (3 * H * D,))
    if (cos_table is None) != (sin_table is None):
        raise ValueError("pass both RoPE tables or neither")
    if cos_table is not None:
        _need(cos_table, "cos_table", torch.float32, (S, D // 2))
        _need(sin_table, "sin_table", torch.float32, (S, D // 2))
    shape = (B, H, S, D)
    q = torch.empty(shape, dtype=torch.bfloat16, device=x.device) if q is None else q
    k = torch.empty(shape, dtype=torch.bfloat16, device=x.device) if k is None else k
    v = torch.empty(shape, dtype=torch.bfloat16, device=x.device) if v is None else v
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, shape)
    st = lib.attn_qkv_rope_proj(_ptr(x), _ptr(w_qkv), _ptr(b_qkv), _ptr(cos_table),
                                _ptr(sin_table), 1 if interleaved else 0, B, S, C, H, D, _ptr(q),
                                _ptr(k), _ptr(v), _stream_ptr(stream))
    _raise_if(st, "attn_qkv_rope_proj")
    return q, k, v


def attn_out_proj(o, w_o, b_o=None, y=None, stream=None):
    """o [B, H, S, D] bf16, w_o [C_out, H D] bf16, b_o [C_out] fp32 or None -> y [B, S, C_out] fp32."""
    lib = load_library()
    _need(o, "o", torch.bfloat16)
    B, H, S, D = o.shape
    _need(w_o, "w_o", torch.bfloat16)
    C_out = w_o.shape[0]
    if w_o.dim() != 2 or w_o.shape[1] != H * D:
        raise ValueError("w_o must be [C_out, H * D]")
    if b_o is not None:
        _need(b_o, "b_o", torch.float32, (C_out,))
    y = torch.empty((B, S, C_out), dtype=torch.float32, device=o.device) if y is None else y
    _need(y, "y", torch.float32, (B, S, C_out))
    st = lib.attn_out_proj(_ptr(o), _ptr(w_o), _ptr(b_o), B, S, H, D, C_out, _ptr(y),
                           _stream_ptr(stream))
    _raise_if(st, "attn_out_proj")
    return y
