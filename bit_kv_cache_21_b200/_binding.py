"""ctypes binding of libkvq.so: argument marshalling only.

Every computation runs in the library's CUDA kernels; this module turns torch
tensors into pointers and the current CUDA stream into a handle, and raises
KvqError on a non-zero status. It fails loudly when libkvq.so is missing.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libkvq.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "kvq.h")

# kvq_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_TIMEOUT, ERR_CUDA = range(6)
# device status bits
DEV_CAPACITY, DEV_TIMEOUT, DEV_SEQLEN = 0x1, 0x2, 0x4
# kvq_dtype
BF16, FP16, FP32 = 0, 1, 2
# kvq_axis
PER_TOKEN, PER_CHANNEL = 0, 1
# debug hooks
DEBUG_WAIT_TIMEOUT_NS, DEBUG_SKIP_TILE = 1, 2


class KvqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, status_string(status), status))


class CacheDesc(ctypes.Structure):
    """Mirror of kvq_cache_desc (include/kvq.h)."""
    _fields_ = [
        ("num_seqs", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("bits_k", ctypes.c_int32),
        ("bits_v", ctypes.c_int32),
        ("group_k", ctypes.c_int32),
        ("group_v", ctypes.c_int32),
        ("axis_k", ctypes.c_int32),
        ("axis_v", ctypes.c_int32),
        ("hadamard_block_k", ctypes.c_int32),
        ("residual_len", ctypes.c_int32),
        ("paged", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("capacity_tokens", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("k_codes", ctypes.c_void_p),
        ("v_codes", ctypes.c_void_p),
        ("k_sz", ctypes.c_void_p),
        ("v_sz", ctypes.c_void_p),
        ("k_res", ctypes.c_void_p),
        ("v_res", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("status", ctypes.c_void_p),
        ("hadamard_signs", ctypes.c_void_p),
        ("k_sink", ctypes.c_void_p),
        ("v_sink", ctypes.c_void_p),
        ("sink_len", ctypes.c_int32),
        ("hybrid", ctypes.c_int32),
    ]


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_S = ctypes.c_size_t
_DESC = ctypes.POINTER(CacheDesc)

_SIGNATURES = {
    "kvq_quantize_append": (_I, [_DESC, _P, _P, _I, _P, _P, _I, _I, _P]),
    "kvq_decode_workspace_size": (_S, [_DESC, _I, _I, _I]),
    "kvq_decode_attention": (_I, [_DESC, _P, _I, _I, _P, _I, _I, ctypes.c_float, _P, _P, _S, _P]),
    "kvq_decode_splitk": (_I, [_DESC, _P, _I, _I, _P, _I, _I, ctypes.c_float, _P, _S, _P]),
    "kvq_decode_attention_static": (_I, [_DESC, _P, _I, _I, _P, _I, _I, ctypes.c_float, _P, _P]),
    "kvq_decode_merge": (_I, [_DESC, _I, _P, _I, _I, _P, _P, _S, _P]),
    "kvq_decode_merge_partial": (_I, [_DESC, _I, _P, _I, _I, _P, _P, _P, _S, _P]),
    "kvq_merge_partials": (_I, [_P, _I, _I, _I, _P, _P]),
    "kvq_remat_kv": (_I, [_DESC, _P, _I, _P, _P, _I, _I, _P, _P, _P]),
    "kvq_rope_tables": (_I, [_P, _P, _I, _I, ctypes.c_double, _P]),
    "kvq_remat_attention_workspace_size": (_S, [_I, _I, _I]),
    "kvq_remat_attention": (_I, [_DESC, _P, _I, _P, _P, _I, _I, _P, _I, _I, ctypes.c_float, _P, _P, _S, _P]),
    "kvq_status_string": (ctypes.c_char_p, [_I]),
    "kvq_debug_set": (_I, [_I, ctypes.c_int64]),
    "kvq_version": (_I, []),
}


def lib():
    """The loaded libkvq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libkvq.so not found at %s; build it with "
                              "`python -m bit_kv_cache_21_b200.build`" % LIB_PATH)
        _lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(_lib, name)
            fn.restype = res
            fn.argtypes = args
    return _lib


def header_symbols():
    """Names of the functions include/kvq.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^KVQ_API\s+[^(;]*?\b(kvq_\w+)\s*\(", text, re.M)))


def status_string(status: int) -> str:
    try:
        return lib().kvq_status_string(status).decode()
    except Exception:  # pragma: no cover
        return "status"


def check(status: int, what: str) -> None:
    if status != OK:
        raise KvqError(status, what)


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def dtype_code(t) -> int:
    import torch
    codes = {torch.bfloat16: BF16, torch.float16: FP16, torch.float32: FP32}
    if t.dtype not in codes:
        raise TypeError("unsupported dtype %s" % t.dtype)
    return codes[t.dtype]


def _require(t, name, dtype=None):
    if t is None:
        raise ValueError("%s is required" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s" % (name, dtype))


def quantize_append(desc: CacheDesc, k_new, v_new, cu_new, seq_lens, stream=None) -> None:
    """kvq_quantize_append: k_new/v_new [N][H][128] (bf16/fp16/fp32), cu_new
    int32 [S+1], seq_lens int32 [S] (advanced in place)."""
    import torch
    _require(k_new, "k_new")
    if v_new is not None:
        _require(v_new, "v_new", k_new.dtype)
    _require(cu_new, "cu_new", torch.int32)
    _require(seq_lens, "seq_lens", torch.int32)
    num_seqs = seq_lens.numel()
    total = k_new.shape[0]
    st = lib().kvq_quantize_append(ctypes.byref(desc), _ptr(k_new), _ptr(v_new), dtype_code(k_new),
                                   _ptr(cu_new), _ptr(seq_lens), num_seqs, total,
                                   _stream_handle(stream))
    check(st, "kvq_quantize_append")


def decode_workspace_size(desc: CacheDesc, num_seqs: int, num_q_heads: int, max_seq_len: int) -> int:
    return int(lib().kvq_decode_workspace_size(ctypes.byref(desc), num_seqs, num_q_heads, max_seq_len))


def _decode_common(desc, q, seq_lens, max_seq_len, workspace):
    import torch
    _require(q, "q")
    _require(seq_lens, "seq_lens", torch.int32)
    num_seqs, num_q_heads = q.shape[0], q.shape[1]
    need = decode_workspace_size(desc, num_seqs, num_q_heads, max_seq_len)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    return num_seqs, num_q_heads, workspace


def decode_attention(desc: CacheDesc, q, seq_lens, max_seq_len: int, softmax_scale: float,
                     out=None, workspace=None, stream=None):
    """kvq_decode_attention: q [S][Hq][128] -> out fp32 [S][Hq][128]."""
    import torch
    num_seqs, num_q_heads, workspace = _decode_common(desc, q, seq_lens, max_seq_len, workspace)
    if out is None:
        out = torch.empty((num_seqs, num_q_heads, 128), dtype=torch.float32, device=q.device)
    _require(out, "out", torch.float32)
    st = lib().kvq_decode_attention(ctypes.byref(desc), _ptr(q), dtype_code(q), num_q_heads,
                                    _ptr(seq_lens), num_seqs, max_seq_len, float(softmax_scale),
                                    _ptr(out), _ptr(workspace), workspace.numel(),
                                    _stream_handle(stream))
    check(st, "kvq_decode_attention")
    return out


def decode_attention_static(desc: CacheDesc, q, seq_lens, max_seq_len: int, softmax_scale: float,
                            out=None, stream=None):
    """kvq_decode_attention_static: decode attention with the library's fixed
    device workspace, for callers that cannot allocate one."""
    import torch
    _require(q, "q")
    _require(seq_lens, "seq_lens", torch.int32)
    num_seqs, num_q_heads = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty((num_seqs, num_q_heads, 128), dtype=torch.float32, device=q.device)
    _require(out, "out", torch.float32)
    st = lib().kvq_decode_attention_static(ctypes.byref(desc), _ptr(q), dtype_code(q), num_q_heads,
                                           _ptr(seq_lens), num_seqs, max_seq_len,
                                           float(softmax_scale), _ptr(out), _stream_handle(stream))
    check(st, "kvq_decode_attention_static")
    return out


def decode_splitk(desc: CacheDesc, q, seq_lens, max_seq_len: int, softmax_scale: float,
                  workspace, stream=None) -> None:
    st = lib().kvq_decode_splitk(ctypes.byref(desc), _ptr(q), dtype_code(q), q.shape[1],
                                 _ptr(seq_lens), q.shape[0], max_seq_len, float(softmax_scale),
                                 _ptr(workspace), workspace.numel(), _stream_handle(stream))
    check(st, "kvq_decode_splitk")


def decode_merge(desc: CacheDesc, num_q_heads: int, seq_lens, max_seq_len: int, out, workspace,
                 stream=None) -> None:
    st = lib().kvq_decode_merge(ctypes.byref(desc), num_q_heads, _ptr(seq_lens), out.shape[0],
                                max_seq_len, _ptr(out), _ptr(workspace), workspace.numel(),
                                _stream_handle(stream))
    check(st, "kvq_decode_merge")


def decode_merge_partial(desc: CacheDesc, num_q_heads: int, seq_lens, max_seq_len: int, o_part, ml,
                         workspace, stream=None) -> None:
    """kvq_decode_merge_partial: this cache's unnormalized partial o_part fp32
    [S][Hq][128] and its (m, l) pairs ml fp32 [S][Hq][2]."""
    import torch
    for t, name in ((o_part, "o_part"), (ml, "ml")):
        if t is None or not t.is_cuda or t.dtype != torch.float32:
            raise ValueError("%s must be a CUDA fp32 tensor" % name)
    st = lib().kvq_decode_merge_partial(ctypes.byref(desc), num_q_heads, _ptr(seq_lens), o_part.shape[0],
                                        max_seq_len, _ptr(o_part), _ptr(ml), _ptr(workspace),
                                        workspace.numel(), _stream_handle(stream))
    check(st, "kvq_decode_merge_partial")


def partial_buffer(num_seqs: int, num_q_heads: int, device, n_part: int = 1):
    """fp32 [n_part][S*Hq*130]: per part the o rows [S][Hq][128], then the
    (m, l) pairs [S][Hq][2] (the layout kvq_merge_partials reads)."""
    import torch
    return torch.empty((n_part, num_seqs * num_q_heads * 130), dtype=torch.float32, device=device)


def partial_views(buf, num_seqs: int, num_q_heads: int):
    """o_part [S][Hq][128] and ml [S][Hq][2] views of one part of partial_buffer."""
    rows = num_seqs * num_q_heads
    return buf[:rows * 128].view(num_seqs, num_q_heads, 128), buf[rows * 128:].view(num_seqs, num_q_heads, 2)


def merge_partials(parts, num_seqs: int, num_q_heads: int, out=None, stream=None):
    """kvq_merge_partials: parts fp32 [n_part][S*Hq*130] (partial_buffer's
    layout) -> out fp32 [S][Hq][128]."""
    import torch
    _require(parts, "parts", torch.float32)
    if parts.dim() != 2 or parts.shape[1] != num_seqs * num_q_heads * 130:
        raise ValueError("parts must be [n_part][num_seqs * num_q_heads * 130]")
    if out is None:
        out = torch.empty((num_seqs, num_q_heads, 128), dtype=torch.float32, device=parts.device)
    _require(out, "out", torch.float32)
    st = lib().kvq_merge_partials(_ptr(parts), parts.shape[0], num_seqs, num_q_heads, _ptr(out),
                                  _stream_handle(stream))
    check(st, "kvq_merge_partials")
    return out


def remat_kv(x_desc: CacheDesc, w_kv, n_kv_heads: int, rope_cos, rope_sin, batch: int,
             ctx_len: int, k_out, v_out, stream=None) -> None:
    """kvq_remat_kv: K, V bf16 [B][H][ctx_len][128] from the quantized X cache."""
    import torch
    _require(w_kv, "w_kv", torch.bfloat16)
    _require(rope_cos, "rope_cos", torch.float32)
    _require(rope_sin, "rope_sin", torch.float32)
    _require(k_out, "k_out", torch.bfloat16)
    _require(v_out, "v_out", torch.bfloat16)
    st = lib().kvq_remat_kv(ctypes.byref(x_desc), _ptr(w_kv), n_kv_heads, _ptr(rope_cos),
                            _ptr(rope_sin), batch, ctx_len, _ptr(k_out), _ptr(v_out),
                            _stream_handle(stream))
    check(st, "kvq_remat_kv")


def remat_attention(x_desc: CacheDesc, w_kv, n_kv_heads: int, rope_cos, rope_sin, batch: int,
                    ctx_len: int, q, softmax_scale: float, out=None, workspace=None, stream=None):
    """kvq_remat_attention: decode attention of q [batch][Hq][128] over K, V
    rematerialized from the X cache on the fly -> out fp32 [batch][Hq][128]."""
    import torch
    _require(w_kv, "w_kv", torch.bfloat16)
    _require(q, "q")
    num_q_heads = q.shape[1]
    if workspace is None:
        need = int(lib().kvq_remat_attention_workspace_size(batch, num_q_heads, ctx_len))
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((batch, num_q_heads, 128), dtype=torch.float32, device=q.device)
    _require(out, "out", torch.float32)
    st = lib().kvq_remat_attention(ctypes.byref(x_desc), _ptr(w_kv), n_kv_heads, _ptr(rope_cos), _ptr(rope_sin),
                                   batch, ctx_len, _ptr(q), dtype_code(q), num_q_heads, float(softmax_scale),
                                   _ptr(out), _ptr(workspace), workspace.numel(), _stream_handle(stream))
    check(st, "kvq_remat_attention")
    return out


def rope_tables(n_pos: int, head_dim: int = 128, theta: float = 500000.0, device="cuda", stream=None):
    """kvq_rope_tables: (cos, sin) fp32 [n_pos][head_dim/2]."""
    import torch
    c = torch.empty((n_pos, head_dim // 2), dtype=torch.float32, device=device)
    s = torch.empty_like(c)
    st = lib().kvq_rope_tables(_ptr(c), _ptr(s), n_pos, head_dim, float(theta), _stream_handle(stream))
    check(st, "kvq_rope_tables")
    return c, s


def debug_set(what: int, value: int) -> None:
    check(lib().kvq_debug_set(what, int(value)), "kvq_debug_set")


def version() -> int:
    return int(lib().kvq_version())
