"""Thin ctypes binding of ``libtq_b200.so`` (declared in ``include/tq.h``).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels. Tensors are torch tensors (device memory and streams come from
PyTorch); their ``data_ptr()`` values and the current CUDA stream handle are
passed through unchanged. There is no CPU fallback: if the library is missing
the first call raises.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtq_b200.so")

TQ_OK = 0
TQ_ERR_INVALID_ARG = -1
TQ_ERR_UNSUPPORTED = -2
TQ_ERR_CAPACITY = -3
TQ_ERR_CUDA = -4

TQ_STATUS_NONFINITE = 1
TQ_STATUS_CAPACITY = 2
TQ_STATUS_TIMEOUT = 4

TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2

# cache formats: int4 K + V; binary16 K + int4 V; binary16 K + V hot tail folded into int4
TQ_K_INT4, TQ_K_FP16, TQ_KV_DELEGATED = 0, 1, 2

# C symbols declared in include/tq.h
EXPORTS = ("tq_cache_layout", "tq_cache_layout_kv", "tq_cache_layout_delegated", "tq_cache_layout_paged",
           "tq_cold_length", "tq_quantize_append", "tq_quantize_append_ex", "tq_quantize_append_paged",
           "tq_append_delegated", "tq_decode_attention", "tq_decode_attention_ex", "tq_decode_attention_delegated",
           "tq_decode_attention_paged", "tq_decode_attention_noalloc", "tq_dequantize_debug", "tq_status_string",
           "tq_last_cuda_error")

TQ_NOALLOC_WORKSPACE_BYTES = 8 << 20


class TqLayout(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("max_seq", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("group_size", ctypes.c_int32),
        ("n_groups", ctypes.c_int32), ("c_d", ctypes.c_float),
        ("sign_seed", ctypes.c_uint64), ("sign_bits", ctypes.c_uint64 * 4),
        ("code_stride_tok", ctypes.c_int64), ("code_stride_seq", ctypes.c_int64),
        ("scale_stride_tok", ctypes.c_int64), ("scale_stride_seq", ctypes.c_int64),
        ("codes_bytes", ctypes.c_uint64), ("scales_bytes", ctypes.c_uint64),
        ("decode_workspace_bytes", ctypes.c_uint64),
        ("max_ctas", ctypes.c_int32), ("k_format", ctypes.c_int32),
        ("k_bytes", ctypes.c_uint64), ("k_stride_tok", ctypes.c_int64), ("k_stride_seq", ctypes.c_int64),
        ("tail_window", ctypes.c_int32), ("fold_chunk", ctypes.c_int32), ("tail_bytes", ctypes.c_uint64),
        ("tail_stride_tok", ctypes.c_int64), ("tail_stride_seq", ctypes.c_int64),
        ("page_tokens", ctypes.c_int32), ("n_pages", ctypes.c_int32), ("max_pages", ctypes.c_int32),
        ("reserved_paged", ctypes.c_int32),
    ]


class TqDecodeOpts(ctypes.Structure):
    _fields_ = [("min_split_tokens", ctypes.c_int32), ("max_ctas", ctypes.c_int32),
                ("after_split_event", ctypes.c_void_p), ("lambda_k", ctypes.c_void_p),
                ("lambda_v", ctypes.c_void_p), ("sparse_v_threshold", ctypes.c_float),
                ("wait_limit_ns", ctypes.c_int64)]


class TqAppendOpts(ctypes.Structure):
    _fields_ = [("lambda_k", ctypes.c_void_p), ("lambda_v", ctypes.c_void_p)]


class TqError(RuntimeError):
    def __init__(self, fn, code):
        lib = _lib()
        msg = lib.tq_status_string(code).decode()
        extra = f" (cuda error {lib.tq_last_cuda_error()})" if code == TQ_ERR_CUDA else ""
        super().__init__(f"{fn} failed: {msg} [{code}]{extra}")
        self.code = code


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                              "(there is no CPU fallback for this library)")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64
        lib.tq_cache_layout.argtypes = [I, I, I, I, I, I, U64, ctypes.POINTER(TqLayout)]
        lib.tq_cache_layout.restype = I
        lib.tq_cache_layout_kv.argtypes = [I, I, I, I, I, I, U64, I, ctypes.POINTER(TqLayout)]
        lib.tq_cache_layout_kv.restype = I
        lib.tq_cache_layout_delegated.argtypes = [I, I, I, I, I, I, U64, I, I, ctypes.POINTER(TqLayout)]
        lib.tq_cache_layout_delegated.restype = I
        lib.tq_cold_length.argtypes = [ctypes.POINTER(TqLayout), ctypes.c_int64]
        lib.tq_cold_length.restype = ctypes.c_int64
        lib.tq_quantize_append.argtypes = [ctypes.POINTER(TqLayout), P, P, I, I, P, P, P, P, P, P, P]
        lib.tq_quantize_append.restype = I
        lib.tq_quantize_append_ex.argtypes = [ctypes.POINTER(TqLayout), P, P, I, I, P, P, P, P, P,
                                              ctypes.POINTER(TqAppendOpts), P, P]
        lib.tq_quantize_append_ex.restype = I
        lib.tq_cache_layout_paged.argtypes = [I, I, I, I, I, I, U64, I, I, I, ctypes.POINTER(TqLayout)]
        lib.tq_cache_layout_paged.restype = I
        lib.tq_quantize_append_paged.argtypes = [ctypes.POINTER(TqLayout), P, P, I, I, P, P, P, P, P, P,
                                                 ctypes.POINTER(TqAppendOpts), P, P]
        lib.tq_quantize_append_paged.restype = I
        lib.tq_decode_attention_paged.argtypes = [ctypes.POINTER(TqLayout), P, I, P, P, P, P, P, P, ctypes.c_float,
                                                  P, P, ctypes.c_size_t, P, ctypes.POINTER(TqDecodeOpts), P]
        lib.tq_decode_attention_paged.restype = I
        lib.tq_append_delegated.argtypes = [ctypes.POINTER(TqLayout), P, P, I, I, P, P, P, P, P, P, P]
        lib.tq_append_delegated.restype = I
        lib.tq_decode_attention_delegated.argtypes = [ctypes.POINTER(TqLayout), P, I, P, P, P, P, P,
                                                      ctypes.c_float, P, P, ctypes.c_size_t, P,
                                                      ctypes.POINTER(TqDecodeOpts), P]
        lib.tq_decode_attention_delegated.restype = I
        lib.tq_decode_attention.argtypes = [ctypes.POINTER(TqLayout), P, I, P, P, P, P, P, ctypes.c_float, P, P,
                                            ctypes.c_size_t, P, P]
        lib.tq_decode_attention.restype = I
        lib.tq_decode_attention_ex.argtypes = [ctypes.POINTER(TqLayout), P, I, P, P, P, P, P, ctypes.c_float, P, P,
                                               ctypes.c_size_t, P, ctypes.POINTER(TqDecodeOpts), P]
        lib.tq_decode_attention_ex.restype = I
        lib.tq_decode_attention_noalloc.argtypes = [ctypes.POINTER(TqLayout), P, I, P, P, P, P, P, ctypes.c_float,
                                                    P, P, P]
        lib.tq_decode_attention_noalloc.restype = I
        lib.tq_dequantize_debug.argtypes = [ctypes.POINTER(TqLayout), P, P, P, I, P, P]
        lib.tq_dequantize_debug.restype = I
        lib.tq_status_string.argtypes = [I]
        lib.tq_status_string.restype = ctypes.c_char_p
        lib.tq_last_cuda_error.argtypes = []
        lib.tq_last_cuda_error.restype = I
        _LIB = lib
    return _LIB


def _check(fn, code):
    if code != TQ_OK:
        raise TqError(fn, code)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    import torch
    return {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16, torch.float16: TQ_F16}[t.dtype]


def tq_cache_layout(batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size=32, sign_seed=0) -> TqLayout:
    out = TqLayout()
    _check("tq_cache_layout", _lib().tq_cache_layout(batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size,
                                                     ctypes.c_uint64(sign_seed), ctypes.byref(out)))
    return out


def tq_cache_layout_kv(batch, max_seq, n_kv_heads, n_q_heads, head_dim, k_format, group_size=32,
                       sign_seed=0) -> TqLayout:
    """Layout with the K storage format: TQ_K_INT4 (symmetric) or TQ_K_FP16 (binary16 K, int4 V)."""
    out = TqLayout()
    _check("tq_cache_layout_kv", _lib().tq_cache_layout_kv(batch, max_seq, n_kv_heads, n_q_heads, head_dim,
                                                           group_size, ctypes.c_uint64(sign_seed), int(k_format),
                                                           ctypes.byref(out)))
    return out


def tq_cache_layout_delegated(batch, max_seq, n_kv_heads, n_q_heads, head_dim, tail_window, fold_chunk,
                              group_size=32, sign_seed=0) -> TqLayout:
    """Delegated hot/cold cache: binary16 K; V in a binary16 tail of tail_window tokens, folded into int4
    fold_chunk tokens at a time."""
    out = TqLayout()
    _check("tq_cache_layout_delegated", _lib().tq_cache_layout_delegated(
        batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size, ctypes.c_uint64(sign_seed), int(tail_window),
        int(fold_chunk), ctypes.byref(out)))
    return out


def tq_cache_layout_paged(batch, max_seq, n_kv_heads, n_q_heads, head_dim, k_format, page_tokens, n_pages,
                          group_size=32, sign_seed=0) -> TqLayout:
    """Paged storage: pools of n_pages pages of page_tokens tokens, addressed through a block table."""
    out = TqLayout()
    _check("tq_cache_layout_paged", _lib().tq_cache_layout_paged(
        batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size, ctypes.c_uint64(sign_seed), int(k_format),
        int(page_tokens), int(n_pages), ctypes.byref(out)))
    return out


def tq_quantize_append_paged(layout, k, v, n_new, start_pos, block_table, k_codes, k_scales, v_codes, v_scales,
                             status=None, stream=None, lambda_k=None, lambda_v=None):
    """Append through the block table (int32 [batch][max_pages] on the device)."""
    for t in (k, v, start_pos, block_table, k_codes, k_scales, v_codes, v_scales, lambda_k, lambda_v):
        assert t is None or t.is_contiguous()
    opts = TqAppendOpts(_ptr(lambda_k), _ptr(lambda_v)) if (lambda_k is not None or lambda_v is not None) else None
    code = _lib().tq_quantize_append_paged(ctypes.byref(layout), _ptr(k), _ptr(v), _dtype_code(k), int(n_new),
                                           _ptr(start_pos), _ptr(block_table), _ptr(k_codes), _ptr(k_scales),
                                           _ptr(v_codes), _ptr(v_scales),
                                           ctypes.byref(opts) if opts is not None else None, _ptr(status),
                                           _stream(stream))
    _check("tq_quantize_append_paged", code)


def tq_decode_attention_paged(layout, q, seq_lens, block_table, k_codes, k_scales, v_codes, v_scales, sm_scale, out,
                              workspace, status=None, stream=None, min_split_tokens=0, max_ctas=0,
                              after_split_event=None, lambda_k=None, lambda_v=None, sparse_v_threshold=0.0):
    """Decode over a paged cache through the block table."""
    for t in (q, seq_lens, block_table, k_codes, k_scales, v_codes, v_scales, out, workspace):
        assert t is None or t.is_contiguous()
    ws_bytes = workspace.numel() * workspace.element_size()
    opts = _decode_opts(min_split_tokens, max_ctas, after_split_event, lambda_k, lambda_v, sparse_v_threshold)
    code = _lib().tq_decode_attention_paged(
        ctypes.byref(layout), _ptr(q), _dtype_code(q), _ptr(seq_lens), _ptr(block_table), _ptr(k_codes),
        _ptr(k_scales), _ptr(v_codes), _ptr(v_scales), ctypes.c_float(sm_scale), _ptr(out), _ptr(workspace),
        ws_bytes, _ptr(status), ctypes.byref(opts) if opts is not None else None, _stream(stream))
    _check("tq_decode_attention_paged", code)


def tq_cold_length(layout, length) -> int:
    """Tokens of a sequence of `length` tokens held as int4 codes (all of them outside the delegated cache)."""
    return int(_lib().tq_cold_length(ctypes.byref(layout), int(length)))


def tq_cache_layout_status(batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size=32, sign_seed=0):
    """Raw status code variant (for callers that test rejection paths)."""
    out = TqLayout()
    code = _lib().tq_cache_layout(batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size,
                                  ctypes.c_uint64(sign_seed), ctypes.byref(out))
    return code, out


def tq_quantize_append(layout, k, v, n_new, start_pos, k_codes, k_scales, v_codes, v_scales, status=None,
                       stream=None, lambda_k=None, lambda_v=None):
    """k, v: [batch][n_new][Hkv][D] (f32/bf16/f16, CUDA, contiguous); start_pos: int32 [batch] on the device.

    lambda_k / lambda_v: optional float32 [D] device vectors (per-channel lambda, tq_quantize_append_ex).
    """
    for t in (k, v, start_pos, k_codes, k_scales, v_codes, v_scales, lambda_k, lambda_v):
        assert t is None or t.is_contiguous()
    if lambda_k is None and lambda_v is None:
        code = _lib().tq_quantize_append(ctypes.byref(layout), _ptr(k), _ptr(v), _dtype_code(k), int(n_new),
                                         _ptr(start_pos), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes),
                                         _ptr(v_scales), _ptr(status), _stream(stream))
        _check("tq_quantize_append", code)
        return
    opts = TqAppendOpts(_ptr(lambda_k), _ptr(lambda_v))
    code = _lib().tq_quantize_append_ex(ctypes.byref(layout), _ptr(k), _ptr(v), _dtype_code(k), int(n_new),
                                        _ptr(start_pos), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes),
                                        _ptr(v_scales), ctypes.byref(opts), _ptr(status), _stream(stream))
    _check("tq_quantize_append_ex", code)


def tq_append_delegated(layout, k, v, n_new, start_pos, k_f16, v_codes, v_scales, v_tail, status=None,
                        stream=None):
    """Delegated-cache append. start_pos[b] must be sequence b's current length."""
    for t in (k, v, start_pos, k_f16, v_codes, v_scales, v_tail):
        assert t is None or t.is_contiguous()
    code = _lib().tq_append_delegated(ctypes.byref(layout), _ptr(k), _ptr(v), _dtype_code(k), int(n_new),
                                      _ptr(start_pos), _ptr(k_f16), _ptr(v_codes), _ptr(v_scales), _ptr(v_tail),
                                      _ptr(status), _stream(stream))
    _check("tq_append_delegated", code)


def _decode_opts(min_split_tokens, max_ctas, after_split_event, lambda_k=None, lambda_v=None,
                 sparse_v_threshold=0.0, wait_limit_ns=0):
    """TqDecodeOpts for the given knobs, or None when all are at their defaults."""
    if not (min_split_tokens or max_ctas or after_split_event is not None or lambda_k is not None
            or lambda_v is not None or sparse_v_threshold or wait_limit_ns):
        return None
    for t in (lambda_k, lambda_v):
        assert t is None or t.is_contiguous()
    ev = ctypes.c_void_p(after_split_event.cuda_event) if after_split_event is not None else None
    return TqDecodeOpts(int(min_split_tokens), int(max_ctas), ev, _ptr(lambda_k), _ptr(lambda_v),
                        float(sparse_v_threshold), int(wait_limit_ns))


def tq_decode_attention_delegated(layout, q, seq_lens, k_f16, v_codes, v_scales, v_tail, sm_scale, out, workspace,
                                  status=None, stream=None, min_split_tokens=0, max_ctas=0, after_split_event=None,
                                  sparse_v_threshold=0.0):
    """Decode over a delegated cache: the cold tokens through the split-K kernel, the hot tail in the merge."""
    for t in (q, seq_lens, k_f16, v_codes, v_scales, v_tail, out, workspace):
        assert t is None or t.is_contiguous()
    ws_bytes = workspace.numel() * workspace.element_size()
    opts = _decode_opts(min_split_tokens, max_ctas, after_split_event, sparse_v_threshold=sparse_v_threshold)
    code = _lib().tq_decode_attention_delegated(
        ctypes.byref(layout), _ptr(q), _dtype_code(q), _ptr(seq_lens), _ptr(k_f16), _ptr(v_codes), _ptr(v_scales),
        _ptr(v_tail), ctypes.c_float(sm_scale), _ptr(out), _ptr(workspace), ws_bytes, _ptr(status),
        ctypes.byref(opts) if opts is not None else None, _stream(stream))
    _check("tq_decode_attention_delegated", code)


def tq_decode_attention(layout, q, seq_lens, k_codes, k_scales, v_codes, v_scales, sm_scale, out, workspace,
                        status=None, stream=None, min_split_tokens=0, max_ctas=0, after_split_event=None,
                        lambda_k=None, lambda_v=None, sparse_v_threshold=0.0, wait_limit_ns=0):
    """q: [batch][Hq][D]; out: float32 [batch][Hq][D]; workspace: >= layout.decode_workspace_bytes bytes.

    lambda_k / lambda_v: the per-channel lambda the cache was written with; sparse_v_threshold: the
    sparse-V rule's threshold (0 = exact); wait_limit_ns: bound on each pipeline wait of the split-K
    kernel (0 = one second). Any of these selects tq_decode_attention_ex.
    """
    for t in (q, seq_lens, k_codes, k_scales, v_codes, v_scales, out, workspace):
        assert t is None or t.is_contiguous()
    ws_bytes = workspace.numel() * workspace.element_size()
    lib = _lib()
    opts = _decode_opts(min_split_tokens, max_ctas, after_split_event, lambda_k, lambda_v, sparse_v_threshold,
                        wait_limit_ns)
    if opts is not None:
        code = lib.tq_decode_attention_ex(ctypes.byref(layout), _ptr(q), _dtype_code(q), _ptr(seq_lens),
                                          _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales),
                                          ctypes.c_float(sm_scale), _ptr(out), _ptr(workspace), ws_bytes,
                                          _ptr(status), ctypes.byref(opts), _stream(stream))
    else:
        code = lib.tq_decode_attention(ctypes.byref(layout), _ptr(q), _dtype_code(q), _ptr(seq_lens),
                                       _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales),
                                       ctypes.c_float(sm_scale), _ptr(out), _ptr(workspace), ws_bytes,
                                       _ptr(status), _stream(stream))
    _check("tq_decode_attention", code)


def tq_decode_attention_noalloc(layout, q, seq_lens, k_codes, k_scales, v_codes, v_scales, sm_scale, out,
                                status=None, stream=None):
    """Decode without a caller workspace, for callers that cannot allocate device memory.

    The split-K scratch comes from a fixed array inside the library's device
    image (TQ_NOALLOC_WORKSPACE_BYTES per GPU), so nothing is allocated here.
    Calls on one device share that array: do not let two of them overlap on
    the GPU. Raises TqError (TQ_ERR_CAPACITY) when the request needs more
    scratch than the array holds.
    """
    for t in (q, seq_lens, k_codes, k_scales, v_codes, v_scales, out):
        assert t is None or t.is_contiguous()
    code = _lib().tq_decode_attention_noalloc(ctypes.byref(layout), _ptr(q), _dtype_code(q), _ptr(seq_lens),
                                              _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales),
                                              ctypes.c_float(sm_scale), _ptr(out), _ptr(status), _stream(stream))
    _check("tq_decode_attention_noalloc", code)


def tq_dequantize_debug(layout, codes, scales, seq_lens, original_domain, out, stream=None):
    code = _lib().tq_dequantize_debug(ctypes.byref(layout), _ptr(codes), _ptr(scales), _ptr(seq_lens),
                                      1 if original_domain else 0, _ptr(out), _stream(stream))
    _check("tq_dequantize_debug", code)


def sign_vector(layout):
    """The layout's +-1 diagonal as a Python list of floats (read from its sign bits)."""
    return [(-1.0 if (layout.sign_bits[i >> 6] >> (i & 63)) & 1 else 1.0) for i in range(layout.head_dim)]


def alloc_cache(layout, device="cuda"):
    """Allocate (k_codes, k_scales, v_codes, v_scales) with the layout's sizes (zero-filled).

    With layout.k_format == TQ_K_FP16 or TQ_KV_DELEGATED, k_codes is the binary16 K buffer
    (k_bytes) and k_scales is None; the delegated cache's V tail comes from alloc_tail.
    """
    import torch
    cb = int(layout.codes_bytes)
    sb = int(layout.scales_bytes)
    k_codes = torch.zeros(int(layout.k_bytes), dtype=torch.uint8, device=device)
    v_codes = torch.zeros(cb, dtype=torch.uint8, device=device)
    if layout.k_format != TQ_K_INT4:
        k_scales = None
    else:
        k_scales = torch.zeros((sb + 1) // 2, dtype=torch.int16, device=device)
    v_scales = torch.zeros((sb + 1) // 2, dtype=torch.int16, device=device)
    return k_codes, k_scales, v_codes, v_scales


def alloc_tail(layout, device="cuda"):
    """The delegated cache's binary16 V tail [batch][tail_window][Hkv][D] as int16 bits (zero-filled)."""
    import torch
    return torch.zeros(int(layout.tail_bytes) // 2, dtype=torch.int16, device=device)


def alloc_workspace(layout, device="cuda"):
    import torch
    return torch.empty(int(layout.decode_workspace_bytes), dtype=torch.uint8, device=device)
