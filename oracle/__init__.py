"""CPU oracle for SRHT + per-group int4 KV quantisation and decode attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package. The
product library (``compressed_domain_attention_b200``) never imports, loads or
calls it, and the two share no code: the oracle is a plain single-threaded C++
file (``tq_oracle.cpp``) reached through ctypes, with numpy arrays in and out.

What each function computes, and the page passage it follows, is documented in
``tq_oracle.cpp``. Parity pins live in ``tests/test_oracle_pins.py``; the sign
vector's generator convention is the one part with no pin ("parity unpinned":
any seeded +-1 diagonal is equally correct).
"""
import ctypes
import os

import numpy as np

from .build import LIB, build_oracle

STATUS_NONFINITE = 1
STATUS_CAPACITY = 2

_lib = None


def _signatures():
    P = ctypes.c_void_p
    i32, i64, u64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float
    return {
        "oracle_status_nonfinite": ([], i32),
        "oracle_status_capacity": ([], i32),
        "oracle_splitmix64": ([u64, ctypes.c_int, P], None),
        "oracle_sign_vector": ([u64, ctypes.c_int, P], None),
        "oracle_norm_const": ([ctypes.c_int], f32),
        "oracle_f32_to_f16": ([P, i64, P], None),
        "oracle_f16_to_f32": ([P, i64, P], None),
        "oracle_fwht": ([P, ctypes.c_int, i64], None),
        "oracle_srht_forward": ([P, P, ctypes.c_int, i64, P], None),
        "oracle_srht_inverse": ([P, P, ctypes.c_int, i64, P], None),
        "oracle_quantize_rotated": ([P, ctypes.c_int, i64, P, P], i32),
        "oracle_pack": ([P, ctypes.c_int, i64, P], None),
        "oracle_unpack": ([P, ctypes.c_int, i64, P], None),
        "oracle_encode": ([P, P, ctypes.c_int, i64, P, P], i32),
        "oracle_quantize_append": ([ctypes.c_int] * 4 + [P, P, P, ctypes.c_int, P, P, P, P, P], i32),
        "oracle_decode_attention": ([ctypes.c_int] * 5 + [P, P, P, P, P, P, P, f32, P, P], i32),
        "oracle_dequantize": ([ctypes.c_int] * 4 + [P, P, P, P, ctypes.c_int, P], i32),
        "oracle_quantize_append_kf16": ([ctypes.c_int] * 4 + [P, P, P, ctypes.c_int, P, P, P, P], i32),
        "oracle_decode_attention_kf16": ([ctypes.c_int] * 5 + [P, P, P, P, P, P, f32, P, P], i32),
        "oracle_cold_length": ([i64, ctypes.c_int, ctypes.c_int], i64),
        "oracle_encode_lambda": ([P, P, P, ctypes.c_int, i64, P, P], i32),
        "oracle_quantize_append_paged": ([ctypes.c_int] * 4 + [P, P, P, ctypes.c_int, P, P] + [ctypes.c_int] * 3
                                         + [P] * 5, i32),
        "oracle_decode_attention_paged": ([ctypes.c_int] * 5 + [P, P, P, P] + [ctypes.c_int] * 3 + [P] * 5
                                          + [f32, P, P], i32),
        "oracle_quantize_append_lambda": ([ctypes.c_int] * 4 + [P, P, P, ctypes.c_int, P, P, P, P, P, P, P], i32),
        "oracle_decode_attention_ext": ([ctypes.c_int] * 5 + [P] * 10 + [f32, ctypes.c_double, P, P, P], i32),
        "oracle_append_delegated": ([ctypes.c_int] * 4 + [P, P, P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int,
                                                          P, P, P, P], i32),
        "oracle_decode_attention_delegated": ([ctypes.c_int] * 5 + [P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                                                    f32, P, P], i32),
    }


def bind(lib):
    """Attach argument/result types to a loaded oracle library (the built one, or a test's variant)."""
    for name, (args, res) in _signatures().items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    assert lib.oracle_status_nonfinite() == STATUS_NONFINITE
    assert lib.oracle_status_capacity() == STATUS_CAPACITY
    return lib


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            build_oracle()
        _lib = bind(ctypes.CDLL(LIB))
    return _lib


def _c(a, dtype):
    """Contiguous array of the exact dtype (copies only if needed)."""
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def splitmix64(seed: int, n: int) -> np.ndarray:
    out = np.empty(n, np.uint64)
    _load().oracle_splitmix64(ctypes.c_uint64(seed), n, _p(out))
    return out


def sign_vector(seed: int, D: int) -> np.ndarray:
    out = np.empty(D, np.float32)
    _load().oracle_sign_vector(ctypes.c_uint64(seed), D, _p(out))
    return out


def norm_const(D: int) -> np.float32:
    return np.float32(_load().oracle_norm_const(D))


def f32_to_f16_bits(x) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().oracle_f32_to_f16(_p(x), x.size, _p(out))
    return out


def f16_bits_to_f32(h) -> np.ndarray:
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    _load().oracle_f16_to_f32(_p(h), h.size, _p(out))
    return out


def fwht(x) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform along the last axis (binary32)."""
    u = _c(x, np.float32).copy()
    D = u.shape[-1]
    _load().oracle_fwht(_p(u), D, u.size // D)
    return u


def srht_forward(x, signs) -> np.ndarray:
    x = _c(x, np.float32)
    s = _c(signs, np.float32)
    D = x.shape[-1]
    y = np.empty_like(x)
    _load().oracle_srht_forward(_p(x), _p(s), D, x.size // D, _p(y))
    return y


def srht_inverse(y, signs) -> np.ndarray:
    y = _c(y, np.float32)
    s = _c(signs, np.float32)
    D = y.shape[-1]
    x = np.empty_like(y)
    _load().oracle_srht_inverse(_p(y), _p(s), D, y.size // D, _p(x))
    return x


def quantize_rotated(y):
    """Per-group abs-max int4 of rotated vectors -> (codes int8 [...,D], scale bits uint16 [...,D/32], status)."""
    y = _c(y, np.float32)
    D = y.shape[-1]
    codes = np.empty(y.shape, np.int8)
    scales = np.empty(y.shape[:-1] + (D // 32,), np.uint16)
    st = _load().oracle_quantize_rotated(_p(y), D, y.size // D, _p(codes), _p(scales))
    return codes, scales, int(st)


def pack(codes) -> np.ndarray:
    codes = _c(codes, np.int8)
    D = codes.shape[-1]
    out = np.empty(codes.shape[:-1] + (D // 2,), np.uint8)
    _load().oracle_pack(_p(codes), D, codes.size // D, _p(out))
    return out


def unpack(packed, D: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    out = np.empty(packed.shape[:-1] + (D,), np.int8)
    _load().oracle_unpack(_p(packed), D, packed.size // (D // 2), _p(out))
    return out


def encode(x, signs):
    """SRHT + quantise + pack raw vectors -> (packed uint8 [...,D/2], scale bits [...,D/32], status)."""
    x = _c(x, np.float32)
    s = _c(signs, np.float32)
    D = x.shape[-1]
    packed = np.empty(x.shape[:-1] + (D // 2,), np.uint8)
    scales = np.empty(x.shape[:-1] + (D // 32,), np.uint16)
    st = _load().oracle_encode(_p(x), _p(s), D, x.size // D, _p(packed), _p(scales))
    return packed, scales, int(st)


def new_cache(batch, max_seq, n_kv, D):
    """Zeroed host cache arrays (codes [B][S][Hkv][D/2] uint8, scales [B][S][Hkv][D/32] uint16)."""
    codes = np.zeros((batch, max_seq, n_kv, D // 2), np.uint8)
    scales = np.zeros((batch, max_seq, n_kv, D // 32), np.uint16)
    return codes, scales


def quantize_append(signs, k, v, start_pos, k_codes, k_scales, v_codes, v_scales) -> int:
    """Append k, v [B][n_new][Hkv][D] at start_pos[b] into the given caches (in place). Returns status bits."""
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    B, n_new, n_kv, D = k.shape
    max_seq = k_codes.shape[1]
    for a, dt in ((k_codes, np.uint8), (v_codes, np.uint8), (k_scales, np.uint16), (v_scales, np.uint16)):
        assert a.dtype == dt and a.flags.c_contiguous
    sp = _c(start_pos, np.int32)
    s = _c(signs, np.float32)
    return int(_load().oracle_quantize_append(B, max_seq, n_kv, D, _p(s), _p(k), _p(v), n_new, _p(sp),
                                              _p(k_codes), _p(k_scales), _p(v_codes), _p(v_scales)))


def decode_attention(signs, q, seq_lens, k_codes, k_scales, v_codes, v_scales, sm_scale, which=None):
    """Decode attention on the packed cache. q [B][Hq][D] -> (out [B][Hq][D] float32, status)."""
    q = _c(q, np.float32)
    B, n_q, D = q.shape
    max_seq, n_kv = k_codes.shape[1], k_codes.shape[2]
    sl = _c(seq_lens, np.int32)
    s = _c(signs, np.float32)
    out = np.zeros((B, n_q, D), np.float32)
    w = None if which is None else _c(which, np.uint8)
    st = _load().oracle_decode_attention(
        B, max_seq, n_kv, n_q, D, _p(s), _p(q), _p(sl),
        _p(_c(k_codes, np.uint8)), _p(_c(k_scales, np.uint16)),
        _p(_c(v_codes, np.uint8)), _p(_c(v_scales, np.uint16)),
        ctypes.c_float(sm_scale), None if w is None else _p(w), _p(out))
    return out, int(st)


def new_k16_cache(batch, max_seq, n_kv, D):
    """Zeroed binary16 K buffer [B][S][Hkv][D] (bits, uint16) for the asymmetric cache."""
    return np.zeros((batch, max_seq, n_kv, D), np.uint16)


def quantize_append_kf16(signs, k, v, start_pos, k_f16, v_codes, v_scales) -> int:
    """Asymmetric append: K stored as binary16 (original domain), V encoded as int4 codes. In place."""
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    B, n_new, n_kv, D = k.shape
    max_seq = v_codes.shape[1]
    assert k_f16.dtype == np.uint16 and k_f16.flags.c_contiguous and k_f16.shape[1] == max_seq
    for a, dt in ((v_codes, np.uint8), (v_scales, np.uint16)):
        assert a.dtype == dt and a.flags.c_contiguous
    sp = _c(start_pos, np.int32)
    s = _c(signs, np.float32)
    return int(_load().oracle_quantize_append_kf16(B, max_seq, n_kv, D, _p(s), _p(k), _p(v), n_new, _p(sp),
                                                   _p(k_f16), _p(v_codes), _p(v_scales)))


def decode_attention_kf16(signs, q, seq_lens, k_f16, v_codes, v_scales, sm_scale, which=None):
    """Decode attention on the asymmetric cache (binary16 K, int4 V). -> (out [B][Hq][D] float32, status)."""
    q = _c(q, np.float32)
    B, n_q, D = q.shape
    max_seq, n_kv = v_codes.shape[1], v_codes.shape[2]
    sl = _c(seq_lens, np.int32)
    s = _c(signs, np.float32)
    out = np.zeros((B, n_q, D), np.float32)
    w = None if which is None else _c(which, np.uint8)
    st = _load().oracle_decode_attention_kf16(
        B, max_seq, n_kv, n_q, D, _p(s), _p(q), _p(sl), _p(_c(k_f16, np.uint16)),
        _p(_c(v_codes, np.uint8)), _p(_c(v_scales, np.uint16)), ctypes.c_float(sm_scale),
        None if w is None else _p(w), _p(out))
    return out, int(st)


def _opt(a, dtype):
    return None if a is None else _c(a, dtype)


def encode_lambda(x, signs, lam):
    """SRHT, per-channel lambda (None = identity), quantise, pack -> (packed, scale bits, status)."""
    x = _c(x, np.float32)
    D = x.shape[-1]
    lam = _opt(lam, np.float32)
    packed = np.empty(x.shape[:-1] + (D // 2,), np.uint8)
    scales = np.empty(x.shape[:-1] + (D // 32,), np.uint16)
    st = _load().oracle_encode_lambda(_p(x), _p(_c(signs, np.float32)), None if lam is None else _p(lam), D,
                                      x.size // D, _p(packed), _p(scales))
    return packed, scales, int(st)


def quantize_append_lambda(signs, k, v, start_pos, lambda_k, lambda_v, k_codes, k_scales, v_codes, v_scales) -> int:
    """quantize_append with per-channel lambda vectors (None = identity). In place."""
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    B, n_new, n_kv, D = k.shape
    max_seq = k_codes.shape[1]
    lk, lv = _opt(lambda_k, np.float32), _opt(lambda_v, np.float32)
    return int(_load().oracle_quantize_append_lambda(
        B, max_seq, n_kv, D, _p(_c(signs, np.float32)), _p(k), _p(v), n_new, _p(_c(start_pos, np.int32)),
        None if lk is None else _p(lk), None if lv is None else _p(lv), _p(k_codes), _p(k_scales), _p(v_codes),
        _p(v_scales)))


def decode_attention_ext(signs, q, seq_lens, k_codes, k_scales, v_codes, v_scales, sm_scale, lambda_k=None,
                         lambda_v=None, tau=0.0, which=None, k_f16=None):
    """Decode with lambda and the sparse-V threshold -> (out, bound, status); bound as in the C comments."""
    q = _c(q, np.float32)
    B, n_q, D = q.shape
    max_seq, n_kv = v_codes.shape[1], v_codes.shape[2]
    out = np.zeros((B, n_q, D), np.float32)
    bound = np.zeros((B, n_q, D), np.float32)
    w = None if which is None else _c(which, np.uint8)
    lk, lv = _opt(lambda_k, np.float32), _opt(lambda_v, np.float32)
    kc = None if k_codes is None else _c(k_codes, np.uint8)
    ks = None if k_scales is None else _c(k_scales, np.uint16)
    kf = None if k_f16 is None else _c(k_f16, np.uint16)
    st = _load().oracle_decode_attention_ext(
        B, max_seq, n_kv, n_q, D, _p(_c(signs, np.float32)), _p(q), _p(_c(seq_lens, np.int32)),
        None if kc is None else _p(kc), None if ks is None else _p(ks), None if kf is None else _p(kf),
        _p(_c(v_codes, np.uint8)), _p(_c(v_scales, np.uint16)), None if lk is None else _p(lk),
        None if lv is None else _p(lv), ctypes.c_float(sm_scale), ctypes.c_double(tau),
        None if w is None else _p(w), _p(out), _p(bound))
    return out, bound, int(st)


def new_pool(n_pages, P, n_kv, D, k_f16=False):
    """Zeroed paged pools: (K codes or binary16 K, K scales or None, V codes, V scales), rows n_pages * P."""
    rows = n_pages * P
    if k_f16:
        kc, ks = np.zeros((rows, n_kv, D), np.uint16), None
    else:
        kc, ks = np.zeros((rows, n_kv, D // 2), np.uint8), np.zeros((rows, n_kv, D // 32), np.uint16)
    return kc, ks, np.zeros((rows, n_kv, D // 2), np.uint8), np.zeros((rows, n_kv, D // 32), np.uint16)


def quantize_append_paged(signs, k, v, start_pos, table, P, max_seq, pools) -> int:
    """Append k, v [B][n_new][Hkv][D] through the block table table [B][max_pages] into pools (in place)."""
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    B, n_new, n_kv, D = k.shape
    kc, ks, vc, vs = pools
    kf16 = kc.dtype == np.uint16
    n_pages = vc.shape[0] // P
    table = _c(table, np.int32)
    return int(_load().oracle_quantize_append_paged(
        B, max_seq, n_kv, D, _p(_c(signs, np.float32)), _p(k), _p(v), n_new, _p(_c(start_pos, np.int32)),
        _p(table), P, table.shape[1], n_pages, None if kf16 else _p(kc), None if kf16 else _p(ks),
        _p(kc) if kf16 else None, _p(vc), _p(vs)))


def decode_attention_paged(signs, q, seq_lens, table, P, max_seq, pools, sm_scale, which=None):
    """Decode over paged pools -> (out [B][Hq][D] float32, status)."""
    q = _c(q, np.float32)
    B, n_q, D = q.shape
    kc, ks, vc, vs = pools
    kf16 = kc.dtype == np.uint16
    n_kv = vc.shape[1]
    n_pages = vc.shape[0] // P
    table = _c(table, np.int32)
    out = np.zeros((B, n_q, D), np.float32)
    w = None if which is None else _c(which, np.uint8)
    st = _load().oracle_decode_attention_paged(
        B, max_seq, n_kv, n_q, D, _p(_c(signs, np.float32)), _p(q), _p(_c(seq_lens, np.int32)), _p(table), P,
        table.shape[1], n_pages, None if kf16 else _p(_c(kc, np.uint8)), None if kf16 else _p(_c(ks, np.uint16)),
        _p(_c(kc, np.uint16)) if kf16 else None, _p(_c(vc, np.uint8)), _p(_c(vs, np.uint16)),
        ctypes.c_float(sm_scale), None if w is None else _p(w), _p(out))
    return out, int(st)


def cold_length(length: int, window: int, fold: int) -> int:
    """Tokens of a delegated-cache sequence of `length` tokens that sit in the int4 body."""
    return int(_load().oracle_cold_length(length, window, fold))


def new_tail(batch, window, n_kv, D):
    """Zeroed binary16 V hot tail [B][W][Hkv][D] (bits, uint16) for the delegated cache."""
    return np.zeros((batch, window, n_kv, D), np.uint16)


def append_delegated(signs, k, v, start_pos, window, fold, k_f16, v_codes, v_scales, v_tail) -> int:
    """Delegated append (binary16 K; V into the binary16 hot tail, folded into int4 codes). In place."""
    k = _c(k, np.float32)
    v = _c(v, np.float32)
    B, n_new, n_kv, D = k.shape
    max_seq = v_codes.shape[1]
    assert k_f16.dtype == np.uint16 and k_f16.flags.c_contiguous and k_f16.shape[1] == max_seq
    assert v_tail.dtype == np.uint16 and v_tail.flags.c_contiguous and v_tail.shape == (B, window, n_kv, D)
    for a, dt in ((v_codes, np.uint8), (v_scales, np.uint16)):
        assert a.dtype == dt and a.flags.c_contiguous
    sp = _c(start_pos, np.int32)
    s = _c(signs, np.float32)
    return int(_load().oracle_append_delegated(B, max_seq, n_kv, D, _p(s), _p(k), _p(v), n_new, _p(sp),
                                               window, fold, _p(k_f16), _p(v_codes), _p(v_scales), _p(v_tail)))


def decode_attention_delegated(signs, q, seq_lens, k_f16, v_codes, v_scales, v_tail, window, fold, sm_scale,
                               which=None):
    """Decode attention on the delegated cache. -> (out [B][Hq][D] float32, status)."""
    q = _c(q, np.float32)
    B, n_q, D = q.shape
    max_seq, n_kv = v_codes.shape[1], v_codes.shape[2]
    sl = _c(seq_lens, np.int32)
    s = _c(signs, np.float32)
    out = np.zeros((B, n_q, D), np.float32)
    w = None if which is None else _c(which, np.uint8)
    st = _load().oracle_decode_attention_delegated(
        B, max_seq, n_kv, n_q, D, _p(s), _p(q), _p(sl), _p(_c(k_f16, np.uint16)),
        _p(_c(v_codes, np.uint8)), _p(_c(v_scales, np.uint16)), _p(_c(v_tail, np.uint16)), window, fold,
        ctypes.c_float(sm_scale), None if w is None else _p(w), _p(out))
    return out, int(st)


def dequantize(signs, codes, scales, seq_lens, original_domain: bool):
    """Dequantise a cache -> float32 [B][S][Hkv][D] (rows past seq_lens[b] are 0)."""
    B, max_seq, n_kv, half = codes.shape
    D = 2 * half
    out = np.empty((B, max_seq, n_kv, D), np.float32)
    st = _load().oracle_dequantize(B, max_seq, n_kv, D, _p(_c(signs, np.float32)),
                                   _p(_c(codes, np.uint8)), _p(_c(scales, np.uint16)),
                                   _p(_c(seq_lens, np.int32)), int(bool(original_domain)), _p(out))
    return out, int(st)
