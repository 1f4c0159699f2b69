"""Host-side tests of the C ABI (no GPU needed, no device work issued).

The library must load on a machine without a GPU, export every symbol that
include/tq.h declares, validate shapes in tq_cache_layout (mlxcel user guide
"TurboQuant KV cache compression", §"Known limitations / head dimension":
power-of-two head dims only, others rejected at cache creation), and reject bad
arguments before touching the device.
"""
import ctypes
import os
import re

import numpy as np
import pytest

from compressed_domain_attention_b200 import tq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from compressed_domain_attention_b200.build import build_library
    build_library()
    return tq._lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    return sorted(set(re.findall(r"^\s*(?:int|int64_t|const char\*)\s+(tq_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 6
    for n in names:
        assert hasattr(lib, n), n
    assert set(tq.EXPORTS) == set(names)


def test_header_status_values_match_binding():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    for name in ("TQ_STATUS_NONFINITE", "TQ_STATUS_CAPACITY", "TQ_STATUS_TIMEOUT"):
        m = re.search(rf"#define {name} (\d+)", text)
        assert int(m.group(1)) == getattr(tq, name)
    for name in ("TQ_OK", "TQ_ERR_INVALID_ARG", "TQ_ERR_UNSUPPORTED", "TQ_ERR_CAPACITY", "TQ_ERR_CUDA"):
        m = re.search(rf"{name} = (-?\d+)", text)
        assert int(m.group(1)) == getattr(tq, name)


def test_status_bits_match_oracle_numbering(orc):
    assert tq.TQ_STATUS_NONFINITE == orc.STATUS_NONFINITE
    assert tq.TQ_STATUS_CAPACITY == orc.STATUS_CAPACITY


@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_layout_fields(lib, orc, D):
    L = tq.tq_cache_layout(3, 100, 8, 32, D, 32, 0)
    assert (L.batch, L.max_seq, L.n_kv_heads, L.n_q_heads, L.head_dim, L.group_size) == (3, 100, 8, 32, D, 32)
    assert L.n_groups == D // 32
    assert np.float32(L.c_d) == orc.norm_const(D)           # computed independently on both sides
    assert tq.sign_vector(L) == list(orc.sign_vector(0, D))  # both draw SplitMix64 independently
    assert L.code_stride_tok == 8 * D // 2
    assert L.code_stride_seq == 100 * 8 * D // 2
    assert L.scale_stride_tok == 8 * D // 32
    assert L.scale_stride_seq == 100 * 8 * D // 32
    assert L.codes_bytes == 3 * 100 * 8 * D // 2
    assert L.scales_bytes >= 3 * 100 * 8 * (D // 32) * 2 + 256 * 8 * (D // 32) * 2
    assert L.max_ctas == 1024
    assert L.decode_workspace_bytes >= (1024 + 3) * 32 * (D + 2) * 4


def test_layout_sign_seed(lib, orc):
    for seed in (1, 12345, 2 ** 63 + 5):
        L = tq.tq_cache_layout(1, 8, 1, 1, 128, 32, seed)
        assert tq.sign_vector(L) == list(orc.sign_vector(seed, 128))


@pytest.mark.parametrize("D", [16, 48, 80, 96, 192, 512, 0, -128])
def test_layout_rejects_head_dims(lib, D):
    code, _ = tq.tq_cache_layout_status(1, 16, 1, 1, D)
    assert code in (tq.TQ_ERR_UNSUPPORTED, tq.TQ_ERR_INVALID_ARG)
    if D in (16, 48, 80, 96, 192, 512):
        assert code == tq.TQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("args,code", [
    ((1, 16, 1, 1, 128, 64), tq.TQ_ERR_UNSUPPORTED),     # group size fixed at 32
    ((1, 16, 3, 4, 128, 32), tq.TQ_ERR_INVALID_ARG),     # n_q not a multiple of n_kv
    ((0, 16, 1, 1, 128, 32), tq.TQ_ERR_INVALID_ARG),
    ((1, 0, 1, 1, 128, 32), tq.TQ_ERR_INVALID_ARG),
    ((1, 16, 0, 1, 128, 32), tq.TQ_ERR_INVALID_ARG),
    ((1 << 16, 1 << 16, 1, 1, 128, 32), tq.TQ_ERR_UNSUPPORTED),  # more than 2^31 cache rows
])
def test_layout_rejects_shapes(lib, args, code):
    got, _ = tq.tq_cache_layout_status(*args)
    assert got == code


def test_layout_null_out(lib):
    assert lib.tq_cache_layout(1, 16, 1, 1, 128, 32, ctypes.c_uint64(0), None) == tq.TQ_ERR_INVALID_ARG


def test_calls_reject_bad_arguments_without_device_work(lib):
    L = tq.tq_cache_layout(2, 64, 2, 4, 128)
    P = ctypes.c_void_p
    fake = P(0x100000)  # never dereferenced: every call below fails validation first
    # NULL pointers
    assert lib.tq_quantize_append(ctypes.byref(L), None, fake, tq.TQ_BF16, 1, fake, fake, fake, fake, fake,
                                  None, None) == tq.TQ_ERR_INVALID_ARG
    # n_new larger than the cache
    assert lib.tq_quantize_append(ctypes.byref(L), fake, fake, tq.TQ_BF16, 65, fake, fake, fake, fake, fake,
                                  None, None) == tq.TQ_ERR_CAPACITY
    # negative n_new, bad dtype
    assert lib.tq_quantize_append(ctypes.byref(L), fake, fake, tq.TQ_BF16, -1, fake, fake, fake, fake, fake,
                                  None, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_quantize_append(ctypes.byref(L), fake, fake, 7, 1, fake, fake, fake, fake, fake,
                                  None, None) == tq.TQ_ERR_INVALID_ARG
    # n_new == 0 is a no-op that succeeds
    assert lib.tq_quantize_append(ctypes.byref(L), None, None, tq.TQ_BF16, 0, None, None, None, None, None,
                                  None, None) == tq.TQ_OK
    # misaligned code buffer
    assert lib.tq_quantize_append(ctypes.byref(L), fake, fake, tq.TQ_BF16, 1, fake, P(0x100004), fake, fake,
                                  fake, None, None) == tq.TQ_ERR_INVALID_ARG
    # decode: NULL workspace, misaligned out, non-finite scale
    args = [ctypes.byref(L), fake, tq.TQ_BF16, fake, fake, fake, fake, fake, ctypes.c_float(0.1), fake]
    assert lib.tq_decode_attention(*args, None, 1 << 30, None, None) == tq.TQ_ERR_INVALID_ARG
    args_bad_out = args[:-1] + [P(0x100008)]
    assert lib.tq_decode_attention(*args_bad_out, fake, 1 << 30, None, None) == tq.TQ_ERR_INVALID_ARG
    args_nan = args[:8] + [ctypes.c_float(float("nan")), fake]
    assert lib.tq_decode_attention(*args_nan, fake, 1 << 30, None, None) == tq.TQ_ERR_INVALID_ARG
    # dequantize: NULL codes
    assert lib.tq_dequantize_debug(ctypes.byref(L), None, fake, fake, 0, fake, None) == tq.TQ_ERR_INVALID_ARG


def test_decode_rejects_unsupported_shapes(lib):
    P = ctypes.c_void_p
    fake = P(0x100000)
    for shape in [(1, 64, 3, 3, 128), (1, 64, 16, 16, 128), (1, 64, 1, 16, 128), (2048, 8, 1, 1, 128)]:
        L = tq.tq_cache_layout(*shape)
        code = lib.tq_decode_attention(ctypes.byref(L), fake, tq.TQ_BF16, fake, fake, fake, fake, fake,
                                       ctypes.c_float(0.1), fake, fake, 1 << 40, None, None)
        assert code == tq.TQ_ERR_UNSUPPORTED, shape


def test_edited_layout_is_rejected(lib):
    L = tq.tq_cache_layout(1, 64, 1, 1, 128)
    L.max_seq = 128  # strides no longer match
    fake = ctypes.c_void_p(0x100000)
    assert lib.tq_quantize_append(ctypes.byref(L), fake, fake, tq.TQ_BF16, 1, fake, fake, fake, fake, fake,
                                  None, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention(None, fake, 0, fake, fake, fake, fake, fake, ctypes.c_float(1.0), fake, fake,
                                   1, None, None) == tq.TQ_ERR_INVALID_ARG


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, 99):
        assert isinstance(lib.tq_status_string(code), bytes)
    assert lib.tq_status_string(-2) == b"unsupported shape"


def test_layout_kv_formats():
    L4 = tq.tq_cache_layout(3, 100, 8, 32, 128)
    Lk = tq.tq_cache_layout_kv(3, 100, 8, 32, 128, tq.TQ_K_INT4)
    assert bytes(L4) == bytes(Lk)
    assert L4.k_format == tq.TQ_K_INT4 and L4.k_bytes == L4.codes_bytes and L4.k_stride_tok == L4.code_stride_tok
    L16 = tq.tq_cache_layout_kv(3, 100, 8, 32, 128, tq.TQ_K_FP16)
    assert L16.k_format == tq.TQ_K_FP16
    assert L16.k_stride_tok == 8 * 128 * 2 and L16.k_stride_seq == 100 * 8 * 128 * 2
    assert L16.k_bytes == 3 * 100 * 8 * 128 * 2
    # V side unchanged
    assert (L16.codes_bytes, L16.scales_bytes, L16.code_stride_tok) == (L4.codes_bytes, L4.scales_bytes,
                                                                        L4.code_stride_tok)
    code, _ = tq.tq_cache_layout_status(3, 100, 8, 32, 128)
    assert code == tq.TQ_OK
    with pytest.raises(tq.TqError) as exc:
        tq.tq_cache_layout_kv(3, 100, 8, 32, 128, 7)
    assert exc.value.code == tq.TQ_ERR_INVALID_ARG


def test_layout_delegated_and_cold_length():
    L = tq.tq_cache_layout_delegated(3, 100, 8, 32, 128, 16, 4)
    assert L.k_format == tq.TQ_KV_DELEGATED and (L.tail_window, L.fold_chunk) == (16, 4)
    assert L.k_bytes == 3 * 100 * 8 * 128 * 2
    assert L.tail_stride_tok == 8 * 128 * 2 and L.tail_stride_seq == 16 * 8 * 128 * 2
    assert L.tail_bytes == 3 * 16 * 8 * 128 * 2
    L4 = tq.tq_cache_layout(3, 100, 8, 32, 128)
    assert (L.codes_bytes, L.scales_bytes) == (L4.codes_bytes, L4.scales_bytes)
    # the worked rule: 0 up to W, then F * ceil((len - W) / F)
    assert [tq.tq_cold_length(L, n) for n in (0, 1, 16, 17, 20, 21, 24, 25, 100)] == [0, 0, 0, 4, 4, 8, 8, 12, 84]
    assert tq.tq_cold_length(L4, 77) == 77
    for bad in ((0, 1), (16, 0), (16, 17), (1025, 1), (-1, 1)):
        with pytest.raises(tq.TqError) as exc:
            tq.tq_cache_layout_delegated(3, 100, 8, 32, 128, *bad)
        assert exc.value.code == tq.TQ_ERR_INVALID_ARG
    with pytest.raises(tq.TqError) as exc:  # the window sizes come only through the delegated constructor
        tq.tq_cache_layout_kv(3, 100, 8, 32, 128, tq.TQ_KV_DELEGATED)
    assert exc.value.code == tq.TQ_ERR_INVALID_ARG


def test_delegated_layout_rejected_by_the_other_entry_points():
    # argument checks run before any device work, so these need no GPU
    import ctypes
    L = tq.tq_cache_layout_delegated(1, 64, 1, 4, 64, 8, 4)
    lib = tq._lib()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the layout check fails first
    assert lib.tq_quantize_append(ctypes.byref(L), fake, fake, 0, 1, fake, fake, None, fake, fake, None,
                                  None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention(ctypes.byref(L), fake, 0, fake, fake, None, fake, fake, ctypes.c_float(0.1),
                                   fake, fake, 1 << 30, None, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention_noalloc(ctypes.byref(L), fake, 0, fake, fake, None, fake, fake,
                                           ctypes.c_float(0.1), fake, None, None) == tq.TQ_ERR_INVALID_ARG
    L16 = tq.tq_cache_layout_kv(1, 64, 1, 4, 64, tq.TQ_K_FP16)
    assert lib.tq_append_delegated(ctypes.byref(L16), fake, fake, 0, 1, fake, fake, fake, fake, fake, None,
                                   None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention_delegated(ctypes.byref(L16), fake, 0, fake, fake, fake, fake, fake,
                                             ctypes.c_float(0.1), fake, fake, 1 << 30, None, None,
                                             None) == tq.TQ_ERR_INVALID_ARG


def test_layout_paged_sizes_and_checks():
    L = tq.tq_cache_layout_paged(4, 1000, 8, 32, 128, tq.TQ_K_INT4, 64, 70)
    assert (L.page_tokens, L.n_pages, L.max_pages) == (64, 70, 16)
    assert L.codes_bytes == 70 * 64 * 8 * 64
    assert L.code_stride_seq == 0 and L.code_stride_tok == 8 * 64
    L16 = tq.tq_cache_layout_paged(4, 1000, 8, 32, 128, tq.TQ_K_FP16, 64, 70)
    assert L16.k_bytes == 70 * 64 * 8 * 128 * 2
    for args, code in (((4, 1000, 8, 32, 128, tq.TQ_K_INT4, 48, 70), tq.TQ_ERR_INVALID_ARG),   # not a power of two
                       ((4, 1000, 8, 32, 128, tq.TQ_K_INT4, 64, 0), tq.TQ_ERR_INVALID_ARG),    # no pages
                       ((4, 1000, 8, 32, 128, tq.TQ_KV_DELEGATED, 64, 70), tq.TQ_ERR_INVALID_ARG),
                       ((4, 1000, 1, 4, 128, tq.TQ_K_INT4, 64, 70), tq.TQ_ERR_UNSUPPORTED)):   # tile of 256 tokens
        with pytest.raises(tq.TqError) as exc:
            tq.tq_cache_layout_paged(*args)
        assert exc.value.code == code
    # the slab entry points refuse a paged layout (no block table), before any device work
    import ctypes
    lib = tq._lib()
    fake = ctypes.c_void_p(1 << 20)
    assert lib.tq_quantize_append(ctypes.byref(L), fake, fake, 0, 1, fake, fake, fake, fake, fake, None,
                                  None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention(ctypes.byref(L), fake, 0, fake, fake, fake, fake, fake, ctypes.c_float(0.1),
                                   fake, fake, 1 << 30, None, None) == tq.TQ_ERR_INVALID_ARG


def test_decode_options_checked_before_device_work(lib):
    # a negative wait bound is refused on the host, before any CUDA call (this runs without a GPU)
    L = tq.tq_cache_layout(1, 64, 1, 4, 128)
    fake = ctypes.c_void_p(1 << 20)
    opts = tq.TqDecodeOpts(0, 0, None, None, None, 0.0, -5)
    assert lib.tq_decode_attention_ex(ctypes.byref(L), fake, tq.TQ_BF16, fake, fake, fake, fake, fake,
                                      ctypes.c_float(0.1), fake, fake, 1 << 30, None, ctypes.byref(opts),
                                      None) == tq.TQ_ERR_INVALID_ARG
    opts = tq.TqDecodeOpts(0, 0, None, None, None, -1.0, 0)
    assert lib.tq_decode_attention_ex(ctypes.byref(L), fake, tq.TQ_BF16, fake, fake, fake, fake, fake,
                                      ctypes.c_float(0.1), fake, fake, 1 << 30, None, ctypes.byref(opts),
                                      None) == tq.TQ_ERR_INVALID_ARG


def test_noalloc_refuses_paged_and_delegated_layouts_before_device_work(lib):
    # the no-alloc entry point has no block-table or hot-tail argument: both layouts are refused
    # before it looks at the device (this runs without a GPU)
    fake = ctypes.c_void_p(1 << 20)
    for L in (tq.tq_cache_layout_paged(2, 256, 8, 32, 128, tq.TQ_K_INT4, 64, 8),
              tq.tq_cache_layout_paged(2, 256, 8, 32, 128, tq.TQ_K_FP16, 64, 8),
              tq.tq_cache_layout_delegated(2, 256, 8, 32, 128, 64, 16)):
        assert lib.tq_decode_attention_noalloc(ctypes.byref(L), fake, tq.TQ_BF16, fake, fake, fake, fake, fake,
                                               ctypes.c_float(0.1), fake, None, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention_noalloc(None, fake, tq.TQ_BF16, fake, fake, fake, fake, fake,
                                           ctypes.c_float(0.1), fake, None, None) == tq.TQ_ERR_INVALID_ARG


def test_decode_options_struct_matches_the_header():
    # field order and types of tq_decode_opts_t as the header declares them
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    body = text[text.index("typedef struct {", text.index("Optional knobs for tq_decode_attention_ex")):
                text.index("} tq_decode_opts_t;")]
    fields = re.findall(r"^\s*(?:const\s+)?(int32_t|void\*|float\*|float|int64_t)\s+(\w+);", body, re.M)
    assert [f for _, f in fields] == [f for f, _ in tq.TqDecodeOpts._fields_]
