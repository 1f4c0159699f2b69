"""Fixtures under tests/golden/: figures the pages print, checked on the host.

llama31_70b_128k_kv_bytes.txt (Open-TQ-Metal, arXiv abstract): the binary16 KV
cache of Llama 3.1 70B at 128K tokens is 40 GB, and the pages' int4 format holds
it in 12.5 GB. The cache layout of that shape must give exactly 40 GiB of
binary16 K+V. This layout stores 4-bit codes plus one binary16 scale per 32
elements: 4.5 bits per element, 11.25 GiB. The pages' 12.5 GB is 5 bits per
element (40 x 5 / 16), so their format keeps one more bit of side data per element.
"""
import os

import pytest

from compressed_domain_attention_b200 import tq

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
GIB = 1 << 30


def read_fixture(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = (s.strip() for s in line.split("="))
            out[k] = float(v) if "." in v else int(v)
    return out


@pytest.fixture(scope="module")
def lib():
    from compressed_domain_attention_b200.build import build_library
    build_library()
    return tq._lib()


def test_llama31_70b_128k_kv_bytes(lib):
    g = read_fixture("llama31_70b_128k_kv_bytes.txt")
    T, H, D = g["context"], g["kv_heads"], g["head_dim"]
    L = tq.tq_cache_layout(1, T, H, 8 * H, D, 32, 0)
    elems = T * H * D  # per layer, per K or V
    # binary16 K and V of every layer: the pages' 40 GB
    assert g["layers"] * 2 * elems * 2 == g["fp16_kv_gib"] * GIB
    # this layout: one codes buffer of 4 bits per element, and the scale array's
    # binary16 entries (one per 32 elements) inside the scales allocation
    assert L.codes_bytes * 8 == 4 * elems
    assert L.scale_stride_seq == T * H * (D // 32)  # binary16 entries per sequence
    scale_bytes = T * H * (D // 32) * 2
    assert L.scales_bytes >= scale_bytes
    packed = g["layers"] * 2 * (L.codes_bytes + scale_bytes)
    assert packed * 16 == g["fp16_kv_gib"] * GIB * 4.5   # 4.5 bits per element
    assert packed / GIB == 11.25
    # the pages' own figures agree with each other, at 5 bits per element
    assert g["fp16_kv_gib"] / g["pages_int4_kv_gib"] == g["pages_compression"]
    assert g["pages_int4_kv_gib"] * 16 == g["fp16_kv_gib"] * 5
