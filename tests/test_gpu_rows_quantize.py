"""GPU parity of the row-wise append kernel.

Appends of more than 65 536 K+V vectors at head_dim 64 and 128 (no hot tail) take
the row-wise kernel (one thread per head vector); shorter ones take the
thread-per-group kernel. Through the C ABI, against the oracle on the same seeded
inputs: codes and binary16 scale bits equal for every input dtype, both head
dims, int4 and binary16 K, the per-channel lambda, special values (non-finite
elements, all-zero vectors, vectors whose scale is a binary16 subnormal) and a
two-sequence batch with different start positions; the status bits agree; rows
outside the append stay untouched. The two kernels also agree with each other
bit for bit on the same data. A sequence whose append would pass max_seq is
skipped with TQ_STATUS_CAPACITY while the other is written; through a block table
with an unmapped entry, that page's tokens are skipped and every other pool row
equals the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
from compressed_domain_attention_b200 import tq
from tests.parity_utils import GpuCache, OracleCache, np_f32

pytestmark = pytest.mark.gpu

B, HKV, N = 2, 4, 4200      # 2 * 2 * 4200 * 4 = 67 200 K+V vectors: the row-wise kernel
START = [0, 5]
CAP = 4210


def inputs(D, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn((B, N, HKV, D), generator=g) * 3
    v = torch.randn((B, N, HKV, D), generator=g)
    k[0, 7, 1, 3] = float("inf")          # a non-finite group: scale +inf, codes 0
    v[1, 9, 2, 0] = float("nan")
    k[1, 11, 0, :] = 0.0                  # an all-zero vector: scale 0
    v[0, 13, 3, :] = 1e-6 * torch.randn(D, generator=g)  # binary16-subnormal scales: the exact path
    return k.to(dtype), v.to(dtype)


def assert_cache_bits(gpu, orc, D):
    kc, ks, vc, vs = gpu.host_arrays()
    for b in range(B):
        lo, hi = START[b], START[b] + N
        assert np.array_equal(vc[b, :hi], orc.vc[b, :hi]), f"V codes differ (sequence {b})"
        assert np.array_equal(vs[b, :hi], orc.vs[b, :hi]), f"V scales differ (sequence {b})"
        assert np.array_equal(kc[b, :hi], orc.kc[b, :hi]), f"K differs (sequence {b})"
        if ks is not None:
            assert np.array_equal(ks[b, :hi], orc.ks[b, :hi]), f"K scales differ (sequence {b})"
        assert not vc[b, :lo].any() and not vc[b, hi:].any(), "rows outside the append were written"


@pytest.mark.parametrize("k_format", [tq.TQ_K_INT4, tq.TQ_K_FP16])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("D", [64, 128])
def test_rows_kernel_bit_exact(D, dtype, k_format):
    kf = k_format == tq.TQ_K_FP16
    k, v = inputs(D, dtype, 100 + D)
    gpu = GpuCache(B, CAP, HKV, HKV, D, k_format=k_format)
    orc = OracleCache(B, CAP, HKV, D, kf16=kf)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gpu.append_all(k.cuda(), v.cuda(), START, status)
    st = 0
    for b in range(B):
        sp = np.array([START[b]], np.int32)
        if kf:
            st |= oracle.quantize_append_kf16(orc.signs, np_f32(k[b])[None], np_f32(v[b])[None], sp,
                                              orc.kc[b:b + 1], orc.vc[b:b + 1], orc.vs[b:b + 1])
        else:
            st |= oracle.quantize_append(orc.signs, np_f32(k[b])[None], np_f32(v[b])[None], sp, orc.kc[b:b + 1],
                                         orc.ks[b:b + 1], orc.vc[b:b + 1], orc.vs[b:b + 1])
    torch.cuda.synchronize()
    assert int(status.item()) == tq.TQ_STATUS_NONFINITE and st == oracle.STATUS_NONFINITE
    assert_cache_bits(gpu, orc, D)


@pytest.mark.parametrize("D", [64, 128])
def test_rows_kernel_lambda_bit_exact(D):
    k, v = inputs(D, torch.bfloat16, 300 + D)
    g = torch.Generator().manual_seed(7)
    lk = torch.exp(torch.rand(D, generator=g) * 2 - 1).float()
    lv = torch.exp(torch.rand(D, generator=g) * 2 - 1).float()
    gpu = GpuCache(B, CAP, HKV, HKV, D)
    sp = torch.tensor(START, dtype=torch.int32, device="cuda")
    tq.tq_quantize_append(gpu.layout, k.cuda().contiguous(), v.cuda().contiguous(), N, sp, gpu.k_codes,
                          gpu.k_scales, gpu.v_codes, gpu.v_scales, None, None, lambda_k=lk.cuda(),
                          lambda_v=lv.cuda())
    orc = OracleCache(B, CAP, HKV, D)
    for b in range(B):
        oracle.quantize_append_lambda(orc.signs, np_f32(k[b])[None], np_f32(v[b])[None],
                                      np.array([START[b]], np.int32), lk.numpy(), lv.numpy(), orc.kc[b:b + 1],
                                      orc.ks[b:b + 1], orc.vc[b:b + 1], orc.vs[b:b + 1])
    torch.cuda.synchronize()
    assert_cache_bits(gpu, orc, D)


@pytest.mark.parametrize("D", [64, 128])
def test_rows_and_group_kernels_agree(D):
    # the same vectors appended in one call (row-wise kernel) and in two calls of half
    # the tokens each (33 600 vectors per call: the thread-per-group kernel)
    k, v = inputs(D, torch.bfloat16, 500 + D)
    one = GpuCache(B, CAP, HKV, HKV, D)
    one.append_all(k.cuda(), v.cuda(), START)
    two = GpuCache(B, CAP, HKV, HKV, D)
    h = N // 2
    two.append_all(k[:, :h].cuda(), v[:, :h].cuda(), START)
    two.append_all(k[:, h:].cuda(), v[:, h:].cuda(), [s + h for s in START])
    torch.cuda.synchronize()
    for x, y in zip(one.host_arrays(), two.host_arrays()):
        assert np.array_equal(x, y)


def test_rows_kernel_capacity_skips_one_sequence():
    # sequence 1 starts at 20: 20 + 4200 > 4210, so its vectors are skipped (status
    # TQ_STATUS_CAPACITY) while sequence 0 is written exactly
    D = 128
    k, v = inputs(D, torch.bfloat16, 700)
    gpu = GpuCache(B, CAP, HKV, HKV, D)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gpu.append_all(k.cuda(), v.cuda(), [0, 20], status)
    orc = OracleCache(B, CAP, HKV, D)
    st = oracle.quantize_append(orc.signs, np_f32(k), np_f32(v), np.array([0, 20], np.int32), orc.kc, orc.ks, orc.vc,
                                orc.vs)
    torch.cuda.synchronize()
    assert int(status.item()) & tq.TQ_STATUS_CAPACITY and st & oracle.STATUS_CAPACITY
    kc, ks, vc, vs = gpu.host_arrays()
    assert np.array_equal(kc, orc.kc) and np.array_equal(ks, orc.ks)
    assert np.array_equal(vc, orc.vc) and np.array_equal(vs, orc.vs)
    assert not vc[1].any() and not kc[1].any(), "the skipped sequence was written"


def test_rows_kernel_paged_with_an_unmapped_page():
    # one sequence of 16 800 tokens x 2 kv heads (67 200 vectors) through a permuted block
    # table of 256-token pages with one entry unmapped: that page's tokens are skipped
    # (TQ_STATUS_CAPACITY), every other pool row equals the oracle's
    D, H, n, P = 128, 2, 16800, 256
    g = torch.Generator().manual_seed(800)
    k = (torch.randn((1, n, H, D), generator=g) * 2).to(torch.bfloat16)
    v = torch.randn((1, n, H, D), generator=g).to(torch.bfloat16)
    max_pages = -(-n // P)
    n_pages = max_pages + 3
    L = tq.tq_cache_layout_paged(1, n, H, 4 * H, D, tq.TQ_K_INT4, P, n_pages)
    rng = np.random.default_rng(5)
    table = rng.permutation(n_pages)[:max_pages].reshape(1, max_pages).astype(np.int32)
    table[0, 5] = -1
    kc, ks, vc, vs = tq.alloc_cache(L)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_quantize_append_paged(L, k.cuda(), v.cuda(), n, torch.zeros(1, dtype=torch.int32, device="cuda"),
                                torch.from_numpy(table).cuda(), kc, ks, vc, vs, status)
    signs = oracle.sign_vector(0, D)
    pools = oracle.new_pool(n_pages, P, H, D, False)
    st = oracle.quantize_append_paged(signs, np_f32(k), np_f32(v), np.zeros(1, np.int32), table, P, n, pools)
    torch.cuda.synchronize()
    assert int(status.item()) & tq.TQ_STATUS_CAPACITY and st & oracle.STATUS_CAPACITY
    rows = n_pages * P
    pk, pks, pv, pvs = pools
    assert np.array_equal(kc.cpu().numpy().reshape(rows, H, D // 2), pk)
    assert np.array_equal(ks[: rows * H * D // 32].cpu().numpy().view(np.uint16).reshape(rows, H, D // 32), pks)
    assert np.array_equal(vc.cpu().numpy().reshape(rows, H, D // 2), pv)
    assert np.array_equal(vs[: rows * H * D // 32].cpu().numpy().view(np.uint16).reshape(rows, H, D // 32), pvs)
