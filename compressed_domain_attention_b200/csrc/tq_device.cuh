// Device helpers shared by the sm_100a kernels of libtq_b200.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tq.h"

namespace tqk {

// ----------------------------------------------------------------------------
// Walsh-Hadamard transform over a vector spread across a group of NG threads,
// each thread holding 32 consecutive elements (thread p of the group holds
// elements [32p, 32p + 32)). The butterfly stages run with stride
// h = 1, 2, ..., D/2 in that order; the pair (i, i+h) with (i & h) == 0 becomes
// (u_i + u_{i+h}, u_i - u_{i+h}). Strides 1..16 are in registers; strides
// 32..D/2 pair thread p with thread p ^ (h/32) through warp shuffles: the lower
// thread forms own + partner, the upper thread partner - own. Every add is an
// explicit round-to-nearest binary32 operation (no contraction), so the result
// is identical to the same stage sequence run element by element.
// `part` is the thread's index in its group; the group's lanes must be
// consecutive and aligned to NG inside the warp; all 32 lanes must call this.
// ----------------------------------------------------------------------------
template <int NG>
__device__ __forceinline__ void fwht_group(float (&u)[32], int part) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & h) == 0) {
        const float a = u[i], b = u[i + h];
        u[i] = __fadd_rn(a, b);
        u[i + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int hh = 1; hh < NG; hh <<= 1) {
    const bool upper = (part & hh) != 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, u[i], hh);
      u[i] = upper ? __fsub_rn(o, u[i]) : __fadd_rn(u[i], o);
    }
  }
}

// The same transform, same stage order and rounding, with the pair operations
// packed: stride 1 runs scalar; strides 2..16 add and subtract element pairs
// (i, i+1) and (i+h, i+h+1) with one f32x2 add and one f32x2 fma (b * -1 + a =
// a - b, one rounding per lane); the strides across threads form partner + own
// or partner - own as one f32x2 fma with a +-1 factor. Bit-identical to
// fwht_group (each lane of a packed op rounds once, exactly as the scalar op).
template <int NG>
__device__ __forceinline__ void fwht_group_x2(float (&u)[32], int part) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float x = u[i], y = u[i + 1];
    u[i] = __fadd_rn(x, y);
    u[i + 1] = __fsub_rn(x, y);
  }
#pragma unroll
  for (int hs = 2; hs < 32; hs <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      if ((i & hs) == 0) {
        const float2 x = make_float2(u[i], u[i + 1]), y = make_float2(u[i + hs], u[i + hs + 1]);
        const float2 sum = __fadd2_rn(x, y);
        const float2 dif = __ffma2_rn(y, make_float2(-1.f, -1.f), x);
        u[i] = sum.x;
        u[i + 1] = sum.y;
        u[i + hs] = dif.x;
        u[i + hs + 1] = dif.y;
      }
    }
  }
#pragma unroll
  for (int hh = 1; hh < NG; hh <<= 1) {
    const float sg = (part & hh) ? -1.f : 1.f;
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, u[i], hh), __shfl_xor_sync(0xffffffffu, u[i + 1], hh));
      const float2 n = __ffma2_rn(make_float2(u[i], u[i + 1]), make_float2(sg, sg), o);
      u[i] = n.x;
      u[i + 1] = n.y;
    }
  }
}

// Bits [32 part, 32 part + 32) of the sign mask: the diagonal of the 32 elements
// thread `part` of a head vector holds.
__device__ __forceinline__ uint32_t sign_word(const uint64_t* sign_bits, int part) {
  return (uint32_t)(sign_bits[part >> 1] >> (32 * (part & 1)));
}

// Element i of a thread's 32: flip its sign by bit i of the thread's sign word (exact).
__device__ __forceinline__ float flip_sign(float x, uint32_t sw, int i) {
  return __uint_as_float(__float_as_uint(x) ^ ((sw << (31 - i)) & 0x80000000u));
}

// Sign flip of element e by bit e of the sign mask (exact).
__device__ __forceinline__ float apply_sign(float x, const uint64_t* sign_bits, int e) {
  const uint32_t bit = (uint32_t)(sign_bits[e >> 6] >> (e & 63)) & 1u;
  return __uint_as_float(__float_as_uint(x) ^ (bit << 31));
}

// Load 32 consecutive elements of dtype `dt` starting at element index `idx`
// of `base` (16-byte aligned run) as binary32 (exact widening).
__device__ __forceinline__ void load32(float (&x)[32], const void* base, int64_t idx, int dt) {
  if (dt == TQ_F32) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(base) + idx);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 w = __ldg(p + j);
      x[4 * j + 0] = __uint_as_float(w.x);
      x[4 * j + 1] = __uint_as_float(w.y);
      x[4 * j + 2] = __uint_as_float(w.z);
      x[4 * j + 3] = __uint_as_float(w.w);
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(base) + idx);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 w = __ldg(p + j);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t lo = ww[k] & 0xffffu, hi = ww[k] >> 16;
        if (dt == TQ_BF16) {
          x[8 * j + 2 * k] = __uint_as_float(lo << 16);
          x[8 * j + 2 * k + 1] = __uint_as_float(hi << 16);
        } else {
          x[8 * j + 2 * k] = __half2float(__ushort_as_half((unsigned short)lo));
          x[8 * j + 2 * k + 1] = __half2float(__ushort_as_half((unsigned short)hi));
        }
      }
    }
  }
}

__device__ __forceinline__ float load_scalar(const void* base, int64_t idx, int dt) {
  if (dt == TQ_F32) return reinterpret_cast<const float*>(base)[idx];
  const uint16_t h = reinterpret_cast<const uint16_t*>(base)[idx];
  if (dt == TQ_BF16) return __uint_as_float((uint32_t)h << 16);
  return __half2float(__ushort_as_half(h));
}

__device__ __forceinline__ void status_or(int32_t* st, int32_t bits) {
  if (st != nullptr && bits != 0) atomicOr(st, bits);
}

// ----------------------------------------------------------------------------
// PTX wrappers: shared-memory addresses, mbarriers, bulk / tensor copies.
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Test whether the phase with the given parity has completed; the hardware may
// suspend the thread up to `hint_ns` before reporting that it has not.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete, giving up after
// `limit_ns` nanoseconds of wall time. Returns false on timeout. A suspending
// test (try_wait) may stay suspended until the phase completes, however short
// its hint, so a bound under 20 us is kept by polling the non-blocking test
// instead; longer bounds suspend up to 20 us per test.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  if (limit_ns < 20000u) {
    while (true) {
      if (mbar_test_wait(bar, parity)) return true;
      if (globaltimer_ns() - t0 > limit_ns) return false;
    }
  }
  while (true) {
    if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// binary32 a / 7 rounded to nearest, by one product with RN(1/7) and one fused
// correction (Markstein's method for division: q0 = RN(a y), r = a - 7 q0 exactly,
// q1 = RN(q0 + r y)); checked equal to the IEEE division for every finite a >= 0 (a GPU test).
__device__ __forceinline__ float div7_rn(float a) {
  constexpr float y = 0.142857149f;  // RN(1/7)
  const float q0 = __fmul_rn(a, y);
  const float r = __fmaf_rn(-7.0f, q0, a);
  return __fmaf_rn(r, y, q0);
}

// Reciprocal with at most one unit in the last place of error (rcp.approx.f32).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// NG consecutive binary16 values at a shared-memory address aligned to 2 NG bytes
// (NG in {1, 2, 4, 8}), widened to binary32 (exact).
template <int NG>
__device__ __forceinline__ void load_scales(float (&f)[NG], const uint8_t* p) {
  if constexpr (NG == 1) {
    f[0] = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(p)));
  } else {
    uint32_t w[NG / 2];
    if constexpr (NG == 2) {
      w[0] = *reinterpret_cast<const uint32_t*>(p);
    } else if constexpr (NG == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      w[0] = v.x;
      w[1] = v.y;
    } else {
      const uint4 v = *reinterpret_cast<const uint4*>(p);
      w[0] = v.x;
      w[1] = v.y;
      w[2] = v.z;
      w[3] = v.w;
    }
#pragma unroll
    for (int i = 0; i < NG / 2; ++i) {
      const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
}

// Hint: bring the line holding p into L2 (no data is returned; no L1 line is allocated).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 3-D tiled tensor load into this CTA's shared memory, completion counted on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1, int c2,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 2-D tiled tensor load into this CTA's shared memory, completion counted on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1, int c2,
                                            int c3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Contiguous bulk copy global -> this CTA's shared memory (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ----------------------------------------------------------------------------
// Tensor-core fragments (legacy warp-level MMA, register operands).
// ----------------------------------------------------------------------------
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t (&r)[2], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t (&r)[2], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}

// D = A(16x16, f16) * B(16x8, f16) + C, f32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A * B + C with C in separate registers (no copy into the accumulator).
__device__ __forceinline__ void mma_f16_16816_c(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                                float c0, float c1, float c2, float c3) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c2), "f"(c3));
}

// Accumulating form without the ordering constraint of a volatile asm.
__device__ __forceinline__ void mma_f16_16816_acc(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 2^x with the hardware approximation (ex2.approx.ftz): used for softmax weights.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2_f2(float2 v) {
  const __half2 h = __float22half2_rn(v);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Explicit shared-memory accesses (32-bit shared-window addresses).
__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds_u2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v));
}
__device__ __forceinline__ void sts_f2(uint32_t addr, float a, float b) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b));
}

__device__ __forceinline__ void sts_f4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d));
}
__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v));
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ __half2 __ushort_as_half2_pair(uint16_t bits) {
  return __halves2half2(__ushort_as_half(bits), __ushort_as_half(bits));
}

// Packed binary16 subtract on raw bit patterns.
__device__ __forceinline__ uint32_t h2_sub_u32(uint32_t a, __half2 b) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), b);
  return *reinterpret_cast<const uint32_t*>(&r);
}

// lop3 with an explicit truth table: (a & b) ^ c.
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace tqk
