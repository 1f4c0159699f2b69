// Quantise-on-append and debug dequantise kernels (sm_100a).
//
// Open-TQ-Metal (abstract, cards page): one fused kernel runs the
// sign-randomised transform, per-group abs-max scaling and int4 nibble packing
// when a K/V vector enters the cache. Here one thread owns one group of 32
// rotated elements; the D/32 threads of a head vector exchange the transform's
// long-stride butterflies through warp shuffles. Every binary32 step is an
// explicit round-to-nearest intrinsic (no contraction), the scale is
// absmax / 7 rounded to binary16 (RNE), and codes are
// clamp(round_half_even(y / scale), -7, 7) against the stored scale, so codes
// and scales are bit-identical to the plain definition.
#include <cuda.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

// max that propagates NaN (max.NaN): the group's abs-max doubles as its non-finite check
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ float2 f2(float x) { return make_float2(x, x); }

// three-input max that propagates NaN, and the plain three-input max
__device__ __forceinline__ float fmax3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Cache row of token t of sequence b: b * max_seq + t, or through the block table
// with paged storage (ok = false for an entry outside [0, n_pages)).
__device__ __forceinline__ int64_t token_row(const QuantizeParams& p, int b, int64_t t, bool& ok) {
  ok = true;
  if (p.page_tokens <= 0) return (int64_t)b * p.max_seq + t;
  const int pg = p.block_table[(int64_t)b * p.max_pages + t / p.page_tokens];
  ok = pg >= 0 && pg < p.n_pages;
  return (int64_t)(ok ? pg : 0) * p.page_tokens + t % p.page_tokens;
}

// Asymmetric cache (mlxcel guide, cache modes: K kept in FP16): thread kt stores
// the binary16 (round to nearest even) of 32 consecutive K elements.
template <int D>
__device__ __forceinline__ void copy_k_f16(const QuantizeParams& p, uint32_t kt) {
  constexpr int NG = D / 32;
  const uint32_t r = kt / NG;
  const int part = (int)(kt % NG);
  const uint32_t bt = fast_div(r, p.div_kv);
  const int h = (int)(r - bt * (uint32_t)p.n_kv);
  const uint32_t b_ = fast_div(bt, p.div_new);
  const int t = (int)(bt - b_ * (uint32_t)p.n_new);
  const int b = (int)b_;
  float u[32];
  load32(u, p.k, (int64_t)r * D + part * 32, p.in_dtype);
  const int64_t pos = p.start_pos[b];
  if (pos < 0 || pos + p.n_new > p.max_seq) {
    if (t == 0 && h == 0 && part == 0) status_or(p.status, TQ_STATUS_CAPACITY);
    return;
  }
  uint32_t w[16];
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const __half2 hv = __floats2half2_rn(u[2 * i], u[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&hv);
    finite = finite && ((w[i] & 0x7C00u) != 0x7C00u) && ((w[i] & 0x7C000000u) != 0x7C000000u);
  }
  if (!finite) status_or(p.status, TQ_STATUS_NONFINITE);
  bool ok;
  const int64_t row = token_row(p, b, pos + t, ok) * p.n_kv + h;
  if (!ok) {
    if (part == 0) status_or(p.status, TQ_STATUS_CAPACITY);
    return;
  }
  uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.k_codes) + row * D + part * 32);
#pragma unroll
  for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

// Delegated cache: store the binary16 of the thread's 32 input V elements in the
// hot tail at slot pos % W (non-finite results set the status, as for K).
template <int D>
__device__ __forceinline__ void write_tail_f16(const QuantizeParams& p, int64_t in_row, int b, int h, int part,
                                               int64_t pos) {
  float u[32];
  load32(u, p.v, in_row * D + part * 32, p.in_dtype);
  uint32_t w[16];
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const __half2 hv = __floats2half2_rn(u[2 * i], u[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&hv);
    finite = finite && ((w[i] & 0x7C00u) != 0x7C00u) && ((w[i] & 0x7C000000u) != 0x7C000000u);
  }
  if (!finite) status_or(p.status, TQ_STATUS_NONFINITE);
  const int64_t slot = ((int64_t)b * p.tail_window + pos % p.tail_window) * p.n_kv + h;
  uint4* dst = reinterpret_cast<uint4*>(p.v_tail + slot * D + part * 32);
#pragma unroll
  for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

template <int D>
__global__ void __launch_bounds__(256, 4) quantize_append_kernel(const __grid_constant__ QuantizeParams p) {
  // Launched as a programmatic dependent of the previous kernel on the stream:
  // nothing is read before this wait. The decode that usually follows may be
  // scheduled from here on; it waits for this grid's completion before reading.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int NG = D / 32;
  // 32-bit indexing throughout (the host launches fewer than 2^32 threads); divisions
  // by the runtime sizes are multiply-and-shift (FastDiv)
  const uint32_t gt = blockIdx.x * blockDim.x + threadIdx.x;
  const int W = p.tail_window;  // > 0 only for the delegated cache
  const uint32_t vecs_k = (uint32_t)p.batch * (uint32_t)p.n_new * (uint32_t)p.n_kv;
  // V work items per (sequence, head): the new tokens, then (delegated) W fold candidates
  const int v_rows = p.n_new + W;
  const uint32_t vec = gt / NG;
  const int part = (int)(gt % NG);
  int which;
  uint32_t r;
  bool in_range;
  if (p.k_f16) {
    // V threads first, then the K copies from the next warp boundary on, so that a
    // warp is all V (its lanes exchange butterflies) or all K.
    const uint32_t thr_v = (uint32_t)p.batch * (uint32_t)v_rows * (uint32_t)p.n_kv * NG;
    const uint32_t kbase = (thr_v + 31) / 32 * 32;
    if (gt >= kbase) {
      if (gt - kbase < vecs_k * NG) copy_k_f16<D>(p, gt - kbase);
      return;
    }
    in_range = gt < thr_v;  // the rest pads the warp
    which = 1;
    r = in_range ? vec : 0;
  } else {
    in_range = vec < 2 * vecs_k;
    which = (in_range && vec >= vecs_k) ? 1 : 0;  // 0 = K, 1 = V
    r = in_range ? vec - (which ? vecs_k : 0u) : 0u;
  }
  const int rows = which ? v_rows : p.n_new;
  const uint32_t bt = fast_div(r, p.div_kv);
  const int h = (int)(r - bt * (uint32_t)p.n_kv);
  const uint32_t b_ = fast_div(bt, which ? p.div_vrows : p.div_new);
  const int t = (int)(bt - b_ * (uint32_t)rows);
  const int b = (int)b_;
  const int64_t in_row = ((int64_t)b * p.n_new + t) * p.n_kv + h;  // input vector of a new token

  float u[32];
  int64_t pos = 0;
  if (in_range) pos = p.start_pos[b];
  bool valid = in_range;
  if (in_range && (pos < 0 || pos + p.n_new > p.max_seq)) {
    valid = false;
    if (which == 0 && t == 0 && h == 0 && part == 0) status_or(p.status, TQ_STATUS_CAPACITY);
  }
  int64_t dst = pos + t;     // position whose codes this item writes
  int64_t tail_pos = -1;     // delegated: new token written to the hot tail after the encode
  if (W == 0) {
    if (in_range) {
      load32(u, which ? p.v : p.k, in_row * D + part * 32, p.in_dtype);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) u[i] = 0.f;
    }
  } else {
    // Delegated cache (mlxcel guide, delegated cache variant): V grows from len0 to
    // len1 tokens; positions below cold_tokens(len1) hold int4 codes, the rest the
    // binary16 tail at slot pos % W. Each item encodes at most one vector, from the
    // input (a new token that is cold at once) or from the tail (an old hot token
    // that folds), and a new hot token then takes its slot. An old token whose slot a
    // new hot token takes is folded by that token's item, before the overwrite.
    const int64_t len0 = pos, len1 = pos + p.n_new;
    const int64_t nc0 = cold_tokens(len0, W, p.fold_chunk), nc1 = cold_tokens(len1, W, p.fold_chunk);
    int src = 0;  // 0 none, 1 input, 2 tail slot of dst
    if (t < p.n_new) {
      if (dst < nc1) {
        src = 1;
      } else {
        tail_pos = dst;
        const int64_t old = len0 - W + (dst - len0) % W;  // the old token in the same slot, if any
        if (old >= nc0 && old >= 0) {
          src = 2;
          dst = old;
        }
      }
    } else {
      dst = nc0 + (t - p.n_new);
      if (dst < min(nc1, len0)) {
        const int64_t lo = max(len0, nc1);
        const int64_t taker = lo + (((dst - lo) % W) + W) % W;  // first new hot token in this slot
        if (taker >= len1) src = 2;
      }
    }
    if (src == 0 || !valid) {
      valid = false;
#pragma unroll
      for (int i = 0; i < 32; ++i) u[i] = 0.f;
    } else if (src == 1) {
      load32(u, p.v, in_row * D + part * 32, p.in_dtype);
#pragma unroll
      for (int i = 0; i < 32; ++i) u[i] = __half2float(__float2half_rn(u[i]));  // the tail's binary16 value
    } else {
      const uint4* hp = reinterpret_cast<const uint4*>(
          p.v_tail + (((int64_t)b * W + dst % W) * p.n_kv + h) * D + part * 32);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 w4 = hp[j];
        const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ww[k]));
          u[8 * j + 2 * k] = f.x;
          u[8 * j + 2 * k + 1] = f.y;
        }
      }
    }
    if (!(in_range && pos >= 0 && pos + p.n_new <= p.max_seq)) tail_pos = -1;
  }
  // sign diagonal, then the Walsh-Hadamard butterflies (strides 1, 2, ..., D/2 in
  // that order, packed pair operations that round each lane once as the scalar steps)
  const uint32_t sw = sign_word(p.sign_bits, part);
#pragma unroll
  for (int i = 0; i < 32; ++i) u[i] = flip_sign(u[i], sw, i);
  fwht_group_x2<NG>(u, part);

  float a = 0.f;
  // per-channel lambda (Open-TQ-Metal abstract: between the transform and the
  // abs-max): one more binary32 multiply per element
  const float* lam = which ? p.lambda_v : p.lambda_k;
  if (lam != nullptr) {
    const float4* l4 = reinterpret_cast<const float4*>(lam + part * 32);
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float4 lv = __ldg(l4 + i / 4);
      const float2 y0 = __fmul2_rn(__fmul2_rn(make_float2(u[i], u[i + 1]), f2(p.c_d)), make_float2(lv.x, lv.y));
      const float2 y1 =
          __fmul2_rn(__fmul2_rn(make_float2(u[i + 2], u[i + 3]), f2(p.c_d)), make_float2(lv.z, lv.w));
      u[i] = y0.x;
      u[i + 1] = y0.y;
      u[i + 2] = y1.x;
      u[i + 3] = y1.y;
      a = fmax_nan(a, fmax_nan(fmax_nan(fabsf(y0.x), fabsf(y0.y)), fmax_nan(fabsf(y1.x), fabsf(y1.y))));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 y = __fmul2_rn(make_float2(u[i], u[i + 1]), f2(p.c_d));
      u[i] = y.x;
      u[i + 1] = y.y;
      a = fmax3_nan(a, fabsf(y.x), fabsf(y.y));
    }
  }
  if (!valid) {
    if (tail_pos >= 0) write_tail_f16<D>(p, in_row, b, h, part, tail_pos);
    return;
  }

  const float sigma32 = __fdiv_rn(a, 7.0f);
  const __half sig16 = __float2half_rn(sigma32);
  const float sigma = __half2float(sig16);
  uint16_t sbits = __half_as_ushort(sig16);
  uint32_t packed[4] = {0u, 0u, 0u, 0u};
  if (!(a <= 3.402823466e38f) || !(fabsf(sigma) <= 65504.f)) {
    sbits = 0x7C00u;
    status_or(p.status, TQ_STATUS_NONFINITE);
  } else if (sigma != 0.f) {
    // code = clamp(rint(fl(y / sigma)), -7, 7). Fast form: r = RN(y * RN(1/sigma)); adding
    // 1.5 * 2^23 rounds r to an integer (ties to even) in the low mantissa bits, whose
    // low nibble is then the two's-complement code. |r - y/sigma| <= 2^-23 |y/sigma| < 2^-20
    // and |fl(y/sigma) - y/sigma| <= 2^-21, so unless r lies within 2^-19 of a
    // half-integer, fl(y/sigma) rounds to the same integer. A binary16-normal sigma keeps
    // |y/sigma| <= 7 (1 + 2^-11) (1 + 2^-24), so no clamp is needed. Otherwise (a tie
    // within 2^-19, probability about 2^-18 per element, or a subnormal sigma) the
    // thread redoes its group with the IEEE division and the clamp.
    bool slow = !(sigma >= 6.103515625e-05f);  // binary16 subnormal scale
    if (!slow) {
      const float inv = __frcp_rn(sigma);
      constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
      uint32_t rb[32];  // the rounded sums: the low byte holds the code (two's complement)
      float dmax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float2 rv = __fmul2_rn(make_float2(u[i], u[i + 1]), f2(inv));
        const float2 rm = __fadd2_rn(rv, f2(kMagic));
        const float2 rr = __fadd2_rn(rm, f2(-kMagic));
        const float2 d = __ffma2_rn(rr, f2(-1.f), rv);  // r - rint(r), exact
        dmax = fmax3(dmax, fabsf(d.x), fabsf(d.y));
        rb[i] = __float_as_uint(rm.x);
        rb[i + 1] = __float_as_uint(rm.y);
      }
      slow = dmax >= 0.49999809265136719f;  // 0.5 - 2^-19
      // byte j of a packed word: code 2j in the low nibble, code 2j + 1 in the high one
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t* e = rb + 8 * k;
        const uint32_t lo = __byte_perm(__byte_perm(e[0], e[2], 0x0040u), __byte_perm(e[4], e[6], 0x0040u), 0x5410u);
        const uint32_t hi = __byte_perm(__byte_perm(e[1], e[3], 0x0040u), __byte_perm(e[5], e[7], 0x0040u), 0x5410u);
        packed[k] = (lo & 0x0F0F0F0Fu) | ((hi << 4) & 0xF0F0F0F0u);
      }
    }
    if (slow) {
#pragma unroll
      for (int k = 0; k < 4; ++k) packed[k] = 0u;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        int c = __float2int_rn(__fdiv_rn(u[i], sigma));
        c = max(-7, min(7, c));
        packed[i >> 3] |= ((uint32_t)c & 0xFu) << (4 * (i & 7));
      }
    }
  }
  bool row_ok;
  const int64_t row = token_row(p, b, dst, row_ok) * p.n_kv + h;
  if (!row_ok) {  // an unmapped page: nothing is written
    if (part == 0) status_or(p.status, TQ_STATUS_CAPACITY);
    return;
  }
  uint8_t* codes = which ? p.v_codes : p.k_codes;
  uint16_t* scales = which ? p.v_scales : p.k_scales;
  *reinterpret_cast<uint4*>(codes + row * (D / 2) + part * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  scales[row * NG + part] = sbits;
  if (tail_pos >= 0) write_tail_f16<D>(p, in_row, b, h, part, tail_pos);
}

// ---------------------------------------------------------------------------
// One thread per head vector (head_dim 64 or 128, caches without a hot tail).
// ---------------------------------------------------------------------------
// In the kernel above a quarter of the instructions go to the butterfly stages
// that cross threads (shuffles) and to per-group index and status work. Here a
// block's input rows arrive by tensor copies in a shared slab with the 128-byte
// swizzle (eight consecutive rows spread each 16-byte column over all banks),
// and each thread keeps its whole vector in registers: the sign diagonal (an XOR
// of the sign bits before widening), all log2(D) butterfly stages, the binary32
// scaling and the per-group encoding. Every operation, rounding and stage order
// is that of quantize_append_kernel, so codes and scales are bit-identical.
template <int D, int DT>
struct RowsCfg {
  static constexpr int ESZ = DT == TQ_F32 ? 4 : 2;    // input element bytes
  static constexpr int EPB = 128 / ESZ;               // elements per 128-byte box row
  static constexpr int NCOL = D / EPB;                // boxes per vector
  static constexpr int TPV = rows_threads_per_vector(D);  // threads per vector (1; the code also runs 2)
  static constexpr int EPT = D / TPV;                 // elements per thread
  static constexpr int BPT = EPT / EPB;               // boxes per thread
  static constexpr int NGT = EPT / 32;                // groups per thread
  static constexpr int VPW = 32 / TPV;                // vectors per warp
  static constexpr int NVB = kRowsThreads / TPV;      // vectors per chunk (the box rows)
  static constexpr int SLAB = NCOL * NVB * 128;       // one chunk's input
  static constexpr int STAGES = 2;                    // chunk c + 2 grid copies in while chunk c is encoded
  static constexpr int NMASK = ESZ == 2 ? D / 2 : D;  // sign masks: per element pair (2-byte input) or element
  static constexpr int OFF_MASK = STAGES * SLAB;
  static constexpr int OFF_BAR = OFF_MASK + 4 * NMASK;
  static constexpr int SMEM = OFF_BAR + 8 * STAGES + 1024;  // + slack to align the slabs to 1024 bytes
  static_assert(NCOL >= 1 && NCOL * EPB == D && BPT >= 1 && BPT * EPB == EPT, "whole 128-byte boxes per thread");
  static_assert(NVB == rows_kernel_box_rows(D), "the host's box height");
};

constexpr uint64_t kRowsWaitNs = 1000000000ull;  // bound on the wait for the block's input copy (1 s)
// Resident blocks per SM the register budget is set for (a head_dim-128 vector in
// registers plus the encoding's temporaries: at most 168 registers per thread).
constexpr int kRowsBlocksPerSm = 3;

// RN(a + c) and RN(a - c) for a binary16 or bfloat16 a (widened exactly) and a binary32 c:
// the mixed-precision add and subtract of sm_100.
template <int DT>
__device__ __forceinline__ float add_mixed(uint16_t a, float c) {
  float d;
  if constexpr (DT == TQ_BF16)
    asm("add.rn.f32.bf16 %0, %1, %2;" : "=f"(d) : "h"(a), "f"(c));
  else
    asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(a), "f"(c));
  return d;
}
template <int DT>
__device__ __forceinline__ float sub_mixed(uint16_t a, float c) {
  float d;
  if constexpr (DT == TQ_BF16)
    asm("sub.rn.f32.bf16 %0, %1, %2;" : "=f"(d) : "h"(a), "f"(c));
  else
    asm("sub.rn.f32.f16 %0, %1, %2;" : "=f"(d) : "h"(a), "f"(c));
  return d;
}

// The thread's EPT input elements (elements hv EPT .. hv EPT + EPT - 1 of the vector in
// row v of the swizzled slab) after the sign diagonal (an XOR of the sign bits,
// exact) and the stride-1 butterflies: for 2-byte inputs each pair (x0, x1) of one
// word becomes (RN(x0 + x1), RN(x0 - x1)) with x0 widened inside the mixed-precision
// add, the scalar step's operands and rounding.
template <int D, int DT>
__device__ __forceinline__ void load_row_stage1(float (&u)[RowsCfg<D, DT>::EPT], const uint8_t* slab, int v, int hv,
                                                const uint32_t* smask) {
  using C = RowsCfg<D, DT>;
  const int sw = v & 7;
#pragma unroll
  for (int bb = 0; bb < C::BPT; ++bb) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 w = *reinterpret_cast<const uint4*>(slab + (hv * C::BPT + bb) * (C::NVB * 128) + v * 128 +
                                                      ((j ^ sw) << 4));
      const int e0 = bb * C::EPB + j * (16 / C::ESZ);  // within the thread's elements
      const int g0 = hv * C::EPT + e0;                 // within the vector
      const uint4 m = *reinterpret_cast<const uint4*>(smask + (C::ESZ == 2 ? g0 / 2 : g0));
      const uint32_t ww[4] = {w.x ^ m.x, w.y ^ m.y, w.z ^ m.z, w.w ^ m.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if constexpr (DT == TQ_F32) {
          u[e0 + k] = __uint_as_float(ww[k]);
        } else {
          const uint16_t x0 = (uint16_t)(ww[k] & 0xffffu);
          float x1;
          if constexpr (DT == TQ_BF16)
            x1 = __uint_as_float(ww[k] & 0xffff0000u);
          else
            x1 = __half2float(__ushort_as_half((uint16_t)(ww[k] >> 16)));
          u[e0 + 2 * k] = add_mixed<DT>(x0, x1);
          u[e0 + 2 * k + 1] = sub_mixed<DT>(x0, x1);
        }
      }
    }
  }
  if constexpr (DT == TQ_F32) {
#pragma unroll
    for (int i = 0; i < C::EPT; i += 2) {
      const float x = u[i], y = u[i + 1];
      u[i] = __fadd_rn(x, y);
      u[i + 1] = __fsub_rn(x, y);
    }
  }
}

// The thread's EPT input elements widened to binary32, without the sign diagonal
// (the asymmetric cache's binary16 K copy).
template <int D, int DT>
__device__ __forceinline__ void load_row_raw(float (&u)[RowsCfg<D, DT>::EPT], const uint8_t* slab, int v, int hv) {
  using C = RowsCfg<D, DT>;
  const int sw = v & 7;
#pragma unroll
  for (int bb = 0; bb < C::BPT; ++bb) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 w = *reinterpret_cast<const uint4*>(slab + (hv * C::BPT + bb) * (C::NVB * 128) + v * 128 +
                                                      ((j ^ sw) << 4));
      const int e0 = bb * C::EPB + j * (16 / C::ESZ);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if constexpr (DT == TQ_F32) {
          u[e0 + k] = __uint_as_float(ww[k]);
        } else if constexpr (DT == TQ_BF16) {
          u[e0 + 2 * k] = __uint_as_float(ww[k] << 16);
          u[e0 + 2 * k + 1] = __uint_as_float(ww[k] & 0xffff0000u);
        } else {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ww[k]));
          u[e0 + 2 * k] = f.x;
          u[e0 + 2 * k + 1] = f.y;
        }
      }
    }
  }
}

// Walsh-Hadamard butterflies of strides 2, 4, ..., N/2 in that order on N elements
// in registers, after the stride-1 step of load_row_stage1 (packed pairs; each lane
// rounds once, as the scalar steps do).
template <int N>
__device__ __forceinline__ void fwht_row_from2(float (&u)[N]) {
#pragma unroll
  for (int hs = 2; hs < N; hs <<= 1) {
#pragma unroll
    for (int i = 0; i < N; i += 2) {
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
}

// Fast encoding of one group (see encode_group for the definition and the exact path):
// returns false, and leaves the group to encode_group, when a is not finite, the
// binary16 scale is zero, subnormal or infinite, or some element lies within
// 2^-19 of a rounding tie. inv is RN(1/sigma) within one ulp (relative error at
// most 2^-23), so |y * inv - y / sigma| <= 7.01 * 2^-23 < 2^-20, |fl(y / sigma) -
// y / sigma| <= 2^-22, and |d| < 0.5 - 2^-19 keeps the true distance to a
// half-integer above 2^-19 - 2^-25, more than the 1.25 * 2^-20 between y * inv
// and fl(y / sigma): both round to the same integer, within [-7, 7].
__device__ __forceinline__ bool encode_group_fast(const float* y, float a, uint32_t (&packed)[4], uint16_t& sbits) {
  const __half sig16 = __float2half_rn(div7_rn(a));
  const float sigma = __half2float(sig16);
  sbits = __half_as_ushort(sig16);
  const bool regular = (a <= 3.402823466e38f) && (sigma >= 6.103515625e-05f) && (sigma <= 65504.f);
  const float inv = rcp_approx(sigma);
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  float dm[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t e[8];
    float dk = 0.f;
#pragma unroll
    for (int q = 0; q < 8; q += 2) {
      const float2 yv = make_float2(y[8 * k + q], y[8 * k + q + 1]);
      const float2 tm = __ffma2_rn(yv, f2(inv), f2(kMagic));
      const float2 nr = __ffma2_rn(tm, f2(-1.f), f2(kMagic));  // -(the integer), exact
      const float2 d = __ffma2_rn(yv, f2(inv), nr);
      dk = fmax3(dk, fabsf(d.x), fabsf(d.y));
      e[q] = __float_as_uint(tm.x);
      e[q + 1] = __float_as_uint(tm.y);
    }
    dm[k] = dk;
    const uint32_t lo = __byte_perm(__byte_perm(e[0], e[2], 0x0040u), __byte_perm(e[4], e[6], 0x0040u), 0x5410u);
    const uint32_t hi = __byte_perm(__byte_perm(e[1], e[3], 0x0040u), __byte_perm(e[5], e[7], 0x0040u), 0x5410u);
    packed[k] = (lo & 0x0F0F0F0Fu) | ((hi << 4) & 0xF0F0F0F0u);
  }
  const float dmax = fmax3(fmax3(dm[0], dm[1], dm[2]), dm[3], 0.f);
  return regular && dmax < 0.49999809265136719f;  // 0.5 - 2^-19
}

// NaN-propagating maximum of |y_0| .. |y_31| as a shallow tree (depth 4).
__device__ __forceinline__ float absmax32_nan(const float* y) {
  float m[11];
#pragma unroll
  for (int k = 0; k < 10; ++k) m[k] = fmax3_nan(fabsf(y[3 * k]), fabsf(y[3 * k + 1]), fabsf(y[3 * k + 2]));
  m[10] = fmax_nan(fabsf(y[30]), fabsf(y[31]));
  const float a0 = fmax3_nan(m[0], m[1], m[2]), a1 = fmax3_nan(m[3], m[4], m[5]);
  const float a2 = fmax3_nan(m[6], m[7], m[8]), a3 = fmax_nan(m[9], m[10]);
  return fmax_nan(fmax3_nan(a0, a1, a2), a3);
}

// Encode one group of 32 rotated, scaled elements: the binary16 scale bits and
// the 16 code bytes (codes 2j and 2j + 1 in the low and high nibble of byte j).
// Same definition as quantize_append_kernel; the fast path rounds with one fused
// multiply-add: RN(y * inv + 1.5 * 2^23) holds the integer nearest the exact
// y * inv in its low mantissa bits, and d = RN(y * inv - that integer) bounds
// its distance from a half-integer. |y * inv - y / sigma| <= 7.01 * 2^-24 and
// |fl(y / sigma) - y / sigma| <= 2^-22, so when every |d| < 0.5 - 2^-19 (the
// true distance to a half-integer then exceeds 2^-19 - 2^-25 > 2^-20) the
// rounded fl(y / sigma) is the same integer, within [-7, 7]. Otherwise, or for a
// binary16-subnormal scale, the group takes the IEEE division and the clamp.
__device__ __forceinline__ uint16_t encode_group(const float* y, float a, uint32_t (&packed)[4],
                                                 int32_t* status) {
  const float sigma32 = __fdiv_rn(a, 7.0f);
  const __half sig16 = __float2half_rn(sigma32);
  const float sigma = __half2float(sig16);
  uint16_t sbits = __half_as_ushort(sig16);
#pragma unroll
  for (int k = 0; k < 4; ++k) packed[k] = 0u;
  if (!(a <= 3.402823466e38f) || !(fabsf(sigma) <= 65504.f)) {
    status_or(status, TQ_STATUS_NONFINITE);
    return 0x7C00u;
  }
  if (sigma == 0.f) return sbits;
  bool slow = !(sigma >= 6.103515625e-05f);  // binary16 subnormal scale
  if (!slow) {
    const float inv = __frcp_rn(sigma);
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    float dmax = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t e[8];
#pragma unroll
      for (int q = 0; q < 8; q += 2) {
        const float2 yv = make_float2(y[8 * k + q], y[8 * k + q + 1]);
        const float2 tm = __ffma2_rn(yv, f2(inv), f2(kMagic));
        const float2 nr = __ffma2_rn(tm, f2(-1.f), f2(kMagic));  // -(the integer), exact
        const float2 d = __ffma2_rn(yv, f2(inv), nr);
        dmax = fmax3(dmax, fabsf(d.x), fabsf(d.y));
        e[q] = __float_as_uint(tm.x);
        e[q + 1] = __float_as_uint(tm.y);
      }
      const uint32_t lo = __byte_perm(__byte_perm(e[0], e[2], 0x0040u), __byte_perm(e[4], e[6], 0x0040u), 0x5410u);
      const uint32_t hi = __byte_perm(__byte_perm(e[1], e[3], 0x0040u), __byte_perm(e[5], e[7], 0x0040u), 0x5410u);
      packed[k] = (lo & 0x0F0F0F0Fu) | ((hi << 4) & 0xF0F0F0F0u);
    }
    slow = dmax >= 0.49999809265136719f;  // 0.5 - 2^-19
  }
  if (slow) {
#pragma unroll
    for (int k = 0; k < 4; ++k) packed[k] = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      int c = __float2int_rn(__fdiv_rn(y[i], sigma));
      c = max(-7, min(7, c));
      packed[i >> 3] |= ((uint32_t)c & 0xFu) << (4 * (i & 7));
    }
  }
  return sbits;
}

template <int D, int DT>
__global__ void __launch_bounds__(kRowsThreads, kRowsBlocksPerSm)
    quantize_rows_kernel(const __grid_constant__ QuantizeParams p, const __grid_constant__ CUtensorMap kin,
                         const __grid_constant__ CUtensorMap vin) {
  using C = RowsCfg<D, DT>;
  constexpr int NG = D / 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* slab = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1024-byte aligned (swizzle)
  uint32_t* smask = reinterpret_cast<uint32_t*>(slab + C::OFF_MASK);
  uint64_t* bar = reinterpret_cast<uint64_t*>(slab + C::OFF_BAR);
  const int tid = threadIdx.x;
  const uint32_t rows = (uint32_t)p.batch * (uint32_t)p.n_new * (uint32_t)p.n_kv;
  const uint32_t nb = (rows + C::NVB - 1) / C::NVB;  // chunks per tensor: K chunks 0 .. nb - 1, then V
  const uint32_t nchunks = 2 * nb;
  // Set-up that reads nothing another kernel writes: the barriers and the sign masks.
  if (tid == 0) {
#pragma unroll
    for (int st = 0; st < C::STAGES; ++st) mbar_init(&bar[st], 1);
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(&kin) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&vin) : "memory");
  }
  for (int i = tid; i < C::NMASK; i += kRowsThreads) {
    if constexpr (C::ESZ == 2) {
      const int e = 2 * i;  // elements e, e + 1: bits 15 and 31 of a word of two inputs
      const uint32_t two = (uint32_t)(p.sign_bits[e >> 6] >> (e & 63)) & 3u;
      smask[i] = ((two & 1u) << 15) | ((two >> 1) << 31);
    } else {
      smask[i] = ((uint32_t)(p.sign_bits[i >> 6] >> (i & 63)) & 1u) << 31;
    }
  }
  // Launched as a programmatic dependent of the previous kernel on the stream:
  // the input is read only after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  uint64_t pol = 0;
  // The block's k-th chunk is blockIdx.x + k * gridDim.x; it goes to stage k % STAGES
  // (that stage's (k / STAGES)-th phase), issued at the start for k < STAGES and in
  // iteration k - STAGES otherwise.
  auto issue = [&](uint32_t c, int st) {  // thread 0: chunk c into stage st
    const bool v = c >= nb;
    const uint32_t r0 = (c - (v ? nb : 0u)) * C::NVB;
    mbar_arrive_expect_tx(&bar[st], C::SLAB);
#pragma unroll
    for (int cc = 0; cc < C::NCOL; ++cc)
      tma_load_2d(slab + st * C::SLAB + cc * (C::NVB * 128), v ? &vin : &kin, &bar[st], cc * C::EPB, (int)r0, pol);
  };
  if (tid == 0) {
    pol = l2_policy_evict_first();
#pragma unroll
    for (int st = 0; st < C::STAGES; ++st) {
      const uint32_t c = blockIdx.x + (uint32_t)st * gridDim.x;
      if (c < nchunks) issue(c, st);
    }
  }
  __syncthreads();  // the barriers' initialisation and the masks are visible to every thread
  // thread -> (vector v of the chunk, part hv of the vector): the TPV parts of a vector
  // sit VPW lanes apart in one warp, so the cross-thread butterfly is one shuffle
  const int lane = tid & 31;
  const int hv = lane / C::VPW;
  const int v = (tid >> 5) * C::VPW + lane % C::VPW;
  int it = 0;
  for (uint32_t c = blockIdx.x; c < nchunks; c += gridDim.x, ++it) {
    const int st = it % C::STAGES;
    const bool ok = mbar_wait_bounded(&bar[st], (uint32_t)((it / C::STAGES) & 1), kRowsWaitNs);
    const int which = c >= nb ? 1 : 0;  // 0 = K, 1 = V
    const bool copy_k = which == 0 && p.k_f16;  // asymmetric cache: K kept as binary16, no transform
    float u[C::EPT];
    if (copy_k)
      load_row_raw<D, DT>(u, slab + st * C::SLAB, v, hv);
    else
      load_row_stage1<D, DT>(u, slab + st * C::SLAB, v, hv, smask);
    // every thread holds its elements: the stage takes the chunk after next (or the
    // block leaves together when a copy never landed)
    if (__syncthreads_or(!ok)) {
      if (tid == 0) {
        status_or(p.status, TQ_STATUS_TIMEOUT);
        // no copy may still be in flight at exit: wait for each stage's last issued
        // chunk (chunks 0 .. it + STAGES - 1 of this block have been issued)
#pragma unroll
        for (int s2 = 0; s2 < C::STAGES; ++s2) {
          int k = it + C::STAGES - 1;
          k -= ((k - s2) % C::STAGES + C::STAGES) % C::STAGES;
          while (k >= 0 && blockIdx.x + (uint32_t)k * gridDim.x >= nchunks) k -= C::STAGES;
          if (k >= 0) (void)mbar_wait_bounded(&bar[s2], (uint32_t)((k / C::STAGES) & 1), kRowsWaitNs);
        }
      }
      return;
    }
    if (tid == 0 && c + C::STAGES * gridDim.x < nchunks) issue(c + C::STAGES * gridDim.x, st);
    // Every thread runs the transform (the parts of a vector exchange through shuffles);
    // only valid vectors are stored.
    const uint32_t r = (c - (which ? nb : 0u)) * C::NVB + (uint32_t)v;
    bool valid = r < rows;
    const uint32_t rr = valid ? r : 0u;
    const uint32_t bt = fast_div(rr, p.div_kv);
    const int h = (int)(rr - bt * (uint32_t)p.n_kv);
    const uint32_t b_ = fast_div(bt, p.div_new);
    const int t = (int)(bt - b_ * (uint32_t)p.n_new);
    const int b = (int)b_;
    const int64_t pos = p.start_pos[b];
    if (valid && (pos < 0 || pos + p.n_new > p.max_seq)) {
      if (which == 0 && t == 0 && h == 0 && hv == 0) status_or(p.status, TQ_STATUS_CAPACITY);
      valid = false;
    }
    int64_t row = 0;
    if (valid) {
      bool row_ok;
      row = token_row(p, b, pos + t, row_ok) * p.n_kv + h;
      if (!row_ok) {  // an unmapped page: nothing is written
        if (hv == 0) status_or(p.status, TQ_STATUS_CAPACITY);
        valid = false;
      }
    }
    if (copy_k) {
      uint32_t w[C::EPT / 2];
      bool finite = true;
#pragma unroll
      for (int i = 0; i < C::EPT / 2; ++i) {
        const __half2 hh = __floats2half2_rn(u[2 * i], u[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&hh);
        finite = finite && ((w[i] & 0x7C00u) != 0x7C00u) && ((w[i] & 0x7C000000u) != 0x7C000000u);
      }
      if (!valid) continue;
      if (!finite) status_or(p.status, TQ_STATUS_NONFINITE);
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.k_codes) + row * D + hv * C::EPT);
#pragma unroll
      for (int j = 0; j < C::EPT / 8; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
      continue;
    }
    fwht_row_from2<C::EPT>(u);
#pragma unroll
    for (int hh = 1; hh < C::TPV; hh <<= 1) {  // strides EPT, 2 EPT, ...: between the parts
      const float sg = (hv & hh) ? -1.f : 1.f;  // upper part: lower - upper; lower part: lower + upper
#pragma unroll
      for (int i = 0; i < C::EPT; i += 2) {
        const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, u[i], hh * C::VPW),
                                     __shfl_xor_sync(0xffffffffu, u[i + 1], hh * C::VPW));
        const float2 n = __ffma2_rn(make_float2(u[i], u[i + 1]), f2(sg), o);
        u[i] = n.x;
        u[i + 1] = n.y;
      }
    }
    if (!valid) continue;
    const float* lam = which ? p.lambda_v : p.lambda_k;
    uint8_t* codes = (which ? p.v_codes : p.k_codes) + row * (D / 2) + hv * (C::EPT / 2);
    // scaling and the abs-max of the thread's groups, then each group's fast encoding
    // (no branch between groups, so their dependency chains interleave); a group that
    // needs the exact path is encoded and stored again afterwards (the later store of
    // the same thread to the same address wins)
    float amax[C::NGT];
#pragma unroll
    for (int g = 0; g < C::NGT; ++g) {
      float* y = u + 32 * g;
      float a = 0.f;
      if (lam != nullptr) {  // per-channel lambda between the transform and the abs-max
        const float4* l4 = reinterpret_cast<const float4*>(lam + hv * C::EPT + 32 * g);
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 lv = __ldg(l4 + i / 4);
          const float2 y0 =
              __fmul2_rn(__fmul2_rn(make_float2(y[i], y[i + 1]), f2(p.c_d)), make_float2(lv.x, lv.y));
          const float2 y1 =
              __fmul2_rn(__fmul2_rn(make_float2(y[i + 2], y[i + 3]), f2(p.c_d)), make_float2(lv.z, lv.w));
          y[i] = y0.x;
          y[i + 1] = y0.y;
          y[i + 2] = y1.x;
          y[i + 3] = y1.y;
          a = fmax_nan(a, fmax_nan(fmax_nan(fabsf(y0.x), fabsf(y0.y)), fmax_nan(fabsf(y1.x), fabsf(y1.y))));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 yv = __fmul2_rn(make_float2(y[i], y[i + 1]), f2(p.c_d));
          y[i] = yv.x;
          y[i + 1] = yv.y;
        }
        a = absmax32_nan(y);
      }
      amax[g] = a;
    }
    uint16_t sb[C::NGT];
    uint32_t redo = 0;
#pragma unroll
    for (int g = 0; g < C::NGT; ++g) {
      uint32_t packed[4];
      if (!encode_group_fast(u + 32 * g, amax[g], packed, sb[g])) redo |= 1u << g;
      *reinterpret_cast<uint4*>(codes + g * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    if (redo != 0) {
#pragma unroll
      for (int g = 0; g < C::NGT; ++g) {
        if (redo & (1u << g)) {
          uint32_t packed[4];
          sb[g] = encode_group(u + 32 * g, amax[g], packed, p.status);
          *reinterpret_cast<uint4*>(codes + g * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
    }
    uint16_t* scales = (which ? p.v_scales : p.k_scales) + row * NG + hv * C::NGT;
    if constexpr (C::NGT == 4) {
      *reinterpret_cast<uint2*>(scales) =
          make_uint2((uint32_t)sb[0] | ((uint32_t)sb[1] << 16), (uint32_t)sb[2] | ((uint32_t)sb[3] << 16));
    } else {
      static_assert(C::NGT == 2, "64 or 128 elements per thread");
      *reinterpret_cast<uint32_t*>(scales) = (uint32_t)sb[0] | ((uint32_t)sb[1] << 16);
    }
  }
}

// Dequantise one group per thread: yhat = code * scale (exact in binary32);
// with original_domain, the inverse rotation x = s o (c_D * H * yhat), the
// same butterfly order as the forward transform.
template <int D>
__global__ void __launch_bounds__(256) dequantize_kernel(const __grid_constant__ DequantParams p) {
  constexpr int NG = D / 32;
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t rows = (int64_t)p.batch * p.max_seq * p.n_kv;
  const int64_t row = gt / NG;
  const int part = (int)(gt % NG);
  const bool in_range = row < rows;
  bool live = false;
  if (in_range) {
    const int64_t bt = row / p.n_kv;
    const int tt = (int)(bt % p.max_seq);
    const int b = (int)(bt / p.max_seq);
    int len = p.seq_lens[b];
    if (len < 0 || len > p.max_seq) {
      if (tt == 0 && part == 0 && row % p.n_kv == 0) status_or(p.status, TQ_STATUS_CAPACITY);
      len = 0;
    }
    live = tt < len;
  }
  float u[32];
  if (live) {
    const uint4 w = *reinterpret_cast<const uint4*>(p.codes + row * (D / 2) + part * 16);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    const float sigma = __half2float(__ushort_as_half(p.scales[row * NG + part]));
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int nib = (int)((ww[i >> 3] >> (4 * (i & 7))) & 0xFu);
      const int c = (nib ^ 8) - 8;
      u[i] = __fmul_rn((float)c, sigma);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) u[i] = 0.f;
  }
  if (p.original_domain) {
    fwht_group<NG>(u, part);
#pragma unroll
    for (int i = 0; i < 32; ++i) u[i] = live ? apply_sign(__fmul_rn(u[i], p.c_d), p.sign_bits, part * 32 + i) : 0.f;
  }
  if (!in_range) return;
  float4* o = reinterpret_cast<float4*>(p.out + row * D + part * 32);
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j] = make_float4(u[4 * j], u[4 * j + 1], u[4 * j + 2], u[4 * j + 3]);
}

template <int D>
static cudaError_t launch_quantize_d(const QuantizeParams& p, cudaStream_t s) {
  const int64_t per_tensor = (int64_t)p.batch * p.n_new * p.n_kv * (D / 32);
  const int64_t per_v = (int64_t)p.batch * (p.n_new + p.tail_window) * p.n_kv * (D / 32);
  const int64_t threads = p.k_f16 ? (per_v + 31) / 32 * 32 + per_tensor : 2 * per_tensor;
  const int64_t blocks = (threads + 255) / 256;
  // programmatic dependent launch: set-up overlaps the previous kernel's tail,
  // griddepcontrol.wait in the kernel orders the reads
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_append_kernel<D>, p);
}

cudaError_t launch_quantize(const QuantizeParams& p, int D, cudaStream_t s) {
  switch (D) {
    case 32: return launch_quantize_d<32>(p, s);
    case 64: return launch_quantize_d<64>(p, s);
    case 128: return launch_quantize_d<128>(p, s);
    case 256: return launch_quantize_d<256>(p, s);
  }
  return cudaErrorInvalidValue;
}

template <int D, int DT>
static cudaError_t launch_rows_dt(const QuantizeParams& p, const TensorMap128& km, const TensorMap128& vm, int sms,
                                  cudaStream_t s) {
  using C = RowsCfg<D, DT>;
  static bool attr_set = false;  // per instantiation; the attribute is per function
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(quantize_rows_kernel<D, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  static int per_sm = 0;  // resident blocks per SM (registers and the two-stage slab)
  if (per_sm == 0) {
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_rows_kernel<D, DT>, kRowsThreads,
                                                                  C::SMEM);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
  }
  const uint32_t rows = (uint32_t)p.batch * (uint32_t)p.n_new * (uint32_t)p.n_kv;
  const uint32_t nchunks = 2u * ((rows + C::NVB - 1) / C::NVB);  // K chunks, then V chunks
  // persistent blocks: chunk c, c + grid, c + 2 grid, ... (each block streams its chunks
  // through the two-stage ring)
  const uint32_t resident = (uint32_t)per_sm * (uint32_t)(sms > 0 ? sms : 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nchunks < resident ? nchunks : resident);
  cfg.blockDim = dim3(kRowsThreads);
  cfg.dynamicSmemBytes = (size_t)C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const CUtensorMap& kmap = *reinterpret_cast<const CUtensorMap*>(&km);
  const CUtensorMap& vmap = *reinterpret_cast<const CUtensorMap*>(&vm);
  return cudaLaunchKernelEx(&cfg, quantize_rows_kernel<D, DT>, p, kmap, vmap);
}

template <int D>
static cudaError_t launch_rows_d(const QuantizeParams& p, const TensorMap128& km, const TensorMap128& vm, int sms,
                                 cudaStream_t s) {
  switch (p.in_dtype) {
    case TQ_BF16: return launch_rows_dt<D, TQ_BF16>(p, km, vm, sms, s);
    case TQ_F16: return launch_rows_dt<D, TQ_F16>(p, km, vm, sms, s);
    case TQ_F32: return launch_rows_dt<D, TQ_F32>(p, km, vm, sms, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_quantize_rows(const QuantizeParams& p, int D, const TensorMap128& km, const TensorMap128& vm,
                                 int sms, cudaStream_t s) {
  if (p.tail_window > 0) return cudaErrorInvalidValue;  // the delegated cache's fold stays on the group kernel
  switch (D) {
    case 64: return launch_rows_d<64>(p, km, vm, sms, s);
    case 128: return launch_rows_d<128>(p, km, vm, sms, s);
  }
  return cudaErrorInvalidValue;
}

template <int D>
static cudaError_t launch_dequant_d(const DequantParams& p, cudaStream_t s) {
  const int64_t threads = (int64_t)p.batch * p.max_seq * p.n_kv * (D / 32);
  const int64_t blocks = (threads + 255) / 256;
  dequantize_kernel<D><<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const DequantParams& p, int D, cudaStream_t s) {
  switch (D) {
    case 32: return launch_dequant_d<32>(p, s);
    case 64: return launch_dequant_d<64>(p, s);
    case 128: return launch_dequant_d<128>(p, s);
    case 256: return launch_dequant_d<256>(p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tqk
