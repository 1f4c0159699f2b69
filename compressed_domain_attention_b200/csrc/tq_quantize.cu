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
