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

template <int D>
__global__ void __launch_bounds__(256) quantize_append_kernel(QuantizeParams p) {
  constexpr int NG = D / 32;
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t vecs_per_tensor = (int64_t)p.batch * p.n_new * p.n_kv;
  const int64_t vec = gt / NG;
  const int part = (int)(gt % NG);
  const bool in_range = vec < 2 * vecs_per_tensor;
  const int which = in_range ? (int)(vec / vecs_per_tensor) : 0;  // 0 = K, 1 = V
  const int64_t r = in_range ? vec % vecs_per_tensor : 0;
  const int h = (int)(r % p.n_kv);
  const int64_t bt = r / p.n_kv;
  const int t = (int)(bt % p.n_new);
  const int b = (int)(bt / p.n_new);

  // the input rows and the start position are independent loads: issue both first
  float u[32];
  int64_t pos = 0;
  if (in_range) {
    load32(u, which ? p.v : p.k, r * D + part * 32, p.in_dtype);
    pos = p.start_pos[b];
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) u[i] = 0.f;
  }
  bool valid = in_range;
  if (in_range && (pos < 0 || pos + p.n_new > p.max_seq)) {
    valid = false;
    if (which == 0 && t == 0 && h == 0 && part == 0) status_or(p.status, TQ_STATUS_CAPACITY);
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) u[i] = apply_sign(u[i], p.sign_bits, part * 32 + i);
  fwht_group<NG>(u, part);  // all lanes participate (shuffles)

  bool finite = true;
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    u[i] = __fmul_rn(u[i], p.c_d);
    finite = finite && (fabsf(u[i]) <= 3.402823466e38f);
    a = fmaxf(a, fabsf(u[i]));
  }
  if (!valid) return;

  const float sigma32 = __fdiv_rn(a, 7.0f);
  const __half sig16 = __float2half_rn(sigma32);
  const float sigma = __half2float(sig16);
  uint16_t sbits = __half_as_ushort(sig16);
  uint32_t packed[4] = {0u, 0u, 0u, 0u};
  if (!finite || !(fabsf(sigma) <= 65504.f)) {
    sbits = 0x7C00u;
    status_or(p.status, TQ_STATUS_NONFINITE);
  } else if (sigma != 0.f) {
    // code = rint(fl(y / sigma)). With inv = RN(1/sigma) and r = RN(y * inv),
    // |r - y/sigma| <= 2^-23 |y/sigma| <= 2^-20 (|y/sigma| <= 7 * (1 + 2^-11) < 8), and
    // |fl(y/sigma) - y/sigma| <= 2^-21. So when r is more than 2^-19 away from every
    // half-integer, y/sigma and fl(y/sigma) are more than 2^-21 away from it too and
    // both round to rint(r). Otherwise (probability about 2^-18 per element) the IEEE
    // division is taken. The result is the same code as the plain definition.
    const float inv = __frcp_rn(sigma);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float r = __fmul_rn(u[i], inv);
      const float rr = rintf(r);
      int c = (int)rr;
      if (fabsf(fabsf(r - rr) - 0.5f) <= 1.9073486328125e-06f)  // 2^-19
        c = __float2int_rn(__fdiv_rn(u[i], sigma));
      c = max(-7, min(7, c));
      packed[i >> 3] |= ((uint32_t)c & 0xFu) << (4 * (i & 7));
    }
  }
  const int64_t row = ((int64_t)b * p.max_seq + pos + t) * p.n_kv + h;
  uint8_t* codes = which ? p.v_codes : p.k_codes;
  uint16_t* scales = which ? p.v_scales : p.k_scales;
  *reinterpret_cast<uint4*>(codes + row * (D / 2) + part * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  scales[row * NG + part] = sbits;
}

// Dequantise one group per thread: yhat = code * scale (exact in binary32);
// with original_domain, the inverse rotation x = s o (c_D * H * yhat), the
// same butterfly order as the forward transform.
template <int D>
__global__ void __launch_bounds__(256) dequantize_kernel(DequantParams p) {
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
  const int64_t threads = 2LL * p.batch * p.n_new * p.n_kv * (D / 32);
  const int64_t blocks = (threads + 255) / 256;
  quantize_append_kernel<D><<<(unsigned)blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
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
