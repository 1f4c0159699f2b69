// Plain CPU oracle for rotation-based int4 KV-cache quantisation and decode
// attention on the packed cache.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call
// this file; only the tests, the smoke check and the benchmark's CPU-baseline
// leg do. It shares no code, header, table or constant with the CUDA library:
// every constant below is computed here from its definition.
//
// Sources (web pages on the method; cited by title and section):
//  [OTQ-A] "Open-TQ-Metal: Fused Compressed-Domain Attention for Long-Context
//          LLM Inference on Apple Silicon", abstract as shown on the
//          thelatestinai.com cards page: the fused quantiser is a
//          sign-randomised transform, per-group abs-max scaling and int4 nibble
//          packing; SRFT and SRHT are said to be indistinguishable in quality.
//  [OTQ-B] the same paper, arXiv abstract on the mlsanity.com index page:
//          attention is computed directly on the compressed representation,
//          with no intermediate dequantised matrices; the attention scale
//          factor (standard 1/sqrt(d) vs 1.0) is a model property.
//  [OTQ-refs] the same index page, "Builds on": online normaliser for softmax;
//          grouped-query attention.
//  [MLX]   mlxcel user guide, "TurboQuant KV cache compression": §"What
//          TurboQuant changes" (a Walsh-Hadamard rotation first, then low-bit
//          storage, unpacked when attention reads it); §"Known limitations /
//          head dimension" (power-of-two head dims only).
//  [MLX-modes] the same guide, §"Cache modes" and §"What TurboQuant changes":
//          the recommended default mode (fp16+turbo4) keeps K in FP16 and
//          compresses only V, because K decides where attention looks.
//  [MLX-deleg] the same guide, §"Cache modes" (turbo4-delegated row: K in FP16,
//          V as an FP16 hot tail plus a Turbo4 cold body) and §"Delegated cache
//          variant" (recent tokens stay FP16, older V tokens are stored in the
//          4-bit form; the FP16 sidecars are folded into it).
//  [OTQ-lam] the Open-TQ-Metal abstract's list of the fused kernel's steps:
//          sign-randomised transform, per-channel lambda, per-group abs-max,
//          int4 pack (lambda sits between the transform and the abs-max).
//  [MLX-sparse] the mlxcel guide, §"Sparse-V dequant threshold": V dequant may
//          be skipped where the attention weight is below a threshold (1e-6).
//  [MLX-paged] the same guide, §"Known limitations / paged KV scheduler": a
//          paged decode storage backend (it cites PagedAttention).
//  [AMD]   "TurboQuant on AMD GPUs" (oracore.dev), §4: Walsh-Hadamard spreads
//          energy evenly and suits kernels better than a dense random rotation.
//
// Where the pages leave a step open the reading taken is stated at that step.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -shared -fPIC.
// No FMA contraction: every fl(.) below is one IEEE binary32 operation.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ---- status bits (oracle-local numbering, mirrored by value in the tests) ----
constexpr int32_t ORC_STATUS_NONFINITE = 1;  // a group held a non-finite value or its scale overflowed fp16
constexpr int32_t ORC_STATUS_CAPACITY = 2;   // an append would run past max_seq, or a length exceeds it

// ---- SplitMix64 (S. Vigna's public-domain generator) -------------------------
// Reading of "fixed seeded +-1 diagonal": state = seed; for i = 0..D-1 draw
// r = next(); s_i = -1 if the top bit of r is set, else +1. One vector per D,
// shared by K, V, q, every head and every layer.
uint64_t splitmix64_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ULL;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// ---- IEEE 754 binary32 -> binary16, round to nearest, ties to even ----------
// Written from the format definitions: binary16 has 5 exponent bits (bias 15)
// and 10 fraction bits; subnormals step by 2^-24.
uint16_t f32_to_f16_rne(float f) {
  uint32_t x;
  std::memcpy(&x, &f, 4);
  const uint32_t sign = (x >> 16) & 0x8000u;
  const uint32_t ebits = (x >> 23) & 0xFFu;
  const uint32_t frac = x & 0x7FFFFFu;
  if (ebits == 0xFFu) {  // inf / NaN
    if (frac == 0) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | 0x7E00u | (frac >> 13));  // quiet NaN
  }
  const int e = (int)ebits - 127;
  if (e > 15) return (uint16_t)(sign | 0x7C00u);  // |f| >= 2^16: overflow
  if (e >= -14) {                                  // binary16 normal range
    uint32_t h = ((uint32_t)(e + 15) << 10) | (frac >> 13);
    const uint32_t rem = frac & 0x1FFFu;
    if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u;  // a carry may reach +inf: correct
    return (uint16_t)(sign | h);
  }
  if (e < -25) return (uint16_t)sign;  // below half the smallest subnormal (and binary32 subnormals)
  // binary16 subnormal: value / 2^-24 = (frac | 2^23) * 2^(e+1)
  const uint32_t sig = frac | 0x800000u;
  const int shift = -(e + 1);  // 14..24
  uint32_t h = sig >> shift;
  const uint32_t rem = sig & ((1u << shift) - 1u);
  const uint32_t half = 1u << (shift - 1);
  if (rem > half || (rem == half && (h & 1u))) h += 1u;
  return (uint16_t)(sign | h);
}

float f16_to_f32(uint16_t h) {
  const uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
  const uint32_t ebits = (h >> 10) & 0x1Fu;
  const uint32_t frac = h & 0x3FFu;
  if (ebits == 0x1Fu) {
    const uint32_t x = sign | 0x7F800000u | (frac << 13);
    float f;
    std::memcpy(&f, &x, 4);
    return f;
  }
  if (ebits == 0) {  // zero or subnormal: frac * 2^-24, exact in binary32
    const float mag = std::ldexp((float)frac, -24);
    return sign ? -mag : mag;
  }
  const uint32_t x = sign | ((ebits - 15 + 127) << 23) | (frac << 13);
  float f;
  std::memcpy(&f, &x, 4);
  return f;
}

// ---- orthonormal Walsh-Hadamard transform -----------------------------------
// [MLX] §"What TurboQuant changes", [AMD] §4. Butterfly order (a reading: the
// pages give none): radix-2 stages with stride h = 1, 2, 4, ..., D/2; within a
// stage every pair (i, i+h) with (i & h) == 0 becomes (u_i + u_{i+h}, u_i - u_{i+h}),
// natural (Sylvester) ordering. The transform is left unnormalised here.
void fwht_unnormalised(float* u, int D) {
  for (int h = 1; h < D; h <<= 1) {
    for (int i = 0; i < D; ++i) {
      if ((i & h) != 0) continue;
      const float a = u[i];
      const float b = u[i + h];
      u[i] = a + b;
      u[i + h] = a - b;
    }
  }
}

// Orthonormal scale c_D = 1/sqrt(D), rounded once to binary32, applied once
// after all butterfly stages (reading of "orthonormal").
float norm_const(int D) { return (float)(1.0 / std::sqrt((double)D)); }

// SRHT forward: y = c_D * H * (s o x). [OTQ-A] "sign-randomized" transform,
// Hadamard variant (SRHT) per [OTQ-A]'s equivalence statement.
void srht_forward_vec(const float* x, const float* s, int D, float* y) {
  std::vector<float> u(D);
  for (int i = 0; i < D; ++i) u[i] = s[i] * x[i];  // exact: a sign flip
  fwht_unnormalised(u.data(), D);
  const float c = norm_const(D);
  for (int i = 0; i < D; ++i) y[i] = u[i] * c;
}

// SRHT inverse: x = s o (c_D * H * y), the transpose of the forward map
// (H is symmetric, c_D*H orthonormal, s o s = 1).
void srht_inverse_vec(const float* y, const float* s, int D, float* x) {
  std::vector<float> u(y, y + D);
  fwht_unnormalised(u.data(), D);
  const float c = norm_const(D);
  for (int i = 0; i < D; ++i) x[i] = s[i] * (u[i] * c);
}

// ---- per-group abs-max int4 quantiser ---------------------------------------
// [OTQ-A]: per-group abs-max + int4. Group = 32 consecutive elements of the
// rotated vector. Readings: scale_32 = fl(absmax / 7); the stored scale is
// its binary16 rounding (RNE); codes are taken against the STORED scale:
// code = clamp(rint_even(fl(y / sigma)), -7, 7). An all-zero group (or one
// whose scale underflows binary16) stores scale +0 and codes 0. A group with a
// non-finite value, or whose scale overflows binary16, stores scale +inf
// (0x7C00), codes 0, and raises ORC_STATUS_NONFINITE.
int32_t quantize_rotated(const float* y, int D, int8_t* codes, uint16_t* scales) {
  int32_t status = 0;
  const int n_groups = D / 32;
  for (int g = 0; g < n_groups; ++g) {
    const float* yg = y + 32 * g;
    bool finite = true;
    float a = 0.0f;
    for (int i = 0; i < 32; ++i) {
      if (!std::isfinite(yg[i])) finite = false;
      const float m = std::fabs(yg[i]);
      if (m > a) a = m;
    }
    const float sigma32 = a / 7.0f;
    const uint16_t sigma16 = f32_to_f16_rne(sigma32);
    const float sigma = f16_to_f32(sigma16);
    if (!finite || !std::isfinite(sigma)) {
      status |= ORC_STATUS_NONFINITE;
      scales[g] = 0x7C00u;
      for (int i = 0; i < 32; ++i) codes[32 * g + i] = 0;
      continue;
    }
    scales[g] = sigma16;
    if (sigma == 0.0f) {
      for (int i = 0; i < 32; ++i) codes[32 * g + i] = 0;
      continue;
    }
    for (int i = 0; i < 32; ++i) {
      const float r = yg[i] / sigma;
      float c = std::nearbyint(r);  // default rounding mode: nearest, ties to even
      if (c > 7.0f) c = 7.0f;
      if (c < -7.0f) c = -7.0f;
      codes[32 * g + i] = (int8_t)c;
    }
  }
  return status;
}

// ---- nibble packing ----------------------------------------------------------
// [OTQ-A] "int4 nibble pack". Reading: two's-complement nibbles, byte j holds
// element 2j in its low nibble and element 2j+1 in its high nibble.
void pack_codes(const int8_t* codes, int D, uint8_t* bytes) {
  for (int j = 0; j < D / 2; ++j) {
    const uint8_t lo = (uint8_t)codes[2 * j] & 0x0Fu;
    const uint8_t hi = (uint8_t)codes[2 * j + 1] & 0x0Fu;
    bytes[j] = (uint8_t)(lo | (hi << 4));
  }
}

int8_t nibble_to_int(uint8_t n) {  // 4-bit two's complement
  return (int8_t)((n & 0x8u) ? (int)n - 16 : (int)n);
}

void unpack_codes(const uint8_t* bytes, int D, int8_t* codes) {
  for (int j = 0; j < D / 2; ++j) {
    codes[2 * j] = nibble_to_int(bytes[j] & 0x0Fu);
    codes[2 * j + 1] = nibble_to_int((uint8_t)(bytes[j] >> 4));
  }
}

// Dequantised rotated vector: yhat_i = code_i * sigma_g (exact in binary32).
void dequantize_rotated(const uint8_t* bytes, const uint16_t* scales, int D, float* yhat) {
  std::vector<int8_t> codes(D);
  unpack_codes(bytes, D, codes.data());
  for (int i = 0; i < D; ++i) yhat[i] = (float)codes[i] * f16_to_f32(scales[i / 32]);
}

// [MLX-modes] binary16 (round to nearest even) of one K row; a non-finite
// result raises ORC_STATUS_NONFINITE (its bits are stored as converted).
int32_t store_k_f16(const float* x, int D, uint16_t* dst) {
  int32_t st = 0;
  for (int i = 0; i < D; ++i) {
    const uint16_t hbits = f32_to_f16_rne(x[i]);
    if ((hbits & 0x7C00u) == 0x7C00u) st |= ORC_STATUS_NONFINITE;
    dst[i] = hbits;
  }
  return st;
}

// ---- delegated hot/cold cache [MLX-deleg] ----
// Reading taken (the guide names the parts, not the policy): the hot tail holds
// the most recent tokens' V in binary16, at most W of them, in a ring of W slots
// per (sequence, kv head), token t in slot t mod W. Tokens leave it oldest first,
// F at a time: a sequence of len tokens has cold_length(len) tokens in the int4
// body, so that W - F < len - cold_length(len) <= W once len > W.
int64_t cold_length(int64_t len, int W, int F) {
  if (len <= W) return 0;
  return (len - W + F - 1) / F * F;
}

// The decode steps shared by the three cache formats. k_f16 == nullptr: int4 K
// (scores against SRHT(q)); otherwise binary16 K (scores against q). v_tail ==
// nullptr: every V token is int4; otherwise tokens t >= cold_length(len_b)
// take their binary16 tail value, mapped to the rotated domain by the forward
// SRHT so that the weighted sum stays in one domain (the transform is linear).
// Optional [OTQ-lam] lambda_k / lambda_v (nullptr = identity): the stored codes
// encode lambda o y, so the rotated-domain value is (code * sigma) / lambda,
// taken in binary64 here. Optional [MLX-sparse] threshold tau > 0: the V term
// of token t is dropped when exp(z_t - max z) < tau (its weight relative to
// the largest score); the softmax sum keeps every token. `bound` (nullable)
// receives, per output element, sum over dropped t of w_t |V_t,i| in the
// original domain (w_t the exact normalised weight), which bounds the change
// any rule that drops a subset of those tokens can make.
int32_t decode_body(int batch, int max_seq, int n_kv, int n_q, int D, const float* s, const float* q,
                    const int32_t* seq_lens, const uint8_t* k_codes, const uint16_t* k_scales,
                    const uint16_t* k_f16, const uint8_t* v_codes, const uint16_t* v_scales,
                    const uint16_t* v_tail, int W, int F, float sm_scale, const uint8_t* which, float* out,
                    const float* lambda_k = nullptr, const float* lambda_v = nullptr, double tau = 0.0,
                    float* bound = nullptr) {
  int32_t st = 0;
  const int G = n_q / n_kv;
  const int64_t cb = D / 2, sb = D / 32;
  std::vector<float> qr(D), yk(D), yv(D), xv(D), o32(D), xb(D);
  std::vector<double> z, acc(D), bnd(D);
  for (int b = 0; b < batch; ++b) {
    const int len = seq_lens[b];
    const int64_t n_cold = v_tail ? cold_length(len, W, F) : len;
    for (int hq = 0; hq < n_q; ++hq) {
      if (which && !which[(int64_t)b * n_q + hq]) continue;
      float* o = out + ((int64_t)b * n_q + hq) * D;
      if (len <= 0 || len > max_seq) {
        if (len > max_seq) st |= ORC_STATUS_CAPACITY;
        for (int i = 0; i < D; ++i) o[i] = 0.0f;
        if (bound)
          for (int i = 0; i < D; ++i) bound[((int64_t)b * n_q + hq) * D + i] = 0.0f;
        continue;
      }
      const int kv = hq / G;
      // int4 K lives in the rotated domain and pairs with SRHT(q); binary16 K
      // (asymmetric cache) is in the original domain and pairs with q itself
      if (k_f16)
        std::memcpy(qr.data(), q + ((int64_t)b * n_q + hq) * D, sizeof(float) * D);
      else
        srht_forward_vec(q + ((int64_t)b * n_q + hq) * D, s, D, qr.data());
      z.assign(len, 0.0);
      for (int t = 0; t < len; ++t) {
        const int64_t row = ((int64_t)b * max_seq + t) * n_kv + kv;
        if (k_f16) {
          for (int i = 0; i < D; ++i) yk[i] = f16_to_f32(k_f16[row * D + i]);
        } else {
          dequantize_rotated(k_codes + row * cb, k_scales + row * sb, D, yk.data());
        }
        double dot = 0.0;
        if (lambda_k && !k_f16) {
          for (int i = 0; i < D; ++i) dot += (double)qr[i] * ((double)yk[i] / (double)lambda_k[i]);
        } else {
          for (int i = 0; i < D; ++i) dot += (double)qr[i] * (double)yk[i];
        }
        z[t] = (double)sm_scale * dot;
      }
      double m = z[0];
      for (int t = 1; t < len; ++t)
        if (z[t] > m) m = z[t];
      double l = 0.0;
      for (int t = 0; t < len; ++t) {
        z[t] = std::exp(z[t] - m);
        l += z[t];
      }
      for (int i = 0; i < D; ++i) acc[i] = 0.0;
      for (int i = 0; i < D; ++i) bnd[i] = 0.0;
      for (int t = 0; t < len; ++t) {
        const int64_t row = ((int64_t)b * max_seq + t) * n_kv + kv;
        // z[t] holds exp(z_t - max z) here: the weight relative to the largest score
        const bool dropped = tau > 0.0 && t < n_cold && z[t] < tau;
        if (dropped) {
          if (bound) {  // the dropped token's V in the original domain
            dequantize_rotated(v_codes + row * cb, v_scales + row * sb, D, xb.data());
            if (lambda_v)
              for (int i = 0; i < D; ++i) xb[i] = (float)((double)xb[i] / (double)lambda_v[i]);
            srht_inverse_vec(xb.data(), s, D, xv.data());
            for (int i = 0; i < D; ++i) bnd[i] += z[t] / l * std::fabs((double)xv[i]);
          }
          continue;
        }
        if (t < n_cold) {
          dequantize_rotated(v_codes + row * cb, v_scales + row * sb, D, yv.data());
        } else {
          const uint16_t* hot = v_tail + (((int64_t)b * W + t % W) * n_kv + kv) * D;
          for (int i = 0; i < D; ++i) xv[i] = f16_to_f32(hot[i]);
          srht_forward_vec(xv.data(), s, D, yv.data());
        }
        const double w = z[t] / l;
        if (lambda_v && t < n_cold) {
          for (int i = 0; i < D; ++i) acc[i] += w * ((double)yv[i] / (double)lambda_v[i]);
        } else {
          for (int i = 0; i < D; ++i) acc[i] += w * (double)yv[i];
        }
      }
      for (int i = 0; i < D; ++i) o32[i] = (float)acc[i];
      srht_inverse_vec(o32.data(), s, D, o);
      if (bound)
        for (int i = 0; i < D; ++i) bound[((int64_t)b * n_q + hq) * D + i] = (float)bnd[i];
    }
  }
  return st;
}



}  // namespace

extern "C" {

// Status bit values, exported so the tests can read them.
int32_t oracle_status_nonfinite() { return ORC_STATUS_NONFINITE; }
int32_t oracle_status_capacity() { return ORC_STATUS_CAPACITY; }

void oracle_splitmix64(uint64_t seed, int n, uint64_t* out) {
  uint64_t st = seed;
  for (int i = 0; i < n; ++i) out[i] = splitmix64_next(st);
}

void oracle_sign_vector(uint64_t seed, int D, float* s) {
  uint64_t st = seed;
  for (int i = 0; i < D; ++i) s[i] = (splitmix64_next(st) >> 63) ? -1.0f : 1.0f;
}

float oracle_norm_const(int D) { return norm_const(D); }

void oracle_f32_to_f16(const float* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = f32_to_f16_rne(x[i]);
}

void oracle_f16_to_f32(const uint16_t* h, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = f16_to_f32(h[i]);
}

void oracle_fwht(float* u, int D, int64_t n_vec) {
  for (int64_t v = 0; v < n_vec; ++v) fwht_unnormalised(u + v * D, D);
}

void oracle_srht_forward(const float* x, const float* s, int D, int64_t n_vec, float* y) {
  for (int64_t v = 0; v < n_vec; ++v) srht_forward_vec(x + v * D, s, D, y + v * D);
}

void oracle_srht_inverse(const float* y, const float* s, int D, int64_t n_vec, float* x) {
  for (int64_t v = 0; v < n_vec; ++v) srht_inverse_vec(y + v * D, s, D, x + v * D);
}

// Quantise already-rotated vectors: codes as int8 (one per element), scales as binary16 bits.
int32_t oracle_quantize_rotated(const float* y, int D, int64_t n_vec, int8_t* codes, uint16_t* scales) {
  int32_t st = 0;
  for (int64_t v = 0; v < n_vec; ++v) st |= quantize_rotated(y + v * D, D, codes + v * D, scales + v * (D / 32));
  return st;
}

void oracle_pack(const int8_t* codes, int D, int64_t n_vec, uint8_t* bytes) {
  for (int64_t v = 0; v < n_vec; ++v) pack_codes(codes + v * D, D, bytes + v * (D / 2));
}

void oracle_unpack(const uint8_t* bytes, int D, int64_t n_vec, int8_t* codes) {
  for (int64_t v = 0; v < n_vec; ++v) unpack_codes(bytes + v * (D / 2), D, codes + v * D);
}

// Full encoding of raw vectors: SRHT, quantise, pack.
int32_t oracle_encode(const float* x, const float* s, int D, int64_t n_vec, uint8_t* bytes, uint16_t* scales) {
  std::vector<float> y(D);
  std::vector<int8_t> codes(D);
  int32_t st = 0;
  for (int64_t v = 0; v < n_vec; ++v) {
    srht_forward_vec(x + v * D, s, D, y.data());
    st |= quantize_rotated(y.data(), D, codes.data(), scales + v * (D / 32));
    pack_codes(codes.data(), D, bytes + v * (D / 2));
  }
  return st;
}

// Append n_new tokens per sequence into caches laid out as
//   codes  [batch][max_seq][n_kv][D/2]  bytes
//   scales [batch][max_seq][n_kv][D/32] binary16
// from inputs k, v [batch][n_new][n_kv][D] (binary32; bf16/fp16 inputs are
// widened exactly by the caller). Token t of sequence b lands at position
// start_pos[b] + t. A sequence whose append would not fit is skipped and
// raises ORC_STATUS_CAPACITY.
int32_t oracle_quantize_append(int batch, int max_seq, int n_kv, int D, const float* s,
                               const float* k, const float* v, int n_new, const int32_t* start_pos,
                               uint8_t* k_codes, uint16_t* k_scales, uint8_t* v_codes, uint16_t* v_scales) {
  int32_t st = 0;
  const int64_t cb = D / 2, sb = D / 32;
  for (int b = 0; b < batch; ++b) {
    const int64_t p0 = start_pos[b];
    if (p0 < 0 || p0 + n_new > max_seq) {
      st |= ORC_STATUS_CAPACITY;
      continue;
    }
    for (int t = 0; t < n_new; ++t) {
      for (int h = 0; h < n_kv; ++h) {
        const int64_t src = (((int64_t)b * n_new + t) * n_kv + h) * D;
        const int64_t row = ((int64_t)b * max_seq + p0 + t) * n_kv + h;
        st |= oracle_encode(k + src, s, D, 1, k_codes + row * cb, k_scales + row * sb);
        st |= oracle_encode(v + src, s, D, 1, v_codes + row * cb, v_scales + row * sb);
      }
    }
  }
  return st;
}

// Decode attention over the packed cache, one query token per sequence.
//   q   [batch][n_q][D] binary32;  out [batch][n_q][D] binary32, original domain.
// GQA map kv = hq / (n_q / n_kv) ([OTQ-refs] grouped-query attention).
// Steps ([OTQ-B]: attention on the compressed representation; the rotation is
// orthogonal, so q.k and sum p.v carry over to the rotated domain):
//  1. q_r = SRHT(q) in binary32, the same steps as the encoder;
//  2. z_t = sm_scale * sum_i q_r,i * yhatK_t,i over t < len_b, accumulated in
//     binary64 (yhat = code * sigma is exact);
//  3. exact two-pass softmax in binary64;
//  4. o~_i = sum_t w_t * yhatV_t,i in binary64, rounded once to binary32;
//  5. out = SRHT^-1(o~) in binary32.
// len_b == 0 gives out = 0. len_b > max_seq raises ORC_STATUS_CAPACITY and
// leaves that sequence's output at 0. `which` (nullable, [batch][n_q]) limits
// the work to the flagged (b, hq) pairs; unflagged outputs are left untouched.
int32_t oracle_decode_attention(int batch, int max_seq, int n_kv, int n_q, int D, const float* s,
                                const float* q, const int32_t* seq_lens,
                                const uint8_t* k_codes, const uint16_t* k_scales,
                                const uint8_t* v_codes, const uint16_t* v_scales,
                                float sm_scale, const uint8_t* which, float* out) {
  return decode_body(batch, max_seq, n_kv, n_q, D, s, q, seq_lens, k_codes, k_scales, nullptr, v_codes, v_scales,
                     nullptr, 0, 0, sm_scale, which, out);
}

// ---- asymmetric cache: K in binary16, V as int4 codes [MLX-modes] ----
// Reading taken: K is stored as the binary16 (round to nearest even) of the
// input element in the ORIGINAL domain (no rotation: nothing is quantised, so
// the rotation has no job on K), layout [batch][max_seq][n_kv][D]; V is encoded
// exactly as in oracle_quantize_append. A K element whose binary16 is not
// finite raises ORC_STATUS_NONFINITE (its bits are stored as converted).
int32_t oracle_quantize_append_kf16(int batch, int max_seq, int n_kv, int D, const float* s,
                                    const float* k, const float* v, int n_new, const int32_t* start_pos,
                                    uint16_t* k_f16, uint8_t* v_codes, uint16_t* v_scales) {
  int32_t st = 0;
  const int64_t cb = D / 2, sb = D / 32;
  for (int b = 0; b < batch; ++b) {
    const int64_t p0 = start_pos[b];
    if (p0 < 0 || p0 + n_new > max_seq) {
      st |= ORC_STATUS_CAPACITY;
      continue;
    }
    for (int t = 0; t < n_new; ++t) {
      for (int h = 0; h < n_kv; ++h) {
        const int64_t src = (((int64_t)b * n_new + t) * n_kv + h) * D;
        const int64_t row = ((int64_t)b * max_seq + p0 + t) * n_kv + h;
        st |= store_k_f16(k + src, D, k_f16 + row * D);
        st |= oracle_encode(v + src, s, D, 1, v_codes + row * cb, v_scales + row * sb);
      }
    }
  }
  return st;
}

// Decode attention over the asymmetric cache: the same steps as
// oracle_decode_attention, except that the scores pair q itself with the binary16
// K values (both in the original domain); the values are still the
// rotated-domain V, mapped back by SRHT^-1 after the weighted sum.
int32_t oracle_decode_attention_kf16(int batch, int max_seq, int n_kv, int n_q, int D, const float* s,
                                     const float* q, const int32_t* seq_lens, const uint16_t* k_f16,
                                     const uint8_t* v_codes, const uint16_t* v_scales, float sm_scale,
                                     const uint8_t* which, float* out) {
  return decode_body(batch, max_seq, n_kv, n_q, D, s, q, seq_lens, nullptr, nullptr, k_f16, v_codes, v_scales,
                     nullptr, 0, 0, sm_scale, which, out);
}

// [OTQ-lam] encoding with a per-channel lambda: y = SRHT(x), then
// y_i <- fl(y_i * lambda_i) (one binary32 multiply), then quantise and pack.
// lambda == nullptr is the identity (oracle_encode).
int32_t oracle_encode_lambda(const float* x, const float* s, const float* lambda, int D, int64_t n_vec,
                             uint8_t* bytes, uint16_t* scales) {
  std::vector<float> y(D);
  std::vector<int8_t> codes(D);
  int32_t st = 0;
  for (int64_t v = 0; v < n_vec; ++v) {
    srht_forward_vec(x + v * D, s, D, y.data());
    if (lambda)
      for (int i = 0; i < D; ++i) y[i] = y[i] * lambda[i];
    st |= quantize_rotated(y.data(), D, codes.data(), scales + v * (D / 32));
    pack_codes(codes.data(), D, bytes + v * (D / 2));
  }
  return st;
}

// oracle_quantize_append with per-channel lambda vectors for K and V (nullable).
int32_t oracle_quantize_append_lambda(int batch, int max_seq, int n_kv, int D, const float* s, const float* k,
                                      const float* v, int n_new, const int32_t* start_pos, const float* lambda_k,
                                      const float* lambda_v, uint8_t* k_codes, uint16_t* k_scales,
                                      uint8_t* v_codes, uint16_t* v_scales) {
  int32_t st = 0;
  const int64_t cb = D / 2, sb = D / 32;
  for (int b = 0; b < batch; ++b) {
    const int64_t p0 = start_pos[b];
    if (p0 < 0 || p0 + n_new > max_seq) {
      st |= ORC_STATUS_CAPACITY;
      continue;
    }
    for (int t = 0; t < n_new; ++t) {
      for (int h = 0; h < n_kv; ++h) {
        const int64_t src = (((int64_t)b * n_new + t) * n_kv + h) * D;
        const int64_t row = ((int64_t)b * max_seq + p0 + t) * n_kv + h;
        st |= oracle_encode_lambda(k + src, s, lambda_k, D, 1, k_codes + row * cb, k_scales + row * sb);
        st |= oracle_encode_lambda(v + src, s, lambda_v, D, 1, v_codes + row * cb, v_scales + row * sb);
      }
    }
  }
  return st;
}

// Decode with the optional extensions: lambda_k (int4 K only) and lambda_v
// [OTQ-lam], the sparse-V threshold tau [MLX-sparse] and its error bound (see
// decode_body). k_f16 != nullptr selects the asymmetric cache (k_codes and
// k_scales unused).
int32_t oracle_decode_attention_ext(int batch, int max_seq, int n_kv, int n_q, int D, const float* s,
                                    const float* q, const int32_t* seq_lens, const uint8_t* k_codes,
                                    const uint16_t* k_scales, const uint16_t* k_f16, const uint8_t* v_codes,
                                    const uint16_t* v_scales, const float* lambda_k, const float* lambda_v,
                                    float sm_scale, double tau, const uint8_t* which, float* out, float* bound) {
  return decode_body(batch, max_seq, n_kv, n_q, D, s, q, seq_lens, k_codes, k_scales, k_f16, v_codes, v_scales,
                     nullptr, 0, 0, sm_scale, which, out, lambda_k, lambda_v, tau, bound);
}

// ---- paged storage [MLX-paged] ----
// Reading taken: a paged cache holds the same rows as the contiguous one, placed
// in a pool of n_pages pages of P tokens; token t of sequence b sits at pool row
// table[b * max_pages + t / P] * P + t % P. Rows are [n_kv][...] as before. An
// entry outside [0, n_pages) is an unmapped page: appends to it are skipped and
// raise ORC_STATUS_CAPACITY. k_f16 != nullptr selects binary16 K (k_codes and
// k_scales unused), as in the asymmetric cache.
int32_t oracle_quantize_append_paged(int batch, int max_seq, int n_kv, int D, const float* s, const float* k,
                                     const float* v, int n_new, const int32_t* start_pos, const int32_t* table,
                                     int P, int max_pages, int n_pages, uint8_t* k_codes, uint16_t* k_scales,
                                     uint16_t* k_f16, uint8_t* v_codes, uint16_t* v_scales) {
  int32_t st = 0;
  const int64_t cb = D / 2, sb = D / 32;
  for (int b = 0; b < batch; ++b) {
    const int64_t p0 = start_pos[b];
    if (p0 < 0 || p0 + n_new > max_seq) {
      st |= ORC_STATUS_CAPACITY;
      continue;
    }
    for (int t = 0; t < n_new; ++t) {
      const int64_t pos = p0 + t;
      const int pg = table[(int64_t)b * max_pages + pos / P];
      if (pg < 0 || pg >= n_pages) {
        st |= ORC_STATUS_CAPACITY;
        continue;
      }
      const int64_t prow = (int64_t)pg * P + pos % P;
      for (int h = 0; h < n_kv; ++h) {
        const int64_t src = (((int64_t)b * n_new + t) * n_kv + h) * D;
        const int64_t row = prow * n_kv + h;
        if (k_f16) {
          st |= store_k_f16(k + src, D, k_f16 + row * D);
        } else {
          st |= oracle_encode(k + src, s, D, 1, k_codes + row * cb, k_scales + row * sb);
        }
        st |= oracle_encode(v + src, s, D, 1, v_codes + row * cb, v_scales + row * sb);
      }
    }
  }
  return st;
}

// Decode over a paged cache: each sequence's rows are gathered through the
// table into the contiguous layout, then the contiguous decode runs unchanged.
int32_t oracle_decode_attention_paged(int batch, int max_seq, int n_kv, int n_q, int D, const float* s,
                                      const float* q, const int32_t* seq_lens, const int32_t* table, int P,
                                      int max_pages, int n_pages, const uint8_t* k_codes, const uint16_t* k_scales,
                                      const uint16_t* k_f16, const uint8_t* v_codes, const uint16_t* v_scales,
                                      float sm_scale, const uint8_t* which, float* out) {
  const int64_t cb = D / 2, sb = D / 32, rows = (int64_t)batch * max_seq * n_kv;
  std::vector<uint8_t> kc(k_f16 ? 0 : rows * cb), vc(rows * cb);
  std::vector<uint16_t> ks(k_f16 ? 0 : rows * sb), kf(k_f16 ? rows * D : 0), vs(rows * sb);
  int32_t st = 0;
  for (int b = 0; b < batch; ++b) {
    const int len = seq_lens[b];
    for (int64_t t = 0; t < len && t < max_seq; ++t) {
      const int pg = table[(int64_t)b * max_pages + t / P];
      if (pg < 0 || pg >= n_pages) {
        st |= ORC_STATUS_CAPACITY;
        continue;  // its rows stay zero
      }
      for (int h = 0; h < n_kv; ++h) {
        const int64_t src = ((int64_t)pg * P + t % P) * n_kv + h;
        const int64_t dst = ((int64_t)b * max_seq + t) * n_kv + h;
        std::memcpy(&vc[dst * cb], v_codes + src * cb, cb);
        std::memcpy(&vs[dst * sb], v_scales + src * sb, sb * 2);
        if (k_f16) {
          std::memcpy(&kf[dst * D], k_f16 + src * D, D * 2);
        } else {
          std::memcpy(&kc[dst * cb], k_codes + src * cb, cb);
          std::memcpy(&ks[dst * sb], k_scales + src * sb, sb * 2);
        }
      }
    }
  }
  st |= decode_body(batch, max_seq, n_kv, n_q, D, s, q, seq_lens, k_f16 ? nullptr : kc.data(),
                    k_f16 ? nullptr : ks.data(), k_f16 ? kf.data() : nullptr, vc.data(), vs.data(), nullptr, 0, 0,
                    sm_scale, which, out);
  return st;
}

// Delegated hot/cold cache [MLX-deleg]: K as binary16 for every token (as in
// the asymmetric cache), V as binary16 in the hot tail v_tail [batch][W][n_kv][D]
// and as int4 codes in the cold body (the usual V caches, at the token's own
// position). Tokens are taken one at a time, in order: when the sequence grows
// from P to P + 1 tokens, every token that cold_length moves out of the tail is
// folded first (its binary16 tail value encoded exactly as a fresh V vector),
// then token P enters the tail. A V element whose binary16 is not finite raises
// ORC_STATUS_NONFINITE. Tail slots of tokens already folded keep stale values.
int32_t oracle_append_delegated(int batch, int max_seq, int n_kv, int D, const float* s, const float* k,
                                const float* v, int n_new, const int32_t* start_pos, int W, int F,
                                uint16_t* k_f16, uint8_t* v_codes, uint16_t* v_scales, uint16_t* v_tail) {
  int32_t st = 0;
  const int64_t cb = D / 2, sb = D / 32;
  std::vector<float> x(D);
  for (int b = 0; b < batch; ++b) {
    const int64_t p0 = start_pos[b];
    if (p0 < 0 || p0 + n_new > max_seq) {
      st |= ORC_STATUS_CAPACITY;
      continue;
    }
    for (int t = 0; t < n_new; ++t) {
      const int64_t P = p0 + t;
      for (int64_t T = cold_length(P, W, F); T < cold_length(P + 1, W, F); ++T) {
        for (int h = 0; h < n_kv; ++h) {
          const uint16_t* hot = v_tail + (((int64_t)b * W + T % W) * n_kv + h) * D;
          for (int i = 0; i < D; ++i) x[i] = f16_to_f32(hot[i]);
          const int64_t row = ((int64_t)b * max_seq + T) * n_kv + h;
          st |= oracle_encode(x.data(), s, D, 1, v_codes + row * cb, v_scales + row * sb);
        }
      }
      for (int h = 0; h < n_kv; ++h) {
        const int64_t src = (((int64_t)b * n_new + t) * n_kv + h) * D;
        const int64_t row = ((int64_t)b * max_seq + P) * n_kv + h;
        uint16_t* hot = v_tail + (((int64_t)b * W + P % W) * n_kv + h) * D;
        for (int i = 0; i < D; ++i) {
          const uint16_t kb = f32_to_f16_rne(k[src + i]);
          const uint16_t vb = f32_to_f16_rne(v[src + i]);
          if ((kb & 0x7C00u) == 0x7C00u || (vb & 0x7C00u) == 0x7C00u) st |= ORC_STATUS_NONFINITE;
          k_f16[row * D + i] = kb;
          hot[i] = vb;
        }
      }
    }
  }
  return st;
}

// Decode attention over the delegated cache: the asymmetric decode's steps
// (binary16 K against q), with V_t = code * sigma for t < cold_length(len_b)
// and SRHT(binary16 tail value) otherwise, then SRHT^-1 of the weighted sum.
int32_t oracle_decode_attention_delegated(int batch, int max_seq, int n_kv, int n_q, int D, const float* s,
                                          const float* q, const int32_t* seq_lens, const uint16_t* k_f16,
                                          const uint8_t* v_codes, const uint16_t* v_scales,
                                          const uint16_t* v_tail, int W, int F, float sm_scale,
                                          const uint8_t* which, float* out) {
  return decode_body(batch, max_seq, n_kv, n_q, D, s, q, seq_lens, nullptr, nullptr, k_f16, v_codes, v_scales,
                     v_tail, W, F, sm_scale, which, out);
}

int64_t oracle_cold_length(int64_t len, int W, int F) { return cold_length(len, W, F); }

// Dequantise a whole cache: out [batch][max_seq][n_kv][D] binary32, rows t >= len_b
// set to 0. original_domain = 0 gives yhat = code * sigma (rotated domain);
// 1 applies the inverse SRHT.
int32_t oracle_dequantize(int batch, int max_seq, int n_kv, int D, const float* s,
                          const uint8_t* codes, const uint16_t* scales, const int32_t* seq_lens,
                          int original_domain, float* out) {
  int32_t st = 0;
  const int64_t cb = D / 2, sb = D / 32;
  std::vector<float> y(D);
  for (int b = 0; b < batch; ++b) {
    int len = seq_lens[b];
    if (len > max_seq) {
      st |= ORC_STATUS_CAPACITY;
      len = 0;
    }
    for (int t = 0; t < max_seq; ++t) {
      for (int h = 0; h < n_kv; ++h) {
        const int64_t row = ((int64_t)b * max_seq + t) * n_kv + h;
        float* o = out + row * D;
        if (t >= len) {
          for (int i = 0; i < D; ++i) o[i] = 0.0f;
          continue;
        }
        dequantize_rotated(codes + row * cb, scales + row * sb, D, y.data());
        if (original_domain)
          srht_inverse_vec(y.data(), s, D, o);
        else
          std::memcpy(o, y.data(), sizeof(float) * D);
      }
    }
  }
  return st;
}

}  // extern "C"
