// Kernel parameter blocks and launchers (internal to libtq_b200).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tqk {

// Division of a 32-bit unsigned n by an invariant divisor d >= 1 with a multiply and
// shifts (the round-up method of Granlund and Montgomery, "Division by invariant
// integers using multiplication"): m = floor(2^32 (2^l - d) / d) + 1 with
// l = ceil(log2 d); q = (t + ((n - t) >> 1)) >> (l - 1), t = umulhi(m, n); d = 1 is
// the identity (l = 0). Exact for every n < 2^32.
struct FastDiv {
  uint32_t d, m, l;
};

__host__ __forceinline__ FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.l = 0;
  while ((1ull << f.l) < d) ++f.l;
  f.m = d <= 1 ? 0u : (uint32_t)((((1ull << 32) * ((1ull << f.l) - d)) / d) + 1);
  return f;
}

#ifdef __CUDACC__
__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv& f) {
  if (f.l == 0) return n;
  const uint32_t t = __umulhi(f.m, n);
  return (t + ((n - t) >> 1)) >> (f.l - 1);
}
#endif

struct QuantizeParams {
  const void* k;
  const void* v;
  int in_dtype;
  int batch, n_new, n_kv, max_seq;
  const int32_t* start_pos;
  uint8_t* k_codes;
  uint16_t* k_scales;
  uint8_t* v_codes;
  uint16_t* v_scales;
  int32_t* status;
  uint64_t sign_bits[4];
  float c_d;
  int k_f16;  // 1: K is stored as binary16 of the input (k_codes is that buffer), k_scales unused
  // delegated cache (tail_window > 0, with k_f16): binary16 V hot tail [batch][W][n_kv][D]
  uint16_t* v_tail;
  int tail_window, fold_chunk;
  const float* lambda_k;  // per-channel lambda in the rotated domain (nullable)
  const float* lambda_v;
  // paged storage (page_tokens > 0): pool row of token t of sequence b =
  // block_table[b * max_pages + t / page_tokens] * page_tokens + t % page_tokens
  const int32_t* block_table;
  int page_tokens, max_pages, n_pages;
  // 32-bit thread indexing (the launch has fewer than 2^32 threads): divisors n_kv,
  // n_new and n_new + tail_window
  FastDiv div_kv, div_new, div_vrows;
};

struct DequantParams {
  const uint8_t* codes;
  const uint16_t* scales;
  const int32_t* seq_lens;
  float* out;
  int batch, max_seq, n_kv, original_domain;
  int32_t* status;
  uint64_t sign_bits[4];
  float c_d;
};

// 128-byte opaque copy of a CUtensorMap (passed by value as a __grid_constant__).
struct alignas(64) TensorMap128 {
  uint64_t words[16];
};

struct DecodeParams {
  const void* q;
  int q_dtype;
  const int32_t* seq_lens;
  const uint16_t* k_scales;
  const uint16_t* v_scales;
  float* ws_ml;    // [slots][n_q][2]: running max (log2 units), running sum
  float* ws_acc;   // [slots][n_q][D]: rotated-domain accumulator, relative to the running max
  float* out;      // [batch][n_q][D]
  int32_t* status;
  int batch, max_seq, n_kv, n_q, group;
  int grid;            // CTAs in the split-K launch
  int min_split;       // smallest token range per CTA
  float sm_scale_log2; // sm_scale * log2(e)
  float c_d;
  uint64_t sign_bits[4];
  int k_f16;  // 1: K tiles are binary16 (original domain), no K scales
  // delegated cache (tail_window > 0, with k_f16): the split-K kernel covers the cold
  // tokens; the merge kernel attends to the hot ones (binary16 K rows and V tail)
  const uint16_t* k16;
  const uint16_t* v_tail;
  int tail_window, fold_chunk;
  int tail_chunks;  // hot-tail partials per sequence (ceil(tail_window / 64)); 0 without a tail
  int tail_slot0;   // workspace slot of sequence 0's first hot-tail partial (after the split-K slots)
  const float* lambda_k;  // per-channel lambda of the cache (nullable): q is divided by lambda_k,
  const float* lambda_v;  // the merged V sum by lambda_v, both in the rotated domain
  float sparse_lt;        // log2 of the sparse-V threshold; -inf = off
  // paged storage (page_tokens > 0): as in QuantizeParams. len_align: each
  // sequence's length is padded to a multiple of it in the split-K token space
  // (the kernel's tile, so that no tile crosses a page), 1 without paging.
  const int32_t* block_table;
  int page_tokens, max_pages, n_pages;
  int len_align;
  uint64_t wait_ns;  // bound on each pipeline wait of the split-K kernel (its copy drain always uses 1 s)
};

// Hot-tail partials per sequence of the delegated cache (64 tokens each).
__host__ __device__ __forceinline__ int tail_chunk_count(int W) { return W > 0 ? (W + 63) / 64 : 0; }

// Cold (int4) tokens of a delegated-cache sequence of len tokens (all of them without a tail).
__host__ __device__ __forceinline__ int64_t cold_tokens(int64_t len, int W, int F) {
  if (W <= 0) return len;
  if (len <= W) return 0;
  return (len - W + F - 1) / F * F;
}

// Decode workspace for a split-K grid of `grid` CTAs: an int64 header (prefix sums of
// the lengths and the per-CTA token range), then (running max, running sum) and a
// D-float accumulator per (slot, q head). Slots: one per CTA plus one per sequence
// (a CTA range and a sequence range intersect at most once for each pair, and the
// slot index sequence + CTA cannot repeat between intersecting pairs), plus the
// delegated cache's hot-tail partials.
__host__ __forceinline__ uint64_t decode_workspace_bytes(int batch, int n_q, int D, int grid, int tail_window) {
  const uint64_t slots =
      (uint64_t)grid + (uint64_t)batch + (uint64_t)batch * (uint64_t)tail_chunk_count(tail_window);
  const uint64_t header = 8ull * (uint64_t)(batch + 2);
  const uint64_t ml = slots * (uint64_t)n_q * 2ull * 4ull;
  const uint64_t acc = slots * (uint64_t)n_q * (uint64_t)D * 4ull;
  return ((header + ml + 255) / 256) * 256 + acc;
}

// Threads per block of the row-wise append kernel, the threads that share one head
// vector, and the rows (vectors) of its input tensor-copy box. One thread per vector:
// splitting a head_dim-128 vector over two threads (one shuffle stage, 128 instead
// of 168 registers, 4 instead of 3 blocks per SM) measured slower (190 against
// 175 us on a 2.1 M-vector prefill).
constexpr int kRowsThreads = 128;
__host__ __device__ constexpr int rows_threads_per_vector(int /*head_dim*/) { return 1; }
__host__ __device__ constexpr int rows_kernel_box_rows(int head_dim) {
  return kRowsThreads / rows_threads_per_vector(head_dim);
}

cudaError_t launch_quantize(const QuantizeParams& p, int head_dim, cudaStream_t s);
// The row-wise append (head_dim 64 or 128, no hot tail): kin / vin view the K / V
// inputs as [batch * n_new * n_kv][head_dim] with boxes of 128 bytes by
// rows_kernel_box_rows(head_dim) rows and the 128-byte swizzle; persistent blocks on
// `sms` SMs.
cudaError_t launch_quantize_rows(const QuantizeParams& p, int head_dim, const TensorMap128& kin,
                                 const TensorMap128& vin, int sms, cudaStream_t s);
cudaError_t launch_dequantize(const DequantParams& p, int head_dim, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams& p, const TensorMap128& kmap, const TensorMap128& vmap, int head_dim,
                          cudaStream_t s, cudaEvent_t after_split);
int decode_smem_bytes(int head_dim, int n_kv, int k_f16);
int decode_tile_tokens(int head_dim, int n_kv, int k_f16);

}  // namespace tqk
