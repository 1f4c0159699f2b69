// C ABI of libtq_b200: argument validation, layout arithmetic, tensor-map
// encoding and kernel launches. See include/tq.h for the contract.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/tq.h"
#include "tq_kernels.h"

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return TQ_ERR_CUDA;
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SplitMix64 (S. Vigna's public-domain generator), used to draw the fixed +-1
// diagonal of the rotation: s_i = -1 iff the top bit of the i-th output is set.
uint64_t splitmix64_step(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ULL;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// Split-K grid ceiling the default workspace is sized for.
constexpr int kMaxCtas = 1024;
constexpr int kMaxBatchDecode = 1024;
constexpr int kMaxTileTokens = 256;

int device_sm_count(int* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  static std::mutex mu;
  static int cache[64] = {0};
  std::lock_guard<std::mutex> lk(mu);
  if (dev < 64 && cache[dev] > 0) {
    *out = cache[dev];
    return TQ_OK;
  }
  int n = 0;
  e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 64) cache[dev] = n;
  *out = n;
  return TQ_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Token rows of a cache buffer: batch * max_seq, or n_pages * page_tokens when paged.
uint64_t pool_rows(const tq_layout_t* L) {
  return L->page_tokens > 0 ? (uint64_t)L->n_pages * (uint64_t)L->page_tokens
                            : (uint64_t)L->batch * (uint64_t)L->max_seq;
}

// 3-D view of a codes buffer: (D/2 bytes, token rows, n_kv heads),
// box (D/2, tile, n_kv); the shared-memory image is [head][tile][D/2] with the
// swizzle matching the row pitch.
int encode_codes_map(const tq_layout_t* L, const uint8_t* base, int tile, tqk::TensorMap128* out) {
  auto enc = get_encode_fn();
  if (enc == nullptr) return cuda_fail(cudaErrorNotSupported);
  const int rb = L->head_dim / 2;
  cuuint64_t dims[3] = {(cuuint64_t)rb, (cuuint64_t)pool_rows(L), (cuuint64_t)L->n_kv_heads};
  cuuint64_t strides[2] = {(cuuint64_t)L->code_stride_tok, (cuuint64_t)rb};
  cuuint32_t box[3] = {(cuuint32_t)rb, (cuuint32_t)tile, (cuuint32_t)L->n_kv_heads};
  cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMapSwizzle sw = rb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : rb == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                     : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUtensorMap m;
  CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = (int)r;
    return TQ_ERR_CUDA;
  }
  static_assert(sizeof(CUtensorMap) == sizeof(tqk::TensorMap128), "tensor map size");
  std::memcpy(out, &m, sizeof(m));
  return TQ_OK;
}

// Appends of more than this many vectors (K and V) take the one-thread-per-vector
// kernel; smaller ones (a decode step's new tokens, short prefills) the
// thread-per-group kernel, whose four-fold parallelism per vector gives a shorter
// launch (measured back to back: 2.8 against 4.1 us on a 512-vector append, 9.6
// against 10.1 us on 65 536 vectors; 224 against 168 us on 2.1 M vectors).
constexpr uint64_t kRowsKernelMinVectors = 65537;

// 2-D view of an append input (K or V) for the row-wise kernel: `rows` vectors of
// D elements of esz bytes, box (128 bytes of a row, rows_kernel_box_rows(D) rows)
// with the 128-byte swizzle.
int encode_rows_map(const void* base, int D, int esz, uint64_t rows, tqk::TensorMap128* out) {
  auto enc = get_encode_fn();
  if (enc == nullptr) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * (cuuint64_t)esz};
  cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)tqk::rows_kernel_box_rows(D)};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMap m;
  CUresult r = enc(&m, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = (int)r;
    return TQ_ERR_CUDA;
  }
  std::memcpy(out, &m, sizeof(m));
  return TQ_OK;
}

// 4-D view of a binary16 K buffer: (64 halves, batch*max_seq tokens, D/64 lines,
// n_kv heads) with strides (token stride, 128 B, 2D B), box (64, tile, D/64, n_kv):
// the shared-memory image is [head][line][tile][64] binary16 with the 128-byte
// swizzle, so 8 consecutive tokens of one line fall on 8 swizzle phases
// (D = 32: one 64-byte line per token, 64-byte swizzle).
int encode_k16_map(const tq_layout_t* L, const uint8_t* base, int tile, tqk::TensorMap128* out) {
  auto enc = get_encode_fn();
  if (enc == nullptr) return cuda_fail(cudaErrorNotSupported);
  const int D = L->head_dim;
  const int inner = D < 64 ? D : 64;
  const int lines = D / inner;
  cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)pool_rows(L), (cuuint64_t)lines, (cuuint64_t)L->n_kv_heads};
  cuuint64_t strides[3] = {(cuuint64_t)L->k_stride_tok, (cuuint64_t)inner * 2, (cuuint64_t)D * 2};
  cuuint32_t box[4] = {(cuuint32_t)inner, (cuuint32_t)tile, (cuuint32_t)lines, (cuuint32_t)L->n_kv_heads};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUtensorMapSwizzle sw = inner == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap m;
  CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<uint8_t*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = (int)r;
    return TQ_ERR_CUDA;
  }
  std::memcpy(out, &m, sizeof(m));
  return TQ_OK;
}

int build_layout(int batch, int max_seq, int n_kv_heads, int n_q_heads, int head_dim, int group_size,
                 uint64_t sign_seed, int k_format, int tail_window, int fold_chunk, int page_tokens, int n_pages,
                 tq_layout_t* out);

int check_layout(const tq_layout_t* L) {
  if (L == nullptr) return TQ_ERR_INVALID_ARG;
  tq_layout_t chk;
  const int r = build_layout(L->batch, L->max_seq, L->n_kv_heads, L->n_q_heads, L->head_dim, L->group_size,
                             L->sign_seed, L->k_format, L->tail_window, L->fold_chunk, L->page_tokens, L->n_pages,
                             &chk);
  if (r != TQ_OK) return r;
  if (std::memcmp(&chk, L, sizeof(chk)) != 0) return TQ_ERR_INVALID_ARG;  // edited or stale layout
  return TQ_OK;
}

void copy_signs(const tq_layout_t* L, uint64_t (&dst)[4]) {
  for (int i = 0; i < 4; ++i) dst[i] = L->sign_bits[i];
}

uint64_t workspace_bytes(int batch, int n_q, int D, int max_ctas, int tail_window = 0) {
  return tqk::decode_workspace_bytes(batch, n_q, D, max_ctas, tail_window);
}

constexpr int kMaxTailWindow = 1024;  // the merge kernel keeps one score per hot token in shared memory

int build_layout(int batch, int max_seq, int n_kv_heads, int n_q_heads, int head_dim, int group_size,
                 uint64_t sign_seed, int k_format, int tail_window, int fold_chunk, int page_tokens, int n_pages,
                 tq_layout_t* out) {
  if (out == nullptr) return TQ_ERR_INVALID_ARG;
  if (page_tokens != 0 || n_pages != 0) {
    if (k_format != TQ_K_INT4 && k_format != TQ_K_FP16) return TQ_ERR_INVALID_ARG;
    if (!is_pow2(page_tokens) || page_tokens > 4096 || n_pages <= 0) return TQ_ERR_INVALID_ARG;
    if ((int64_t)n_pages * page_tokens > (int64_t)INT32_MAX) return TQ_ERR_UNSUPPORTED;
  }
  if (k_format != TQ_K_INT4 && k_format != TQ_K_FP16 && k_format != TQ_KV_DELEGATED) return TQ_ERR_INVALID_ARG;
  if (k_format == TQ_KV_DELEGATED) {
    if (tail_window < 1 || tail_window > kMaxTailWindow || fold_chunk < 1 || fold_chunk > tail_window)
      return TQ_ERR_INVALID_ARG;
  } else if (tail_window != 0 || fold_chunk != 0) {
    return TQ_ERR_INVALID_ARG;
  }
  if (batch <= 0 || max_seq <= 0 || n_kv_heads <= 0 || n_q_heads <= 0) return TQ_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads != 0) return TQ_ERR_INVALID_ARG;
  // mlxcel §"Known limitations / head dimension": power-of-two head dims only.
  if (!is_pow2(head_dim) || head_dim < 32 || head_dim > 256) return TQ_ERR_UNSUPPORTED;
  if (group_size != 32) return TQ_ERR_UNSUPPORTED;
  if ((int64_t)batch * (int64_t)max_seq > (int64_t)INT32_MAX) return TQ_ERR_UNSUPPORTED;  // tensor-copy coordinates
  if (page_tokens > 0) {  // no decode tile may cross a page
    const int tile = tqk::decode_tile_tokens(head_dim, n_kv_heads, k_format == TQ_K_FP16 ? 1 : 0);
    if (tile <= 0 || page_tokens % tile != 0) return TQ_ERR_UNSUPPORTED;
  }
  const int64_t rows = page_tokens > 0 ? (int64_t)n_pages * page_tokens : (int64_t)batch * max_seq;
  tq_layout_t L;
  std::memset(&L, 0, sizeof(L));
  L.batch = batch;
  L.max_seq = max_seq;
  L.n_kv_heads = n_kv_heads;
  L.n_q_heads = n_q_heads;
  L.head_dim = head_dim;
  L.group_size = group_size;
  L.n_groups = head_dim / 32;
  L.c_d = (float)(1.0 / std::sqrt((double)head_dim));
  L.sign_seed = sign_seed;
  uint64_t st = sign_seed;
  for (int i = 0; i < head_dim; ++i)
    if (splitmix64_step(st) >> 63) L.sign_bits[i >> 6] |= 1ull << (i & 63);
  L.code_stride_tok = (int64_t)n_kv_heads * head_dim / 2;
  L.code_stride_seq = (int64_t)max_seq * L.code_stride_tok;
  L.scale_stride_tok = (int64_t)n_kv_heads * L.n_groups;
  L.scale_stride_seq = (int64_t)max_seq * L.scale_stride_tok;
  L.codes_bytes = (uint64_t)rows * (uint64_t)L.code_stride_tok;
  const uint64_t srow = (uint64_t)L.scale_stride_tok * 2ull;
  L.scales_bytes = (uint64_t)rows * srow + kMaxTileTokens * srow + 32ull;
  L.max_ctas = kMaxCtas;
  L.decode_workspace_bytes =
      workspace_bytes(batch, n_q_heads, head_dim, kMaxCtas, k_format == TQ_KV_DELEGATED ? tail_window : 0);
  L.k_format = k_format;
  if (k_format != TQ_K_INT4) {
    L.k_stride_tok = (int64_t)n_kv_heads * head_dim * 2;
    L.k_stride_seq = (int64_t)max_seq * L.k_stride_tok;
    L.k_bytes = (uint64_t)rows * (uint64_t)L.k_stride_tok;
  } else {
    L.k_stride_tok = L.code_stride_tok;
    L.k_stride_seq = L.code_stride_seq;
    L.k_bytes = L.codes_bytes;
  }
  if (page_tokens > 0) {
    L.page_tokens = page_tokens;
    L.n_pages = n_pages;
    L.max_pages = (max_seq + page_tokens - 1) / page_tokens;
    L.code_stride_seq = 0;  // no per-sequence slabs
    L.scale_stride_seq = 0;
    L.k_stride_seq = 0;
  }
  if (k_format == TQ_KV_DELEGATED) {
    L.tail_window = tail_window;
    L.fold_chunk = fold_chunk;
    L.tail_stride_tok = (int64_t)n_kv_heads * head_dim * 2;
    L.tail_stride_seq = (int64_t)tail_window * L.tail_stride_tok;
    L.tail_bytes = (uint64_t)batch * (uint64_t)L.tail_stride_seq;
  }
  *out = L;
  return TQ_OK;
}

}  // namespace

extern "C" {

int tq_cache_layout(int batch, int max_seq, int n_kv_heads, int n_q_heads, int head_dim, int group_size,
                    uint64_t sign_seed, tq_layout_t* out) {
  return build_layout(batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size, sign_seed, TQ_K_INT4, 0, 0, 0, 0,
                      out);
}

int tq_cache_layout_kv(int batch, int max_seq, int n_kv_heads, int n_q_heads, int head_dim, int group_size,
                       uint64_t sign_seed, int k_format, tq_layout_t* out) {
  if (k_format == TQ_KV_DELEGATED) return TQ_ERR_INVALID_ARG;  // needs the window sizes
  return build_layout(batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size, sign_seed, k_format, 0, 0, 0, 0,
                      out);
}

int tq_cache_layout_delegated(int batch, int max_seq, int n_kv_heads, int n_q_heads, int head_dim, int group_size,
                              uint64_t sign_seed, int tail_window, int fold_chunk, tq_layout_t* out) {
  return build_layout(batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size, sign_seed, TQ_KV_DELEGATED,
                      tail_window, fold_chunk, 0, 0, out);
}

int tq_cache_layout_paged(int batch, int max_seq, int n_kv_heads, int n_q_heads, int head_dim, int group_size,
                          uint64_t sign_seed, int k_format, int page_tokens, int n_pages, tq_layout_t* out) {
  if (page_tokens <= 0 || n_pages <= 0) return TQ_ERR_INVALID_ARG;
  return build_layout(batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size, sign_seed, k_format, 0, 0,
                      page_tokens, n_pages, out);
}

int64_t tq_cold_length(const tq_layout_t* layout, int64_t len) {
  if (layout == nullptr || len < 0) return -1;
  return tqk::cold_tokens(len, layout->tail_window, layout->fold_chunk);
}

namespace {

int append_impl(const tq_layout_t* layout, const void* k, const void* v, int in_dtype, int n_new,
                const int32_t* d_start_pos, uint8_t* k_codes, uint16_t* k_scales, uint8_t* v_codes,
                uint16_t* v_scales, uint16_t* v_tail, const tq_append_opts_t* opts, int32_t* d_status,
                void* stream, const int32_t* d_block_table = nullptr) {
  if ((layout->page_tokens > 0) != (d_block_table != nullptr)) return TQ_ERR_INVALID_ARG;
  const float* lam_k = opts ? opts->lambda_k : nullptr;
  const float* lam_v = opts ? opts->lambda_v : nullptr;
  // lambda scales quantised vectors: not binary16 K, not the delegated cache's tail
  if (lam_k && layout->k_format != TQ_K_INT4) return TQ_ERR_INVALID_ARG;
  if ((lam_k || lam_v) && layout->k_format == TQ_KV_DELEGATED) return TQ_ERR_INVALID_ARG;
  if ((lam_k && !aligned16(lam_k)) || (lam_v && !aligned16(lam_v))) return TQ_ERR_INVALID_ARG;
  if (n_new < 0) return TQ_ERR_INVALID_ARG;
  if (n_new > layout->max_seq) return TQ_ERR_CAPACITY;
  if (in_dtype != TQ_F32 && in_dtype != TQ_BF16 && in_dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
  if (n_new == 0) return TQ_OK;
  const bool kf16 = layout->k_format != TQ_K_INT4;
  const bool deleg = layout->k_format == TQ_KV_DELEGATED;
  if (!k || !v || !d_start_pos || !k_codes || (!kf16 && !k_scales) || !v_codes || !v_scales || (deleg && !v_tail))
    return TQ_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_codes) || !aligned16(v_codes) || (deleg && !aligned16(v_tail)))
    return TQ_ERR_INVALID_ARG;
  const int64_t v_rows = (int64_t)n_new + (deleg ? layout->tail_window : 0);
  // the kernel indexes its threads in 32 bits: K and V items (padded to whole warps)
  // must number fewer than 2^32
  if ((int64_t)layout->batch * v_rows * layout->n_kv_heads * layout->n_groups * 2 + 64 >= (int64_t)1 << 32)
    return TQ_ERR_UNSUPPORTED;
  tqk::QuantizeParams p;
  p.k = k;
  p.v = v;
  p.in_dtype = in_dtype;
  p.batch = layout->batch;
  p.n_new = n_new;
  p.n_kv = layout->n_kv_heads;
  p.max_seq = layout->max_seq;
  p.start_pos = d_start_pos;
  p.k_codes = k_codes;
  p.k_scales = k_scales;
  p.v_codes = v_codes;
  p.v_scales = v_scales;
  p.status = d_status;
  copy_signs(layout, p.sign_bits);
  p.c_d = layout->c_d;
  p.k_f16 = kf16 ? 1 : 0;
  p.v_tail = v_tail;
  p.tail_window = layout->tail_window;
  p.fold_chunk = layout->fold_chunk;
  p.lambda_k = lam_k;
  p.lambda_v = lam_v;
  p.block_table = d_block_table;
  p.page_tokens = layout->page_tokens;
  p.max_pages = layout->max_pages;
  p.n_pages = layout->n_pages;
  p.div_kv = tqk::make_fastdiv((uint32_t)layout->n_kv_heads);
  p.div_new = tqk::make_fastdiv((uint32_t)n_new);
  p.div_vrows = tqk::make_fastdiv((uint32_t)v_rows);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int D = layout->head_dim;
  cudaError_t e;
  const uint64_t vectors = 2ull * (uint64_t)layout->batch * (uint64_t)n_new * (uint64_t)layout->n_kv_heads;
  if (!deleg && (D == 64 || D == 128) && vectors >= kRowsKernelMinVectors) {
    // one thread per vector, input rows by tensor copies
    const int esz = in_dtype == TQ_F32 ? 4 : 2;
    const uint64_t rows = (uint64_t)layout->batch * (uint64_t)n_new * (uint64_t)layout->n_kv_heads;
    tqk::TensorMap128 kin, vin;
    int rc = encode_rows_map(k, D, esz, rows, &kin);
    if (rc != TQ_OK) return rc;
    rc = encode_rows_map(v, D, esz, rows, &vin);
    if (rc != TQ_OK) return rc;
    int sms = 0;
    rc = device_sm_count(&sms);
    if (rc != TQ_OK) return rc;
    e = tqk::launch_quantize_rows(p, D, kin, vin, sms, s);
  } else {
    e = tqk::launch_quantize(p, D, s);
  }
  return e == cudaSuccess ? TQ_OK : cuda_fail(e);
}

}  // namespace

int tq_quantize_append(const tq_layout_t* layout, const void* k, const void* v, int in_dtype, int n_new,
                       const int32_t* d_start_pos, uint8_t* k_codes, uint16_t* k_scales, uint8_t* v_codes,
                       uint16_t* v_scales, int32_t* d_status, void* stream) {
  int r = check_layout(layout);
  if (r != TQ_OK) return r;
  if (layout->k_format == TQ_KV_DELEGATED || layout->page_tokens > 0) return TQ_ERR_INVALID_ARG;
  return append_impl(layout, k, v, in_dtype, n_new, d_start_pos, k_codes, k_scales, v_codes, v_scales, nullptr,
                     nullptr, d_status, stream);
}

int tq_quantize_append_ex(const tq_layout_t* layout, const void* k, const void* v, int in_dtype, int n_new,
                          const int32_t* d_start_pos, uint8_t* k_codes, uint16_t* k_scales, uint8_t* v_codes,
                          uint16_t* v_scales, const tq_append_opts_t* opts, int32_t* d_status, void* stream) {
  int r = check_layout(layout);
  if (r != TQ_OK) return r;
  if (layout->k_format == TQ_KV_DELEGATED || layout->page_tokens > 0) return TQ_ERR_INVALID_ARG;
  return append_impl(layout, k, v, in_dtype, n_new, d_start_pos, k_codes, k_scales, v_codes, v_scales, nullptr,
                     opts, d_status, stream);
}

int tq_quantize_append_paged(const tq_layout_t* layout, const void* k, const void* v, int in_dtype, int n_new,
                             const int32_t* d_start_pos, const int32_t* d_block_table, uint8_t* k_codes,
                             uint16_t* k_scales, uint8_t* v_codes, uint16_t* v_scales, const tq_append_opts_t* opts,
                             int32_t* d_status, void* stream) {
  int r = check_layout(layout);
  if (r != TQ_OK) return r;
  if (layout->page_tokens <= 0 || d_block_table == nullptr) return TQ_ERR_INVALID_ARG;
  return append_impl(layout, k, v, in_dtype, n_new, d_start_pos, k_codes, k_scales, v_codes, v_scales, nullptr,
                     opts, d_status, stream, d_block_table);
}

int tq_append_delegated(const tq_layout_t* layout, const void* k, const void* v, int in_dtype, int n_new,
                        const int32_t* d_start_pos, uint16_t* k_f16, uint8_t* v_codes, uint16_t* v_scales,
                        uint16_t* v_tail, int32_t* d_status, void* stream) {
  int r = check_layout(layout);
  if (r != TQ_OK) return r;
  if (layout->k_format != TQ_KV_DELEGATED) return TQ_ERR_INVALID_ARG;
  return append_impl(layout, k, v, in_dtype, n_new, d_start_pos, reinterpret_cast<uint8_t*>(k_f16), nullptr,
                     v_codes, v_scales, v_tail, nullptr, d_status, stream);
}

namespace {

int decode_impl(const tq_layout_t* layout, const void* q, int q_dtype, const int32_t* d_seq_lens,
                const uint8_t* k_codes, const uint16_t* k_scales, const uint8_t* v_codes, const uint16_t* v_scales,
                const uint16_t* v_tail, float sm_scale, float* out, void* workspace, size_t ws_bytes,
                int32_t* d_status, const tq_decode_opts_t* opts, void* stream,
                const int32_t* d_block_table = nullptr) {
  int r = TQ_OK;
  if ((layout->page_tokens > 0) != (d_block_table != nullptr)) return TQ_ERR_INVALID_ARG;
  const int D = layout->head_dim, Hkv = layout->n_kv_heads, Hq = layout->n_q_heads;
  const int G = Hq / Hkv;
  if (layout->batch > kMaxBatchDecode) return TQ_ERR_UNSUPPORTED;
  if (!(Hkv == 1 || Hkv == 2 || Hkv == 4 || Hkv == 8) || G > 8) return TQ_ERR_UNSUPPORTED;
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16 && q_dtype != TQ_F16) return TQ_ERR_INVALID_ARG;
  const bool kf16 = layout->k_format != TQ_K_INT4;
  const bool deleg = layout->k_format == TQ_KV_DELEGATED;
  // binary16 K tiles: the stage ring holds them only up to head_dim 128
  if (kf16 && D > 128) return TQ_ERR_UNSUPPORTED;
  if (!q || !d_seq_lens || !k_codes || (!kf16 && !k_scales) || !v_codes || !v_scales || !out || !workspace ||
      (deleg && !v_tail))
    return TQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_codes) || !aligned16(v_codes) || (!kf16 && !aligned16(k_scales)) ||
      !aligned16(v_scales) || !aligned16(out) || !aligned16(workspace) || (deleg && !aligned16(v_tail)))
    return TQ_ERR_INVALID_ARG;
  if (!std::isfinite(sm_scale)) return TQ_ERR_INVALID_ARG;
  // options: every check here is on the host, before any CUDA call
  int req_ctas = 0;
  int min_split = 64;  // measured: a 4096-token decode runs 2 us faster over 64-token ranges than 128
  cudaEvent_t ev = nullptr;
  const float* lam_k = nullptr;
  const float* lam_v = nullptr;
  float sparse_lt = -INFINITY;
  uint64_t wait_ns = 1000000000ull;  // 1 s
  if (opts != nullptr) {
    if (opts->wait_limit_ns < 0) return TQ_ERR_INVALID_ARG;
    if (opts->wait_limit_ns > 0) wait_ns = (uint64_t)opts->wait_limit_ns;
    if (opts->max_ctas < 0 || opts->max_ctas > layout->max_ctas || opts->min_split_tokens < 0)
      return TQ_ERR_INVALID_ARG;
    req_ctas = opts->max_ctas;
    if (opts->min_split_tokens > 0) min_split = opts->min_split_tokens;
    ev = reinterpret_cast<cudaEvent_t>(opts->after_split_event);
    lam_k = opts->lambda_k;
    lam_v = opts->lambda_v;
    if (lam_k && kf16) return TQ_ERR_INVALID_ARG;             // binary16 K carries no lambda
    if ((lam_k || lam_v) && deleg) return TQ_ERR_INVALID_ARG;  // nor does the binary16 tail
    if ((lam_k && !aligned16(lam_k)) || (lam_v && !aligned16(lam_v))) return TQ_ERR_INVALID_ARG;
    const float tau = opts->sparse_v_threshold;
    if (!(tau >= 0.f) || !std::isfinite(tau)) return TQ_ERR_INVALID_ARG;
    if (tau > 0.f) sparse_lt = std::log2(tau);
  }
  int sms = 0;
  r = device_sm_count(&sms);
  if (r != TQ_OK) return r;
  int grid = req_ctas > 0 ? req_ctas : sms;
  if (sparse_lt > -INFINITY && D != 64 && D != 128) return TQ_ERR_UNSUPPORTED;  // sparse-V kernels: D 64, 128
  if (grid > layout->max_ctas) grid = layout->max_ctas;
  const int W = deleg ? layout->tail_window : 0;
  if (ws_bytes < workspace_bytes(layout->batch, Hq, D, grid, W)) return TQ_ERR_INVALID_ARG;
  if (tqk::decode_smem_bytes(D, Hkv, kf16 ? 1 : 0) <= 0) return TQ_ERR_UNSUPPORTED;

  tqk::TensorMap128 km, vm;
  const int tile = tqk::decode_tile_tokens(D, Hkv, kf16 ? 1 : 0);
  r = kf16 ? encode_k16_map(layout, k_codes, tile, &km) : encode_codes_map(layout, k_codes, tile, &km);
  if (r != TQ_OK) return r;
  r = encode_codes_map(layout, v_codes, tile, &vm);
  if (r != TQ_OK) return r;

  tqk::DecodeParams p;
  p.q = q;
  p.q_dtype = q_dtype;
  p.seq_lens = d_seq_lens;
  p.k_scales = k_scales;
  p.v_scales = v_scales;
  const uint64_t slots =
      (uint64_t)grid + (uint64_t)layout->batch + (uint64_t)layout->batch * (uint64_t)tqk::tail_chunk_count(W);
  const uint64_t header_ml = ((8ull * (uint64_t)(layout->batch + 2) + slots * Hq * 8ull + 255) / 256) * 256;
  p.ws_ml = reinterpret_cast<float*>(workspace);
  p.ws_acc = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + header_ml);
  p.out = out;
  p.status = d_status;
  p.batch = layout->batch;
  p.max_seq = layout->max_seq;
  p.n_kv = Hkv;
  p.n_q = Hq;
  p.group = G;
  p.grid = grid;
  p.min_split = min_split;
  p.sm_scale_log2 = sm_scale * 1.4426950408889634f;
  p.c_d = layout->c_d;
  copy_signs(layout, p.sign_bits);
  p.k_f16 = kf16 ? 1 : 0;
  p.k16 = kf16 ? reinterpret_cast<const uint16_t*>(k_codes) : nullptr;
  p.v_tail = v_tail;
  p.tail_window = layout->tail_window;
  p.fold_chunk = layout->fold_chunk;
  p.tail_chunks = tqk::tail_chunk_count(W);
  p.tail_slot0 = grid + layout->batch;
  p.lambda_k = lam_k;
  p.lambda_v = lam_v;
  p.sparse_lt = sparse_lt;
  p.block_table = d_block_table;
  p.page_tokens = layout->page_tokens;
  p.max_pages = layout->max_pages;
  p.n_pages = layout->n_pages;
  p.len_align = layout->page_tokens > 0 ? tile : 1;
  p.wait_ns = wait_ns;
  cudaError_t e = tqk::launch_decode(p, km, vm, D, reinterpret_cast<cudaStream_t>(stream), ev);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e);
}

}  // namespace

int tq_decode_attention_ex(const tq_layout_t* layout, const void* q, int q_dtype, const int32_t* d_seq_lens,
                           const uint8_t* k_codes, const uint16_t* k_scales, const uint8_t* v_codes,
                           const uint16_t* v_scales, float sm_scale, float* out, void* workspace, size_t ws_bytes,
                           int32_t* d_status, const tq_decode_opts_t* opts, void* stream) {
  int r = check_layout(layout);
  if (r != TQ_OK) return r;
  if (layout->k_format == TQ_KV_DELEGATED || layout->page_tokens > 0) return TQ_ERR_INVALID_ARG;
  return decode_impl(layout, q, q_dtype, d_seq_lens, k_codes, k_scales, v_codes, v_scales, nullptr, sm_scale, out,
                     workspace, ws_bytes, d_status, opts, stream);
}

int tq_decode_attention_paged(const tq_layout_t* layout, const void* q, int q_dtype, const int32_t* d_seq_lens,
                              const int32_t* d_block_table, const uint8_t* k_codes, const uint16_t* k_scales,
                              const uint8_t* v_codes, const uint16_t* v_scales, float sm_scale, float* out,
                              void* workspace, size_t ws_bytes, int32_t* d_status, const tq_decode_opts_t* opts,
                              void* stream) {
  int r = check_layout(layout);
  if (r != TQ_OK) return r;
  if (layout->page_tokens <= 0 || d_block_table == nullptr) return TQ_ERR_INVALID_ARG;
  return decode_impl(layout, q, q_dtype, d_seq_lens, k_codes, k_scales, v_codes, v_scales, nullptr, sm_scale, out,
                     workspace, ws_bytes, d_status, opts, stream, d_block_table);
}

int tq_decode_attention_delegated(const tq_layout_t* layout, const void* q, int q_dtype, const int32_t* d_seq_lens,
                                  const uint16_t* k_f16, const uint8_t* v_codes, const uint16_t* v_scales,
                                  const uint16_t* v_tail, float sm_scale, float* out, void* workspace,
                                  size_t ws_bytes, int32_t* d_status, const tq_decode_opts_t* opts, void* stream) {
  int r = check_layout(layout);
  if (r != TQ_OK) return r;
  if (layout->k_format != TQ_KV_DELEGATED) return TQ_ERR_INVALID_ARG;
  return decode_impl(layout, q, q_dtype, d_seq_lens, reinterpret_cast<const uint8_t*>(k_f16), nullptr, v_codes,
                     v_scales, v_tail, sm_scale, out, workspace, ws_bytes, d_status, opts, stream);
}

int tq_decode_attention(const tq_layout_t* layout, const void* q, int q_dtype, const int32_t* d_seq_lens,
                        const uint8_t* k_codes, const uint16_t* k_scales, const uint8_t* v_codes,
                        const uint16_t* v_scales, float sm_scale, float* out, void* workspace, size_t ws_bytes,
                        int32_t* d_status, void* stream) {
  return tq_decode_attention_ex(layout, q, q_dtype, d_seq_lens, k_codes, k_scales, v_codes, v_scales, sm_scale, out,
                                workspace, ws_bytes, d_status, nullptr, stream);
}

int tq_dequantize_debug(const tq_layout_t* layout, const uint8_t* codes, const uint16_t* scales,
                        const int32_t* d_seq_lens, int original_domain, float* out, void* stream) {
  int r = check_layout(layout);
  if (r != TQ_OK) return r;
  if (!codes || !scales || !d_seq_lens || !out) return TQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(out)) return TQ_ERR_INVALID_ARG;
  tqk::DequantParams p;
  p.codes = codes;
  p.scales = scales;
  p.seq_lens = d_seq_lens;
  p.out = out;
  p.batch = layout->batch;
  p.max_seq = layout->max_seq;
  p.n_kv = layout->n_kv_heads;
  p.original_domain = original_domain ? 1 : 0;
  p.status = nullptr;
  copy_signs(layout, p.sign_bits);
  p.c_d = layout->c_d;
  cudaError_t e = tqk::launch_dequantize(p, layout->head_dim, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TQ_OK : cuda_fail(e);
}

const char* tq_status_string(int status) {
  switch (status) {
    case TQ_OK: return "ok";
    case TQ_ERR_INVALID_ARG: return "invalid argument";
    case TQ_ERR_UNSUPPORTED: return "unsupported shape";
    case TQ_ERR_CAPACITY: return "capacity exceeded";
    case TQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

int tq_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
