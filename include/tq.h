/*
 * tq.h - C ABI of the B200 (sm_100a) library for rotation-based int4 KV-cache
 * quantisation and decode attention computed on the packed cache.
 *
 * The method (sources cited by page title and section):
 *  - "Open-TQ-Metal: Fused Compressed-Domain Attention for Long-Context LLM
 *    Inference on Apple Silicon", abstract (cards page): each cached K/V head
 *    vector goes through one fused quantiser: a sign-randomised transform,
 *    per-group abs-max scaling, int4 codes packed two per byte. The paper
 *    exposes it as a cache object that quantises on append.
 *  - the same paper's arXiv abstract: attention runs directly on the
 *    compressed representation with no intermediate dequantised K/V matrix;
 *    the attention scale (1/sqrt(d) or a model's own, e.g. 1.0) is an input.
 *  - mlxcel user guide "TurboQuant KV cache compression", §"What TurboQuant
 *    changes" (Walsh-Hadamard rotation before low-bit storage) and §"Known
 *    limitations / head dimension" (power-of-two head dims only; others are
 *    rejected when the cache is created).
 *  - "TurboQuant on AMD GPUs", §4: the Walsh-Hadamard transform is used as the
 *    rotation because it spreads energy evenly and suits GPU kernels.
 *  - the mlxcel guide, §"Cache modes": the recommended default mode keeps K in
 *    FP16 and compresses only V (K decides where attention looks, V is mixed
 *    after); that asymmetric cache is TQ_K_FP16 below.
 *  - the mlxcel guide, §"Cache modes" (turbo4-delegated row) and §"Delegated
 *    cache variant": K in FP16, the most recent V tokens kept in FP16 and older
 *    ones stored in the 4-bit form; that cache is TQ_KV_DELEGATED below.
 *
 * Conventions fixed by this library where the pages are silent:
 *  - rotation: y = c_D * H * (s o x), H the Sylvester Hadamard matrix applied
 *    as radix-2 butterflies with stride 1, 2, ..., D/2; c_D = binary32(1/sqrt(D))
 *    applied once; s a +-1 vector drawn from SplitMix64(sign_seed), shared by
 *    K, V, q and every head;
 *  - groups of 32 consecutive rotated elements; scale = binary16(absmax / 7),
 *    codes = clamp(round_half_even(y / scale), -7, 7) against the stored scale;
 *  - packing: two's-complement nibbles, element 2j in the low nibble of byte j.
 *
 * Memory (all buffers are owned by the caller; the library allocates nothing
 * and keeps no state between calls):
 *  - codes  [batch][max_seq][n_kv_heads][head_dim/2]  uint8   (one buffer for K, one for V)
 *  - scales [batch][max_seq][n_kv_heads][head_dim/32] binary16 bits (one for K, one for V)
 *  - with k_format TQ_K_FP16, K is instead one binary16 buffer
 *    [batch][max_seq][n_kv_heads][head_dim] (k_bytes) in the original domain and
 *    has no scales; V keeps its codes and scales.
 *  - with k_format TQ_KV_DELEGATED, K is the binary16 buffer as above and V
 *    has, besides its codes and scales, a binary16 hot tail
 *    [batch][tail_window][n_kv_heads][head_dim] (tail_bytes): token t of a
 *    sequence of len tokens is "cold" (int4 codes at position t) when
 *    t < tq_cold_length(layout, len), else "hot" (binary16 in tail slot
 *    t % tail_window).
 *    Allocate `scales_bytes` (slightly more than the array): decode reads
 *    scale rows in tile-sized blocks that may run past the last valid token.
 *  - every device buffer must be 16-byte aligned (cudaMalloc gives 256).
 *
 * Errors: argument errors return a negative tq_status and launch nothing.
 * Errors found on the device (a length past max_seq, a non-finite group, a
 * bounded wait that ran out) are OR-ed into *d_status when d_status is not
 * NULL (bits TQ_STATUS_*); the affected unit is skipped, never trapped.
 * All calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 * default stream). The library never aborts the process.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = -1, /* NULL pointer, bad size, misaligned buffer, workspace too small */
  TQ_ERR_UNSUPPORTED = -2, /* head_dim not a power of two in [32, 256], group_size != 32, shape limits */
  TQ_ERR_CAPACITY = -3,    /* n_new larger than max_seq */
  TQ_ERR_CUDA = -4         /* a CUDA launch or runtime call failed (see tq_last_cuda_error) */
} tq_status;

/* Bits OR-ed into *d_status by device code. */
#define TQ_STATUS_NONFINITE 1 /* a group held a non-finite value, or its scale overflowed binary16: stored as scale +inf, codes 0 */
#define TQ_STATUS_CAPACITY 2  /* an append past max_seq (that sequence skipped), or seq_len outside [0, max_seq] (treated as 0) */
#define TQ_STATUS_TIMEOUT 4   /* a bounded pipeline wait ran out; that work unit's output is incomplete */

typedef enum { TQ_F32 = 0, TQ_BF16 = 1, TQ_F16 = 2 } tq_dtype;

/* How K is stored (V is always rotated int4 codes + binary16 group scales). */
typedef enum {
  TQ_K_INT4 = 0,      /* K encoded like V (the symmetric cache) */
  TQ_K_FP16 = 1,      /* K as binary16 (round to nearest even) of the input, original domain */
  TQ_KV_DELEGATED = 2 /* K as TQ_K_FP16; V as a binary16 hot tail folded into int4 codes (tq_cache_layout_delegated) */
} tq_k_format;

/* Filled by tq_cache_layout; plain data, caller-owned, never modified by the library. */
typedef struct {
  int32_t batch, max_seq, n_kv_heads, n_q_heads, head_dim, group_size;
  int32_t n_groups;            /* head_dim / 32 */
  float c_d;                   /* binary32(1/sqrt(head_dim)) */
  uint64_t sign_seed;
  uint64_t sign_bits[4];       /* bit i set <=> s_i = -1 (head_dim <= 256) */
  int64_t code_stride_tok;     /* bytes between tokens of one sequence   = n_kv * D/2 */
  int64_t code_stride_seq;     /* bytes between sequences                 = max_seq * n_kv * D/2 */
  int64_t scale_stride_tok;    /* binary16 elements between tokens         = n_kv * D/32 */
  int64_t scale_stride_seq;    /* binary16 elements between sequences      = max_seq * n_kv * D/32 */
  uint64_t codes_bytes;        /* allocation size of ONE codes buffer (K or V) */
  uint64_t scales_bytes;       /* allocation size of ONE scales buffer, including read-ahead padding */
  uint64_t decode_workspace_bytes; /* workspace tq_decode_attention needs with default options */
  int32_t max_ctas;            /* largest split-K grid the workspace size allows */
  int32_t k_format;            /* tq_k_format */
  uint64_t k_bytes;            /* allocation size of the K buffer (codes_bytes for TQ_K_INT4) */
  int64_t k_stride_tok;        /* bytes between tokens of one sequence in the K buffer */
  int64_t k_stride_seq;        /* bytes between sequences in the K buffer */
  int32_t tail_window;         /* TQ_KV_DELEGATED: hot V tokens kept in binary16 (W); 0 otherwise */
  int32_t fold_chunk;          /* TQ_KV_DELEGATED: tokens folded into the int4 body at a time (F); 0 otherwise */
  uint64_t tail_bytes;         /* allocation size of the hot tail (0 unless TQ_KV_DELEGATED) */
  int64_t tail_stride_tok;     /* bytes between tail slots of one sequence = n_kv * D * 2 */
  int64_t tail_stride_seq;     /* bytes between sequences in the tail     = W * n_kv * D * 2 */
  int32_t page_tokens;         /* paged storage: tokens per page (P); 0 = per-sequence slabs */
  int32_t n_pages;             /* paged storage: pages in each pool */
  int32_t max_pages;           /* paged storage: block-table entries per sequence = ceil(max_seq / P) */
  int32_t reserved_paged;
} tq_layout_t;

/* Optional knobs for tq_decode_attention_ex / _delegated (NULL = defaults; zero-fill unused fields). */
typedef struct {
  int32_t min_split_tokens; /* 0 = default (64); otherwise the smallest token range one CTA takes */
  int32_t max_ctas;         /* 0 = default (one per SM); otherwise the split-K grid, <= layout.max_ctas */
  void* after_split_event;  /* a cudaEvent_t recorded on `stream` between the split-K and merge kernels, or NULL */
  /* Per-channel lambda the cache was written with (tq_append_opts_t), device
   * float32 [head_dim], 16-byte aligned, positive and finite; NULL = identity.
   * lambda_k only with int4 K; neither with the delegated cache. */
  const float* lambda_k;
  const float* lambda_v;
  /* Sparse-V threshold (mlxcel guide, §"Sparse-V dequant threshold"; the guide's
   * default is 1e-6): 0 = off (exact attention). Otherwise the V term of an int4
   * V token is dropped when its softmax weight relative to the running maximum
   * of its split range is below the threshold; the softmax sum keeps every
   * token. A dropped token's normalised weight is then below the threshold too,
   * so the output moves by at most sum over dropped t of w_t |V_t|. A unit of
   * 16-32 tokens whose weights all fall below skips its V decode and MMAs.
   * Head dims 64 and 128 (otherwise TQ_ERR_UNSUPPORTED). */
  float sparse_v_threshold;
  /* Bound on every pipeline wait of the split-K kernel (a warp waiting for a
   * tile's copies, its converted scales, or a free stage), in nanoseconds of
   * the GPU's global timer: 0 = the default of one second; negative is
   * TQ_ERR_INVALID_ARG. A wait that runs out sets TQ_STATUS_TIMEOUT, the warp
   * stops reading tiles (its partials are then incomplete) and the call still
   * returns; the copy engine's copies already in flight are always waited for
   * (with the default bound) before a block exits. A short bound is a way to
   * exercise that path; no real input needs anything but the default. */
  int64_t wait_limit_ns;
} tq_decode_opts_t;

/* Optional knobs for tq_quantize_append_ex (NULL = defaults). */
typedef struct {
  /* Per-channel lambda (Open-TQ-Metal abstract: the fused quantiser's steps are
   * the transform, a per-channel lambda, the per-group abs-max and the pack):
   * the rotated vector y is multiplied by lambda (one binary32 multiply per
   * element) before the abs-max. Device float32 [head_dim], 16-byte aligned,
   * positive and finite (not checked on the device); NULL = identity. lambda_k
   * only with int4 K. The decode must be given the same vectors. */
  const float* lambda_k;
  const float* lambda_v;
} tq_append_opts_t;

/*
 * Validate a cache shape and fill *out. Host only: no device work, no CUDA
 * call. head_dim must be a power of two in [32, 256] (mlxcel §"Known
 * limitations / head dimension"); group_size must be 32; n_q_heads must be a
 * multiple of n_kv_heads (grouped-query attention, kv head = q head / G).
 * Returns TQ_OK, TQ_ERR_INVALID_ARG or TQ_ERR_UNSUPPORTED.
 */
int tq_cache_layout(int batch, int max_seq, int n_kv_heads, int n_q_heads, int head_dim,
                    int group_size, uint64_t sign_seed, tq_layout_t* out);

/*
 * As tq_cache_layout, with the K storage format (tq_k_format). TQ_K_FP16 is the
 * asymmetric cache of the mlxcel guide's recommended mode: K kept as binary16
 * (an input beyond the binary16 range is stored as +-inf and sets
 * TQ_STATUS_NONFINITE), V compressed. tq_cache_layout(...) equals
 * tq_cache_layout_kv(..., TQ_K_INT4, out). Unknown formats: TQ_ERR_INVALID_ARG.
 */
int tq_cache_layout_kv(int batch, int max_seq, int n_kv_heads, int n_q_heads, int head_dim,
                       int group_size, uint64_t sign_seed, int k_format, tq_layout_t* out);

/*
 * Delegated hot/cold cache (mlxcel guide, §"Cache modes", turbo4-delegated row,
 * and §"Delegated cache variant"; the pages give no window sizes, so both are
 * the caller's). K is stored as in TQ_K_FP16. V keeps the most recent tokens in
 * binary16 in a ring of tail_window (W) slots per (sequence, kv head) and folds
 * the oldest, fold_chunk (F) at a time, into the int4 body: a sequence of len
 * tokens has tq_cold_length(len) = 0 for len <= W, else
 * F * ceil((len - W) / F) cold tokens, so between W - F + 1 and W stay hot.
 * 1 <= F <= W <= 1024; other arguments as tq_cache_layout_kv. Host only.
 */
int tq_cache_layout_delegated(int batch, int max_seq, int n_kv_heads, int n_q_heads, int head_dim,
                              int group_size, uint64_t sign_seed, int tail_window, int fold_chunk,
                              tq_layout_t* out);

/*
 * Paged storage (mlxcel guide, §"Known limitations / paged KV scheduler": the
 * paged decode storage backend; it cites PagedAttention). The caches become
 * pools of n_pages pages of P = page_tokens tokens: codes
 * [n_pages * P][n_kv_heads][head_dim/2], scales [n_pages * P][n_kv_heads][head_dim/32]
 * (binary16 K [n_pages * P][n_kv_heads][head_dim] with TQ_K_FP16), i.e. the
 * contiguous layout with batch * max_seq rows replaced by n_pages * P rows. A
 * caller-owned device block table int32 [batch][max_pages] maps token t of
 * sequence b to pool row table[b][t / P] * P + t % P. P is a power of two,
 * at least the decode kernel's token tile for this shape (16 to 256; else
 * TQ_ERR_UNSUPPORTED) and at most 4096. k_format TQ_K_INT4 or TQ_K_FP16.
 */
int tq_cache_layout_paged(int batch, int max_seq, int n_kv_heads, int n_q_heads, int head_dim, int group_size,
                          uint64_t sign_seed, int k_format, int page_tokens, int n_pages, tq_layout_t* out);

/*
 * tq_quantize_append_ex on a paged layout. d_block_table: device int32
 * [batch][max_pages]; every page a token lands in must be mapped (an entry
 * outside [0, n_pages) skips that token's vectors and sets TQ_STATUS_CAPACITY).
 */
int tq_quantize_append_paged(const tq_layout_t* layout, const void* k, const void* v, int in_dtype, int n_new,
                             const int32_t* d_start_pos, const int32_t* d_block_table, uint8_t* k_codes,
                             uint16_t* k_scales, uint8_t* v_codes, uint16_t* v_scales, const tq_append_opts_t* opts,
                             int32_t* d_status, void* stream);

/*
 * tq_decode_attention_ex on a paged layout: the split-K kernel's token tiles
 * are read through the block table (each tile lies in one page). A table entry
 * outside [0, n_pages) on a sequence's token range reads zeros for that tile
 * and sets TQ_STATUS_CAPACITY. Workspace as layout->decode_workspace_bytes.
 */
int tq_decode_attention_paged(const tq_layout_t* layout, const void* q, int q_dtype, const int32_t* d_seq_lens,
                              const int32_t* d_block_table, const uint8_t* k_codes, const uint16_t* k_scales,
                              const uint8_t* v_codes, const uint16_t* v_scales, float sm_scale, float* out,
                              void* workspace, size_t ws_bytes, int32_t* d_status, const tq_decode_opts_t* opts,
                              void* stream);

/* Cold (int4) tokens of a delegated-cache sequence of len tokens; len for other
 * formats; -1 for a NULL layout or len < 0. Host only. */
int64_t tq_cold_length(const tq_layout_t* layout, int64_t len);

/*
 * Quantise and append n_new tokens to every sequence (Open-TQ-Metal abstract:
 * the fused sign-randomised transform + per-group abs-max + int4 nibble pack,
 * run when the cache is appended to).
 *   k, v         device, [batch][n_new][n_kv_heads][head_dim] of in_dtype
 *   d_start_pos  device int32 [batch]: token t of sequence b is written at
 *                position d_start_pos[b] + t. A sequence whose append would
 *                pass max_seq (or a negative start) is skipped and sets
 *                TQ_STATUS_CAPACITY.
 *   k_codes, v_codes, k_scales, v_scales   device caches (layout above). With
 *                layout->k_format == TQ_K_FP16, k_codes is the binary16 K buffer
 *                and k_scales is not used (may be NULL).
 * n_new == 0 is a no-op. Codes and scales are bit-exact with the reference
 * definition (IEEE binary32 steps, no contraction, round-half-even).
 * A TQ_KV_DELEGATED layout returns TQ_ERR_INVALID_ARG (use tq_append_delegated).
 */
int tq_quantize_append(const tq_layout_t* layout, const void* k, const void* v, int in_dtype,
                       int n_new, const int32_t* d_start_pos, uint8_t* k_codes, uint16_t* k_scales,
                       uint8_t* v_codes, uint16_t* v_scales, int32_t* d_status, void* stream);

/* tq_quantize_append with options (opts may be NULL). */
int tq_quantize_append_ex(const tq_layout_t* layout, const void* k, const void* v, int in_dtype, int n_new,
                          const int32_t* d_start_pos, uint8_t* k_codes, uint16_t* k_scales, uint8_t* v_codes,
                          uint16_t* v_scales, const tq_append_opts_t* opts, int32_t* d_status, void* stream);

/*
 * One decode query per sequence over its packed cache (Open-TQ-Metal arXiv
 * abstract: attention directly on the compressed representation).
 *   q            device [batch][n_q_heads][head_dim] of q_dtype
 *   d_seq_lens   device int32 [batch]: attend to positions [0, len_b); len_b == 0
 *                gives a zero output row; len_b outside [0, max_seq] is treated
 *                as 0 and sets TQ_STATUS_CAPACITY.
 *   sm_scale     softmax scale (1/sqrt(head_dim) for standard models)
 *   out          device float32 [batch][n_q_heads][head_dim], original (unrotated) domain
 *   workspace    device scratch of at least layout.decode_workspace_bytes
 *                (split-K partials: running max, sum and rotated-domain
 *                accumulator per q head and split; no dequantised K/V is
 *                ever written)
 * The query is rotated by the same transform, K and V nibbles are unpacked in
 * registers, softmax runs online over split-K token ranges, the partials are
 * merged, and one inverse transform produces the output. With
 * layout->k_format == TQ_K_FP16, k_codes is the binary16 K buffer (k_scales
 * unused, may be NULL): the scores use the unrotated query against it, the V
 * side is unchanged.
 * Limits: batch <= 1024; n_kv_heads in {1, 2, 4, 8}; n_q_heads / n_kv_heads <= 8
 * (otherwise TQ_ERR_UNSUPPORTED).
 */
int tq_decode_attention(const tq_layout_t* layout, const void* q, int q_dtype,
                        const int32_t* d_seq_lens, const uint8_t* k_codes, const uint16_t* k_scales,
                        const uint8_t* v_codes, const uint16_t* v_scales, float sm_scale, float* out,
                        void* workspace, size_t ws_bytes, int32_t* d_status, void* stream);

/*
 * Append to a delegated cache (layout from tq_cache_layout_delegated). Every
 * new K vector is stored as binary16. Each sequence's V grows from
 * len0 = d_start_pos[b] to len1 = len0 + n_new tokens: tokens that end up
 * hot are written to the tail as binary16; tokens below tq_cold_length(len1)
 * are encoded (SRHT, per-group abs-max, int4) from their binary16 value -
 * taken from the tail if they were hot before, from the input otherwise - so
 * the cache does not depend on how the tokens were split into calls.
 *   v_tail   device binary16 [batch][W][n_kv_heads][head_dim] (layout->tail_bytes)
 * d_start_pos[b] must be the sequence's current length: the tail holds the
 * tokens [tq_cold_length(len0), len0) only. Slots of folded tokens keep stale
 * values. Other arguments, limits and status bits as tq_quantize_append.
 */
int tq_append_delegated(const tq_layout_t* layout, const void* k, const void* v, int in_dtype, int n_new,
                        const int32_t* d_start_pos, uint16_t* k_f16, uint8_t* v_codes, uint16_t* v_scales,
                        uint16_t* v_tail, int32_t* d_status, void* stream);

/*
 * Decode over a delegated cache: the split-K kernel runs on the cold tokens
 * [0, tq_cold_length(len_b)) exactly as for TQ_K_FP16; the merge kernel also
 * attends to the hot tokens (binary16 K and V, fp32 arithmetic) and combines
 * the two segments by their running max and sum before writing the output.
 * Arguments as tq_decode_attention_ex, plus v_tail; the workspace is
 * layout->decode_workspace_bytes as usual. head_dim <= 128.
 */
int tq_decode_attention_delegated(const tq_layout_t* layout, const void* q, int q_dtype,
                                  const int32_t* d_seq_lens, const uint16_t* k_f16, const uint8_t* v_codes,
                                  const uint16_t* v_scales, const uint16_t* v_tail, float sm_scale, float* out,
                                  void* workspace, size_t ws_bytes, int32_t* d_status,
                                  const tq_decode_opts_t* opts, void* stream);

/* tq_decode_attention with explicit options (opts may be NULL). A
 * TQ_KV_DELEGATED layout returns TQ_ERR_INVALID_ARG here and in
 * tq_decode_attention / tq_decode_attention_noalloc. */
int tq_decode_attention_ex(const tq_layout_t* layout, const void* q, int q_dtype,
                           const int32_t* d_seq_lens, const uint8_t* k_codes, const uint16_t* k_scales,
                           const uint8_t* v_codes, const uint16_t* v_scales, float sm_scale, float* out,
                           void* workspace, size_t ws_bytes, int32_t* d_status,
                           const tq_decode_opts_t* opts, void* stream);

/*
 * Decode for callers that cannot allocate device memory. (The paper has no
 * counterpart: this is a deployment variant of tq_decode_attention.)
 *
 * Who needs it: code that runs where a cudaMalloc is not allowed or not
 * possible - inside a memory pool or custom allocator that must not re-enter
 * itself, runtimes with a fixed device-memory plan made at start-up, plug-ins
 * that are handed only their input and output tensors. tq_decode_attention
 * needs a caller-allocated workspace; this call instead uses a scratch array
 * of TQ_NOALLOC_WORKSPACE_BYTES that is part of the library's own device image
 * (a static device array: every GPU that loads the library holds it until the
 * process exits). Inputs, outputs, results and limits are otherwise those of
 * tq_decode_attention with the default one-CTA-per-SM split.
 *
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it, keyed on
 *    the device and on the unique id of the current context; make that first
 *    call before any stream capture on that device. After cudaDeviceReset (or
 *    in another context) the next call looks the address up again, so that
 *    call too should come before any capture.
 *  - A request whose workspace would exceed TQ_NOALLOC_WORKSPACE_BYTES
 *    (roughly (SMs + batch) * n_q_heads * (head_dim + 2) * 4 bytes) returns
 *    TQ_ERR_CAPACITY and launches nothing.
 *  - Every call on a device shares the one array, which keeps the last call's
 *    contents (nothing in it needs clearing: each call writes all it reads).
 *    Calls that can overlap on the GPU (different streams, or other threads)
 *    race on it: serialise them.
 *  - Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define TQ_NOALLOC_WORKSPACE_BYTES (8u << 20)
int tq_decode_attention_noalloc(const tq_layout_t* layout, const void* q, int q_dtype,
                                const int32_t* d_seq_lens, const uint8_t* k_codes, const uint16_t* k_scales,
                                const uint8_t* v_codes, const uint16_t* v_scales, float sm_scale, float* out,
                                int32_t* d_status, void* stream);

/*
 * Debug / comparator path: dequantise a whole cache into a dense float32
 * array out [batch][max_seq][n_kv_heads][head_dim]; rows at t >= d_seq_lens[b]
 * are written as 0. original_domain = 0 gives code * scale (rotated domain);
 * 1 also applies the inverse rotation. This is the "dequantise-then-attend"
 * baseline's first half (Open-TQ-Metal arXiv abstract); the decode path never
 * calls it.
 */
int tq_dequantize_debug(const tq_layout_t* layout, const uint8_t* codes, const uint16_t* scales,
                        const int32_t* d_seq_lens, int original_domain, float* out, void* stream);

/* Human-readable text for a tq_status value. Never NULL. */
const char* tq_status_string(int status);

/* The last CUDA error code seen by a call that returned TQ_ERR_CUDA (0 if none). */
int tq_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
