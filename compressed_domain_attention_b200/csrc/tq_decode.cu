// Split-K decode attention on the packed int4 cache (sm_100a).
//
// Open-TQ-Metal (arXiv abstract): attention is computed directly on the
// compressed representation, never materialising a dequantised K/V matrix.
// The rotation is orthogonal, so q.k and sum_t p_t v_t can be evaluated in the
// rotated domain: the query is rotated once, the packed codes are unpacked in
// registers, and one inverse rotation is applied to the merged output. The
// softmax is the online (running max / running sum) form of the "online
// normaliser" paper the index page lists under "Builds on", merged across
// split-K token ranges by a log-sum-exp combine.
//
// Kernel 1 (decode_split_kernel): one CTA per SM. The flattened token space of
// all sequences is cut into equal ranges, one per CTA; a range may straddle
// sequences, and each (sequence, range) piece writes one partial
// (running max m, running sum l, rotated-domain accumulator acc[D]) per q head
// into the workspace slot (sequence + CTA index), which is unique.
//   warp 8      : producer. One lane streams token tiles of the contiguous
//                 [tile][Hkv][D/2] code slabs (3-D tensor copies, swizzled to
//                 the row pitch) and the [tile][Hkv][D/32] binary16 scale slabs
//                 (bulk copies) into a 3- or 4-stage shared-memory ring guarded
//                 by mbarriers.
//   warp 9      : converter. Turns each stage's binary16 scales into fp32 in
//                 the order the consumer lanes read them (conflict-free), with
//                 tokens past the segment end set to 0.
//   warps 0..7  : consumers. Warp w owns KV head w % Hkv and 32-token units
//                 (16 at D = 256) of each tile. Scores and P.V run on the tensor cores with
//                 register fragments (mma.m16n8k16, f16 in, f32 accumulate):
//                 * Q.K^T: A = the rotated query of the group's q heads in
//                   two binary16 pieces (hi + lo, rows 0-7 and 8-15), B = K
//                   codes. A code nibble u (offset binary) enters the tensor
//                   core as the exact binary16 subnormal u * 2^-24 (a single
//                   lop3 per pair); the "-8" offset is folded into the
//                   accumulator's initial value, and the per-group scale is
//                   applied in binary32 after each group's two MMAs.
//                 * P.V: A = V codes (pairs of tokens at one channel, from a
//                   transposing ldmatrix, same subnormal encoding), B = P
//                   times the per-(token, group) V scale, rounded once to
//                   binary16. The V codes enter signed (one binary16
//                   subtract per pair removes the +8): an offset kept in
//                   the accumulator would drift, because the tensor core's
//                   fp32 sums round toward zero.
// Kernel 2 (decode_merge_kernel): per (sequence, q head) the partials are
// combined, normalised, and the inverse SRHT maps the result back to the
// original domain.
#include <cuda.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

constexpr int kConsumerWarps = 8;
constexpr int kProducerWarp = kConsumerWarps;       // one lane issues the copies
constexpr int kConverterWarp = kConsumerWarps + 1;  // first of the binary16 -> fp32 scale warps
constexpr int kConverterWarps = 3;                  // one on each scheduler without the producer
constexpr int kThreads = (kConsumerWarps + 1 + kConverterWarps) * 32;
constexpr int kMaxBatch = 1024;
constexpr int kMergeThreads = 128;     // merge blocks when (sequence, head) pairs are many
constexpr int kMergeThreadsFew = 512;  // and when they number fewer than twice the split CTAs
constexpr uint64_t kDrainLimitNs = 1000000000ull;  // 1 s bound on the producer's wait for its copies in flight

// KF16: K tiles are binary16 in the original domain (asymmetric cache), the V
// side is unchanged; no K scales are copied or converted.
template <int D, int HKV, bool KF16 = false>
struct DecodeCfg {
  static constexpr int NG = D / 32;                  // groups per head vector
  static constexpr int RB = D / 2;                   // V (and int4 K) code bytes per (token, head)
  static constexpr int KRB = KF16 ? 2 * D : RB;      // K bytes per (token, head)
  static constexpr int WPH = kConsumerWarps / HKV;   // consumer warps per KV head
  // tokens per warp work unit (16 where a 32-token binary16 K tile would not fit)
  static constexpr int UNIT = (KF16 && D == 128) || D == 256 ? 16 : 32;
  static constexpr int NT = UNIT / 8;                // 8-token n-tiles per unit
  static constexpr int KSP = UNIT / 16;              // 16-token k-steps of P.V per unit
  // units per warp per stage: K tile of at most 16 KB (int4) or 32 KB (binary16)
  static constexpr int UPW_A0 = KF16 ? 4096 / (UNIT * KRB) : 2048 / (UNIT * RB);
  static constexpr int UPW_A = UPW_A0 > 0 ? UPW_A0 : 1;
  static constexpr int UPW_B = 256 / (UNIT * WPH) > 0 ? 256 / (UNIT * WPH) : 1;
  static constexpr int UPW = UPW_A < UPW_B ? UPW_A : UPW_B;
  static constexpr int T_TILE = UNIT * UPW * WPH;    // tokens per stage (<= 256)
  static constexpr int UNITS_TILE = T_TILE / UNIT;
  static constexpr int CODE_BYTES = T_TILE * HKV * RB;   // V tile
  static constexpr int K_BYTES = T_TILE * HKV * KRB;     // K tile
  static constexpr int SROW = HKV * NG * 2;          // raw scale bytes per token (all heads)
  static constexpr int SCALE_SLAB = ((T_TILE * SROW + 15) / 16) * 16 + 16;
  static constexpr int SC_HEAD = T_TILE * NG + 4;    // fp32 scale floats per head (16 B pad)
  static constexpr int SC_KV = HKV * SC_HEAD;
  static constexpr int NSC = KF16 ? 1 : 2;           // scale sets in a stage (K and V, or V)
  // stage: [K tile][V tile][raw scale slabs (K, V)][fp32 scales (K, V)]
  static constexpr int OFF_VCODE = K_BYTES;
  static constexpr int OFF_RAW = K_BYTES + CODE_BYTES;           // first raw slab
  static constexpr int OFF_RAWV = OFF_RAW + (NSC - 1) * SCALE_SLAB;
  static constexpr int OFF_SC32 = OFF_RAW + NSC * SCALE_SLAB;
  static constexpr int OFF_SCV = OFF_SC32 + (NSC - 1) * SC_KV * 4;  // fp32 V scales
  static constexpr int STAGE_BYTES = ((OFF_SC32 + NSC * SC_KV * 4 + 1023) / 1024) * 1024;
  static constexpr uint32_t STAGE_TX = K_BYTES + CODE_BYTES + NSC * SCALE_SLAB;
  static constexpr int STAGES = D == 256 ? 3 : 4;
  static constexpr int QSTRIDE = D + 4;              // floats per staged q row (padded)
  static constexpr int SCRATCH = ((8 * QSTRIDE * 4 + 64 + 127) / 128) * 128;  // per consumer warp
  static constexpr int SWZ = RB == 128 ? 7 : RB == 64 ? 3 : RB == 32 ? 1 : 0;
  // binary16 K: 128-byte lines (64 halves; one 64-byte line at D = 32), swizzled
  static constexpr int KLINE = D < 64 ? 2 * D : 128;
  static constexpr int KNCH = 2 * D / KLINE;         // lines per (token, head)
  static constexpr int KSWZ = KLINE == 128 ? 7 : 3;
  static constexpr int OFF_SCRATCH = STAGES * STAGE_BYTES;
  static constexpr int OFF_BARS = OFF_SCRATCH + kConsumerWarps * SCRATCH;
  static constexpr int OFF_MISC = OFF_BARS + 3 * STAGES * 8;
  static constexpr int OFF_PREFIX = OFF_MISC + 64;
  static constexpr int SMEM_MAX = OFF_PREFIX + 8 * (kMaxBatch + 1) + 8 * 16;
  static_assert(T_TILE <= 256, "tensor-copy box limit");
  static_assert((T_TILE & (T_TILE - 1)) == 0, "paged storage rounds lengths to tiles with a mask");
  static_assert(CODE_BYTES % 1024 == 0 && K_BYTES % 1024 == 0, "tiles must stay swizzle-aligned");
  static_assert((2 * NG * NT) % 4 == 0, "ldmatrix.x4 batches");
  static_assert(SMEM_MAX <= 232448, "shared memory per block");
  static_assert(!KF16 || D <= 128, "binary16 K tiles up to head_dim 128");
};

// Workspace header: int64 prefix[batch + 1], int64 range_tokens.
__device__ __forceinline__ int64_t* ws_header(float* ws_ml) { return reinterpret_cast<int64_t*>(ws_ml); }

// Exclusive prefix sum of the validated lengths into prefix[0..batch]; all
// threads of the block call this. Lengths outside [0, max_seq] count as 0.
__device__ void block_prefix_lengths(const DecodeParams& p, int64_t* prefix, int64_t* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int PER = (kMaxBatch + kThreads - 1) / kThreads;
  int64_t v[PER];
  int64_t local = 0;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int b = tid * PER + i;
    int64_t L = 0;
    if (b < p.batch) {
      const int x = p.seq_lens[b];
      if (x < 0 || x > p.max_seq) {
        bad = true;
      } else {  // padded to whole tiles with paged storage (len_align 1 otherwise)
        L = cold_tokens(x, p.tail_window, p.fold_chunk);
        L = (L + p.len_align - 1) & ~(int64_t)(p.len_align - 1);  // len_align is a power of two
      }
    }
    v[i] = L;
    local += L;
  }
  if (bad && blockIdx.x == 0) status_or(p.status, TQ_STATUS_CAPACITY);
  int64_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (tid == 0) {
    int64_t run = 0;
    for (int w = 0; w < kThreads / 32; ++w) {
      const int64_t t = warp_tot[w];
      warp_tot[w] = run;
      run += t;
    }
  }
  __syncthreads();
  int64_t run = warp_tot[warp] + incl - local;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int b = tid * PER + i;
    if (b < p.batch) prefix[b] = run;
    run += v[i];
  }
  if (tid == kThreads - 1) prefix[p.batch] = run;  // the last thread's running total is the full sum
  __syncthreads();
}

// First cache row of the tile of sequence b starting at token t0: b * max_seq + t0,
// or through the block table with paged storage (the tile lies in one page). An
// unmapped page gives ok = false and row 0 (the producer then points its tensor
// copies past the pool, where they read zeros, and copies its scales from row 0;
// the converters must locate the scales at the same row).
__device__ __forceinline__ int64_t tile_first_row(const DecodeParams& p, int b, int t0, bool& ok) {
  ok = true;
  if (p.page_tokens <= 0) return (int64_t)b * p.max_seq + t0;
  const int pg = p.block_table[(int64_t)b * p.max_pages + t0 / p.page_tokens];
  ok = pg >= 0 && pg < p.n_pages;
  return ok ? (int64_t)pg * p.page_tokens + t0 % p.page_tokens : 0;
}

// Tile walk shared by the producer and the consumers: visits every
// (sequence b, token offset t0, tokens valid in the tile) of this CTA's range.
struct TileWalker {
  const int64_t* prefix;
  int batch;
  int64_t lo, hi;
  int b;
  int seg_lo, seg_hi, t0;  // token offsets within sequence b (< max_seq)
  const int32_t* lens;     // paged storage: true lengths (the prefix holds padded ones); else nullptr
  int max_seq;

  __device__ void start(const int64_t* pf, int nb, int64_t l, int64_t h, const int32_t* true_lens = nullptr,
                        int ms = 0) {
    prefix = pf;
    batch = nb;
    lo = l;
    hi = h;
    lens = true_lens;
    max_seq = ms;
    // first sequence whose token range ends after lo
    int a = 0, z = nb - 1;
    while (a < z) {
      const int m = (a + z) >> 1;
      if (pf[m + 1] > lo) z = m; else a = m + 1;
    }
    b = a;
    seg_lo = seg_hi = t0 = 0;
    next_segment_from(b);
  }
  // position on the first non-empty segment at or after sequence bb
  __device__ void next_segment_from(int bb) {
    for (b = bb; b < batch && prefix[b] < hi; ++b) {
      const int64_t s0 = max(lo, prefix[b]) - prefix[b];
      int64_t s1 = min(hi, prefix[b + 1]) - prefix[b];
      if (lens != nullptr) {  // the padding past the true length is never read
        const int x = lens[b];
        s1 = min(s1, (int64_t)((x < 0 || x > max_seq) ? 0 : x));
      }
      if (s0 < s1) {
        seg_lo = (int)s0;
        seg_hi = (int)s1;
        t0 = (int)s0;
        return;
      }
    }
    b = batch;  // done
  }
  __device__ bool done() const { return b >= batch; }
  // advance to the next tile; returns true when a new segment starts
  template <int T_TILE>
  __device__ bool advance() {
    t0 += T_TILE;
    if (t0 < seg_hi) return false;
    next_segment_from(b + 1);
    return true;
  }
};

// TOK_M (query groups of at most 4 heads): the score MMAs put 16 tokens in M and
// the query's binary16 hi/lo pieces of 4 heads in the 8 N columns, which halves
// their count; otherwise the 8 heads' hi (rows 0-7) and lo (rows 8-15) pieces
// are the M rows and the tokens the N columns.
template <int D, int HKV, bool TOK_M, bool KF16, bool SPARSE = false>
__global__ void __launch_bounds__(kThreads, 1)
    decode_split_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap) {
  using C = DecodeCfg<D, HKV, KF16>;
  constexpr int NG = C::NG, RB = C::RB, T_TILE = C::T_TILE, UPW = C::UPW, NT = C::NT, KSP = C::KSP;
  constexpr int UNIT = C::UNIT, STAGES = C::STAGES;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BARS);  // copies landed
  uint64_t* ready = full + STAGES;                                  // fp32 scales written
  uint64_t* empty = ready + STAGES;                                 // stage free again
  int* misc = reinterpret_cast<int*>(smem + C::OFF_MISC);           // [0] abort flag
  int64_t* prefix = reinterpret_cast<int64_t*>(smem + C::OFF_PREFIX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Launched as a programmatic dependent of whatever kernel precedes it on the stream
  // (typically the append). Set-up that reads nothing another kernel writes (barrier
  // initialisation, tensor-map prefetch) runs before the dependency wait; no global
  // memory is read before it. L2 prefetches (hints that return no data) of the
  // lengths and the query may go first: L2 is where any later store to them lands.
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], kConverterWarps);
      mbar_init(&empty[s], kConsumerWarps + kConverterWarps);
    }
    misc[0] = 0;
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(&kmap) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&vmap) : "memory");
  } else if (warp == 1) {
    // every block reads all lengths for its prefix sums (one 128-byte line per 32)
    for (int i = lane * 32; i < p.batch; i += 32 * 32) prefetch_l2(p.seq_lens + i);
    if (lane == 0) {
      // the query is read by every block's prologue once the prefix sums are known:
      // each block prefetches one slice of it
      const uint32_t qbytes =
          (uint32_t)p.batch * (uint32_t)p.n_q * (uint32_t)(D * (p.q_dtype == TQ_F32 ? 4 : 2));
      const uint32_t per = ((qbytes + gridDim.x - 1) / gridDim.x + 127u) & ~127u;  // whole 128-byte lines
      const uint32_t o0 = blockIdx.x * per;
      if (o0 < qbytes) {
        const uint32_t n = min(per, qbytes - o0);  // a multiple of 16 (rows of D >= 32 elements)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                     ::"l"(reinterpret_cast<const uint8_t*>(p.q) + o0), "r"(n)
                     : "memory");
      }
    }
  }
  __syncthreads();  // the barriers' initialisation is visible to every thread
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (p.batch == 1) {
    // one sequence: every thread takes its length itself and writes the same two prefix
    // words (each thread reads back its own values), with no block barrier on the way
    // to the first tile copies
    int x = p.seq_lens[0];
    if (x < 0 || x > p.max_seq) {
      if (blockIdx.x == 0 && tid == 0) status_or(p.status, TQ_STATUS_CAPACITY);
      x = 0;
    }
    int64_t L = cold_tokens(x, p.tail_window, p.fold_chunk);
    L = (L + p.len_align - 1) & ~(int64_t)(p.len_align - 1);
    prefix[0] = 0;
    prefix[1] = L;
  } else {
    block_prefix_lengths(p, prefix, prefix + (p.batch + 1));
  }
  const int64_t T_sum = prefix[p.batch];
  // T_sum < 2^32 (batch * max_seq <= INT32_MAX, plus at most a tile of padding per
  // sequence), so the split range takes a 32-bit division
  int64_t R = (uint32_t)(T_sum + p.grid - 1) / (uint32_t)p.grid;
  if (R < p.min_split) R = p.min_split;
  const int64_t r_align = p.len_align > 16 ? p.len_align : 16;  // whole tiles with paged storage (a power of two)
  R = (R + r_align - 1) & ~(r_align - 1);
  if (blockIdx.x == 0) {  // header for the merge kernel
    int64_t* hdr = ws_header(p.ws_ml);
    for (int i = tid; i <= p.batch; i += kThreads) hdr[i] = prefix[i];
    if (tid == 0) hdr[p.batch + 1] = R;
  }
  // the merge grid may be scheduled from here on; it waits for this grid's completion
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t lo = (int64_t)blockIdx.x * R;
  const int64_t hi = min(lo + R, T_sum);
  if (lo >= hi) return;
  // the swizzle decode below assumes 1024-byte aligned stage buffers
  if ((smem_u32(smem) & 1023u) != 0) {
    if (tid == 0) status_or(p.status, TQ_STATUS_TIMEOUT);
    return;
  }

  TileWalker walk;
  walk.start(prefix, p.batch, lo, hi, p.page_tokens > 0 ? p.seq_lens : nullptr, p.max_seq);

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    const uint64_t pol = l2_policy_evict_first();
    const uint8_t* ks_base = reinterpret_cast<const uint8_t*>(p.k_scales);
    const uint8_t* vs_base = reinterpret_cast<const uint8_t*>(p.v_scales);
    int issued = 0;
    bool dead = false;
    for (; !walk.done(); walk.advance<T_TILE>()) {
      const int stage = issued % STAGES;
      const uint32_t n = (uint32_t)(issued / STAGES);
      if (!mbar_wait_bounded(&empty[stage], (n & 1u) ^ 1u, p.wait_ns)) {
        dead = true;
        break;
      }
      // The copies of the tile that last used this stage have landed: a warp that gave up
      // on a wait arrives on `empty` without reading, so `empty` alone does not show it,
      // and `full` must never be re-armed while a phase of it is still waiting for bytes.
      if (n > 0 && !mbar_wait_bounded(&full[stage], (n - 1u) & 1u, kDrainLimitNs)) {
        dead = true;
        break;
      }
      if (*reinterpret_cast<volatile int*>(&misc[0]) != 0) break;
      uint8_t* sb = smem + stage * C::STAGE_BYTES;
      mbar_arrive_expect_tx(&full[stage], C::STAGE_TX);
      // paged storage: the tile lies in one page (tiles start at multiples of the tile
      // size, pages hold whole tiles)
      bool mapped;
      const int srow = (int)tile_first_row(p, walk.b, walk.t0, mapped);  // first scale row of the tile
      if (!mapped) status_or(p.status, TQ_STATUS_CAPACITY);
      const int row = mapped ? srow : p.n_pages * p.page_tokens;  // past the pool: zero-filled copies
      if constexpr (KF16)
        tma_load_4d(sb, &kmap, &full[stage], 0, row, 0, 0, pol);
      else
        tma_load_3d(sb, &kmap, &full[stage], 0, row, 0, pol);
      tma_load_3d(sb + C::OFF_VCODE, &vmap, &full[stage], 0, row, 0, pol);
      const int64_t soff = (int64_t)srow * C::SROW;  // byte offset of the tile's first scale row
      const int64_t salign = soff & ~(int64_t)15;
      if constexpr (!KF16) bulk_load(sb + C::OFF_RAW, ks_base + salign, C::SCALE_SLAB, &full[stage], pol);
      bulk_load(sb + C::OFF_RAWV, vs_base + salign, C::SCALE_SLAB, &full[stage], pol);
      ++issued;
    }
    if (dead) {
      misc[0] = 1;
      status_or(p.status, TQ_STATUS_TIMEOUT);
    }
    // drain: no copy may still be in flight when this thread exits (each stage holds at
    // most one tile's copies, those of the last STAGES tiles issued)
    for (int k = max(0, issued - STAGES); k < issued; ++k)
      (void)mbar_wait_bounded(&full[k % STAGES], (uint32_t)((k / STAGES) & 1), kDrainLimitNs);
    return;
  }

  if (warp >= kConverterWarp) {
    // ------------------------------------------------------------ converters
    // binary16 scale rows [token][head][group] -> fp32 [head][unit][group][tig][n-tile][e],
    // the order in which a consumer lane reads them; tokens past the segment end get 0.
    // Lane work item k covers the token pair (2j, 2j + 1) of one head: both tokens land
    // next to each other (e = 0, 1), so each group is one 8-byte store. Item i = lane +
    // 32 k' takes head hh = i % HKV and, from r = i / HKV, the n-tile r % NT, the pair
    // tg = (r / NT) % 4 within it and the unit r / (4 NT): the lanes of one store then
    // spread over heads and n-tiles, which fall in different banks of the fp32 layout
    // (the order "pairs of one n-tile first" put 4 lanes on each bank pair; it stays
    // with 4 kv heads, where it conflicts less). The
    // shared-memory offsets are the same for every tile. The kConverterWarps warps share
    // the items of a tile.
    constexpr int PAIRS = T_TILE / 2 * HKV;
    constexpr int ITEMS = (PAIRS + 32 * kConverterWarps - 1) / (32 * kConverterWarps);
    const int cw = warp - kConverterWarp;
    // With TOK_M the K scales go to [head][unit][group][token mod 8][m-tile][e] instead
    // (the lanes of a score row read the tokens gid + 8e + 16 m-tile): two 4-byte stores.
    constexpr int MT = UNIT / 16;
    uint32_t src_off[ITEMS], dst_off[ITEMS], dstk_off[ITEMS];
    int tok_of[ITEMS];
#pragma unroll
    for (int k = 0; k < ITEMS; ++k) {
      const int i = lane + 32 * (cw + kConverterWarps * k);
      const int r = i / HKV, hh = i % HKV;
      // a bijection on the pairs; with 4 kv heads the plain order conflicts less
      const int j = HKV == 4 ? r : (r / (4 * NT)) * (UNIT / 2) + 4 * (r % NT) + (r / NT) % 4;
      const int t = 2 * j;
      const int u = t / UNIT, tau = t % UNIT;
      const int nt = tau >> 3, tg = (tau & 7) >> 1;
      src_off[k] = (uint32_t)((t * HKV + hh) * NG * 2);
      dst_off[k] = (uint32_t)(4 * (hh * C::SC_HEAD + (u * NG * 4 + tg) * (2 * NT) + nt * 2));
      dstk_off[k] = (uint32_t)(4 * (hh * C::SC_HEAD + (u * NG * 8 + (tau & 7)) * (2 * MT) + (tau >> 3)));
      tok_of[k] = i < PAIRS ? t : 1 << 30;
    }
    bool dead = false;
    int tile_i = 0;
    for (; !walk.done(); walk.advance<T_TILE>(), ++tile_i) {
      const int stage = tile_i % STAGES;
      const uint32_t par = (uint32_t)((tile_i / STAGES) & 1);
      // (a producer that gave up issues nothing more: these waits then run out)
      if (!dead && !mbar_wait_bounded(&full[stage], par, p.wait_ns)) {
        dead = true;
        if (lane == 0) status_or(p.status, TQ_STATUS_TIMEOUT);
      }
      if (!dead) {
        uint8_t* sb = smem + stage * C::STAGE_BYTES;
        bool mapped;
        const int64_t row0 = tile_first_row(p, walk.b, walk.t0, mapped);  // the producer's scale row
        const int soff = (int)((row0 * C::SROW) & 15);
        // an unmapped page's tile reads as zeros: its codes come from past the pool (zero
        // fill) and its scales are set to 0 here (the slab the producer copied is row 0's)
        const int nv = mapped ? min(T_TILE, walk.seg_hi - walk.t0) : 0;
        const uint32_t sc = smem_u32(sb + C::OFF_SC32);
        const bool part_tile = nv < T_TILE;  // the same for every lane: tokens past nv get 0
#pragma unroll
        for (int kv = KF16 ? 1 : 0; kv < 2; ++kv) {  // binary16 K has no scales
          // the NG scales of a (token, head) are NG x 2 contiguous bytes: one vector load each
          // for the item's two tokens (plain shared loads, which the compiler may batch)
          const uint8_t* raw = sb + (kv ? C::OFF_RAWV : C::OFF_RAW) + soff;
          const uint32_t dst = kv ? smem_u32(sb + C::OFF_SCV) : sc;
#pragma unroll
          for (int k = 0; k < ITEMS; ++k) {
            const int t = tok_of[k];
            if (t >= T_TILE) continue;
            float f0[NG], f1[NG];
            load_scales<NG>(f0, raw + src_off[k]);
            load_scales<NG>(f1, raw + src_off[k] + HKV * NG * 2);
            if (part_tile) {
              const bool ok0 = t < nv, ok1 = t + 1 < nv;
#pragma unroll
              for (int g = 0; g < NG; ++g) {
                f0[g] = ok0 ? f0[g] : 0.f;
                f1[g] = ok1 ? f1[g] : 0.f;
              }
            }
#pragma unroll
            for (int g = 0; g < NG; ++g) {
              if (TOK_M && kv == 0) {
                const uint32_t a = dst + dstk_off[k] + 4 * (g * 8 * 2 * MT);
                sts_f32(a, f0[g]);
                sts_f32(a + 4 * 2 * MT, f1[g]);
              } else {
                sts_f2(dst + dst_off[k] + 4 * (g * 4 * 2 * NT), f0[g], f1[g]);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ready[tile_i % STAGES]);
        mbar_arrive(&empty[tile_i % STAGES]);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int h = warp % HKV;
  const int sub = warp / HKV;
  const int gid = lane >> 2, tig = lane & 3;
  const int G = p.group;
  float* scratch = reinterpret_cast<float*>(smem + C::OFF_SCRATCH + warp * C::SCRATCH);
  const uint32_t smem_base = smem_u32(smem);

  // Per-lane ldmatrix offsets inside a head's [tile][D/2] block, relative to the
  // unit's first row. A unit spans UNIT * RB bytes (a multiple of 1024 B, as is a
  // head block), so the swizzle phase of a row only depends on its row inside
  // the unit. K batch k covers matrices m = 4k..4k+3, m = (group m / NT,
  // n-tile m % NT); V batch k the same with token blocks instead of n-tiles.
  constexpr int NB = NG * NT / 4;
  uint32_t k_off[NB], v_off[NB];
  {
    const int rr = lane & 7, mi = lane >> 3;
#pragma unroll
    for (int kb = 0; kb < NB; ++kb) {
      const int m = 4 * kb + mi;
      const int row = (m % NT) * 8 + rr;
      const int grp = m / NT;
      const int swz = ((h * T_TILE * RB + row * RB) >> 7) & C::SWZ;
      k_off[kb] = (uint32_t)(row * RB + ((grp ^ swz) << 4));
      v_off[kb] = k_off[kb];
    }
  }
  static_assert((UNIT * RB) % 1024 == 0 || C::SWZ == 0 || (UNIT * RB) % ((C::SWZ + 1) * 128) == 0,
                "unit rows must keep the swizzle phase");
  // binary16 K: per-lane ldmatrix offsets of k-step kk inside the head's
  // [line][tile][64] binary16 block, relative to the unit's first token (unit and head
  // offsets are whole multiples of the swizzle period). Row layout (K as B): matrix m = lane / 8
  // is (8-token n-tile m / 2, dims + 8 (m % 2)); tokens-in-M (K as A): matrix m is
  // (token rows 8 (m % 2) .., dims + 8 (m / 2)).
  uint32_t k16_off[KF16 ? 2 * NG : 1];
  if constexpr (KF16) {
    const int m = lane >> 3, r = lane & 7;
    const int tok = TOK_M ? (m & 1) * 8 + r : (m >> 1) * 8 + r;
    const int dadd = TOK_M ? 8 * (m >> 1) : 8 * (m & 1);
    constexpr int HPL = C::KLINE / 2;  // halves per line
#pragma unroll
    for (int kk = 0; kk < 2 * NG; ++kk) {
      const int dims = 16 * kk + dadd;
      const int ch = dims / HPL;
      const int line = ch * T_TILE + tok;
      const int sw = ((line * C::KLINE) >> 7) & C::KSWZ;
      k16_off[kk] = (uint32_t)(line * C::KLINE + ((((dims % HPL) >> 3) ^ sw) << 4));
    }
  }
  static_assert(!KF16 || (UNIT % 16 == 0 && T_TILE % 8 == 0), "binary16 K swizzle phase");

  uint32_t qA[NG][2][4];
  float biasK[NG];
  float f_h = 1.f;
  float acc[NG][2][4];
  float m_run = -INFINITY, l_run = 0.f;
  bool dead = false;
  int tile_i = 0;

  constexpr bool sparse = SPARSE;  // sparse-V threshold set (a separate instantiation)
  while (!walk.done()) {
    const int b = walk.b;
    const int seg_hi = walk.seg_hi;
    // ---------------- segment prologue: rotate this warp's q heads, build fragments
    {
      constexpr int HP = 32 / NG;  // heads rotated per pass
      const int part = lane % NG;
      const uint32_t sw = sign_word(p.sign_bits, part);
      // 1/sqrt(D) of the rotation and the softmax scale in log2 units; binary16 K is not
      // rotated, so neither is q
      const float qs = KF16 ? p.sm_scale_log2 : p.c_d * p.sm_scale_log2;
      for (int j0 = 0; j0 < 8 && j0 < G; j0 += HP) {  // rows j >= G are never read
        const int j = j0 + lane / NG;
        float u[32];
        if (j < G && j < 8) {
          load32(u, p.q, ((int64_t)b * p.n_q + (int64_t)h * G + j) * D + part * 32, p.q_dtype);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = 0.f;
        }
        if constexpr (!KF16) {
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = flip_sign(u[i], sw, i);
          fwht_group_x2<NG>(u, part);
          if (p.lambda_k != nullptr) {  // the cache holds lambda o y: q pairs with y / lambda
            const float4* l4 = reinterpret_cast<const float4*>(p.lambda_k + part * 32);
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 lv = __ldg(l4 + i / 4);
              u[i] = __fdividef(u[i], lv.x);  // a few ulp: far inside the decode tolerance
              u[i + 1] = __fdividef(u[i + 1], lv.y);
              u[i + 2] = __fdividef(u[i + 2], lv.z);
              u[i + 3] = __fdividef(u[i + 3], lv.w);
            }
          }
        }
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 y = __fmul2_rn(make_float2(u[i], u[i + 1]), make_float2(qs, qs));
          u[i] = y.x;
          u[i + 1] = y.y;
          mx = fmaxf(mx, fmaxf(fabsf(y.x), fabsf(y.y)));
        }
#pragma unroll
        for (int o = 1; o < NG; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int e = 0;
        if (mx > 0.f) (void)frexpf(mx, &e);
        const int sh = min(100, max(-100, 14 - e));  // scaled max < 2^14
        if (j < 8) {
          const float sc = __int_as_float((127 + sh) << 23);  // 2^sh, exact scaling
          float4* row = reinterpret_cast<float4*>(scratch + j * C::QSTRIDE + part * 32);
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float2 a = __fmul2_rn(make_float2(u[i], u[i + 1]), make_float2(sc, sc));
            const float2 c = __fmul2_rn(make_float2(u[i + 2], u[i + 3]), make_float2(sc, sc));
            row[i / 4] = make_float4(a.x, a.y, c.x, c.y);
          }
          if (part == 0) reinterpret_cast<int*>(scratch + 8 * C::QSTRIDE)[j] = sh;
        }
      }
      __syncwarp();
      // q pieces in the score operand's k order: k-step ks of a group takes the lane's
      // nibbles {2ks, 2ks + 4} (low position) and {2ks + 1, 2ks + 5} (high position, q / 16).
      // TOK_M: lane (gid, tig) holds piece gid & 1 (hi, lo) of head gid >> 1 as the B
      // operand; otherwise head gid's hi (A rows 0-7) and lo (rows 8-15) pieces.
      const int qh = TOK_M ? (gid >> 1) : gid;
      const float* row = scratch + qh * C::QSTRIDE;
      if constexpr (KF16) {
        // binary16 K: natural k order, k-step kk covers dims 16 kk .. 16 kk + 15; the lane
        // holds dims (2 tig, 2 tig + 1) and (8 + 2 tig, 9 + 2 tig) of it; no code offset
#pragma unroll
        for (int kk = 0; kk < 2 * NG; ++kk) {
          float2 x0 = make_float2(0.f, 0.f), x1 = x0;
          if (qh < G) {
            x0 = *reinterpret_cast<const float2*>(row + 16 * kk + 2 * tig);
            x1 = *reinterpret_cast<const float2*>(row + 16 * kk + 8 + 2 * tig);
          }
          const __half2 h0 = __float22half2_rn(x0), h1 = __float22half2_rn(x1);
          const float2 b0f = __half22float2(h0), b1f = __half22float2(h1);
          const __half2 l0 = __float22half2_rn(make_float2(x0.x - b0f.x, x0.y - b0f.y));
          const __half2 l1 = __float22half2_rn(make_float2(x1.x - b1f.x, x1.y - b1f.y));
          const uint32_t ah0 = *reinterpret_cast<const uint32_t*>(&h0), al0 = *reinterpret_cast<const uint32_t*>(&l0);
          const uint32_t ah1 = *reinterpret_cast<const uint32_t*>(&h1), al1 = *reinterpret_cast<const uint32_t*>(&l1);
          if constexpr (TOK_M) {
            qA[kk / 2][kk % 2][0] = (gid & 1) ? al0 : ah0;
            qA[kk / 2][kk % 2][1] = (gid & 1) ? al1 : ah1;
          } else {
            qA[kk / 2][kk % 2][0] = ah0;
            qA[kk / 2][kk % 2][1] = al0;
            qA[kk / 2][kk % 2][2] = ah1;
            qA[kk / 2][kk % 2][3] = al1;
          }
        }
#pragma unroll
        for (int g = 0; g < NG; ++g) biasK[g] = 0.f;
      } else {
  #pragma unroll
        for (int g = 0; g < NG; ++g) {
          float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
          if (qh < G) {
            v0 = *reinterpret_cast<const float4*>(row + 32 * g + 8 * tig);
            v1 = *reinterpret_cast<const float4*>(row + 32 * g + 8 * tig + 4);
          }
          const float qv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
          // the code offset term -8 * sum(q) (the high-position pieces carry q / 16 against a
          // 16x nibble, so every element enters with weight 1); q itself stands for its hi + lo
          // pieces, which agree with it to 2^-22
          float bsum = ((qv[0] + qv[1]) + (qv[2] + qv[3])) + ((qv[4] + qv[5]) + (qv[6] + qv[7]));
  #pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const float2 lo = make_float2(qv[2 * ks], qv[2 * ks + 4]);
            const float2 hi = __fmul2_rn(make_float2(qv[2 * ks + 1], qv[2 * ks + 5]), make_float2(0.0625f, 0.0625f));
            const __half2 lo_h = __float22half2_rn(lo), hi_h = __float22half2_rn(hi);
            // residual pieces: x - fp16(x) is exact in binary32, then rounded to binary16
            const float2 lo_b = __half22float2(lo_h), hi_b = __half22float2(hi_h);
            const __half2 lo_l = __float22half2_rn(make_float2(lo.x - lo_b.x, lo.y - lo_b.y));
            const __half2 hi_l = __float22half2_rn(make_float2(hi.x - hi_b.x, hi.y - hi_b.y));
            const uint32_t ah = *reinterpret_cast<const uint32_t*>(&lo_h);
            const uint32_t al = *reinterpret_cast<const uint32_t*>(&lo_l);
            const uint32_t ch = *reinterpret_cast<const uint32_t*>(&hi_h);
            const uint32_t cl = *reinterpret_cast<const uint32_t*>(&hi_l);
            if constexpr (TOK_M) {
              qA[g][ks][0] = (gid & 1) ? al : ah;
              qA[g][ks][1] = (gid & 1) ? cl : ch;
            } else {
              qA[g][ks][0] = ah;
              qA[g][ks][1] = al;
              qA[g][ks][2] = ch;
              qA[g][ks][3] = cl;
            }
          }
          bsum += __shfl_xor_sync(0xffffffffu, bsum, 1);
          bsum += __shfl_xor_sync(0xffffffffu, bsum, 2);
          // TOK_M: the score lanes hold head tig, whose sum sits in lane 8 * tig (gid = 2 tig)
          if constexpr (TOK_M) bsum = __shfl_sync(0xffffffffu, bsum, (8 * tig) & 31);
          biasK[g] = -bsum * (8.0f * 5.9604644775390625e-08f);  // 8 * 2^-24
        }
      }
      const int sh_h = TOK_M ? tig : gid;  // the head of this lane's scores
      const int sh = (sh_h < G) ? reinterpret_cast<const int*>(scratch + 8 * C::QSTRIDE)[sh_h] : 0;
      // MMA units -> log2 units: 2^(24 - sh) for the subnormal-coded nibbles, 2^-sh for binary16 K
      f_h = __int_as_float((127 + (KF16 ? 0 : 24) - sh) << 23);
      __syncwarp();
#pragma unroll
      for (int g = 0; g < NG; ++g) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          acc[g][0][r] = 0.f;
          acc[g][1][r] = 0.f;
        }
      }
      m_run = -INFINITY;
      l_run = 0.f;
    }

    // ---------------- token tiles of this segment
    bool seg_end = false;
    while (!seg_end) {
      const int stage = tile_i % STAGES;
      const uint32_t par = (uint32_t)((tile_i / STAGES) & 1);
      // The converters arrive on `ready` only after they observed `full` complete, so
      // its completion (release by the converters, acquire here) also orders this
      // warp's reads after the stage's tensor copies.
      if (!dead && !mbar_wait_bounded(&ready[stage], par, p.wait_ns)) {
        dead = true;
        if (lane == 0) status_or(p.status, TQ_STATUS_TIMEOUT);
      }
      if (!dead) {
        const uint32_t sbase = smem_base + stage * C::STAGE_BYTES;
        const uint32_t kc = sbase + h * T_TILE * C::KRB;
        const uint32_t vc = sbase + C::OFF_VCODE + h * T_TILE * RB;
        const uint32_t sck = sbase + C::OFF_SC32 + 4 * h * C::SC_HEAD;
        const uint32_t scv = sbase + C::OFF_SCV + 4 * h * C::SC_HEAD;
        // tokens of the segment left in this tile, from this warp's first row on
        const int left = min(T_TILE, seg_hi - walk.t0) - sub * UPW * UNIT;
#pragma unroll 1
        for (int u = 0; u < UPW; ++u) {
          const int uu = sub * UPW + u;  // unit index within the tile
          const int r0 = uu * UNIT;      // first tile row of this unit
          if (u * UNIT >= left) break;
          const int nv = min(UNIT, left - u * UNIT);

          // P^T fragments for P.V, per 16-token k-step: tokens (2 tig, 2 tig + 1) and
          // (2 tig + 8, 2 tig + 9) of head gid
          float2 pb[KSP][2];
          bool pv_live = true;  // cleared by the sparse-V rule when no weight of the unit is kept
          (void)pv_live;
          if constexpr (TOK_M) {
            // --- scores S[token 16 mt + gid + 8 e][head tig], per group g. A = K codes (rows:
            //     tokens gid, gid + 8 of the m-tile), B = q pieces (columns 2j, 2j + 1: hi, lo
            //     of head j).
            constexpr int MT = UNIT / 16;
            float2 s2[MT];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) s2[mt] = make_float2(0.f, 0.f);
            if constexpr (KF16) {
              // A = binary16 K rows (tokens) straight from ldmatrix, B = q pieces; no scales
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 2 * NG; ++kk) {
                  uint32_t kw[4];
                  ldmatrix_x4(kw, kc + (r0 + 16 * mt) * C::KLINE + k16_off[kk]);
                  mma_f16_16816_acc(c, kw, qA[kk / 2][kk % 2][0], qA[kk / 2][kk % 2][1]);
                }
                s2[mt] = make_float2(c[0] + c[1], c[2] + c[3]);  // hi + lo columns
              }
            } else {

  #pragma unroll
              for (int g4 = 0; g4 < NG * NT; g4 += 4) {
                uint32_t kw[4];
                ldmatrix_x4(kw, kc + r0 * RB + k_off[g4 / 4]);
                float skm[4 / NT > 0 ? 4 / NT : 1][2 * MT];
  #pragma unroll
                for (int gi = 0; gi < (4 / NT > 0 ? 4 / NT : 1); ++gi) {
                  const int g = g4 / NT + gi;
                  const uint32_t a0 = sck + 4 * (((uu * NG + g) * 8 + gid) * (2 * MT));
                  if constexpr (MT == 2) {
                    const float4 v = lds_f4(a0);
                    skm[gi][0] = v.x;
                    skm[gi][1] = v.y;
                    skm[gi][2] = v.z;
                    skm[gi][3] = v.w;
                  } else {
                    const float2 v = lds_f2(a0);
                    skm[gi][0] = v.x;
                    skm[gi][1] = v.y;
                  }
                }
  #pragma unroll
                for (int i = 0; i < 4; i += 2) {
                  const int g = (g4 + i) / NT, mt = ((g4 + i) % NT) >> 1;
                  const int gi = g - g4 / NT;
                  const uint32_t wa = kw[i], wb = kw[i + 1];  // tokens gid and gid + 8 of m-tile mt
                  float c[4];
                  uint32_t a[4];
                  a[0] = and_xor(wa, 0x000F000Fu, 0x00080008u);
                  a[1] = and_xor(wb, 0x000F000Fu, 0x00080008u);
                  a[2] = and_xor(wa, 0x00F000F0u, 0x00800080u);
                  a[3] = and_xor(wb, 0x00F000F0u, 0x00800080u);
                  mma_f16_16816_c(c, a, qA[g][0][0], qA[g][0][1], 0.f, 0.f, 0.f, 0.f);
                  const uint32_t wa8 = wa >> 8, wb8 = wb >> 8;
                  a[0] = and_xor(wa8, 0x000F000Fu, 0x00080008u);
                  a[1] = and_xor(wb8, 0x000F000Fu, 0x00080008u);
                  a[2] = and_xor(wa8, 0x00F000F0u, 0x00800080u);
                  a[3] = and_xor(wb8, 0x00F000F0u, 0x00800080u);
                  mma_f16_16816_acc(c, a, qA[g][1][0], qA[g][1][1]);
                  // hi + lo columns, plus the offset term -8 * sum(q) of the offset-binary code
                  const float2 x = __fadd2_rn(make_float2(c[0] + c[1], c[2] + c[3]), make_float2(biasK[g], biasK[g]));
                  s2[mt] = __ffma2_rn(make_float2(skm[gi][2 * mt], skm[gi][2 * mt + 1]), x, s2[mt]);
                }
              }
            }
            if (nv < UNIT) {
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                if (16 * mt + gid >= nv) s2[mt].x = -INFINITY;
                if (16 * mt + gid + 8 >= nv) s2[mt].y = -INFINITY;
              }
            }
            // --- online softmax (head tig; lanes with the same tig share a head)
            float mx = fmaxf(s2[0].x, s2[0].y);
#pragma unroll
            for (int mt = 1; mt < MT; ++mt) mx = fmaxf(mx, fmaxf(s2[mt].x, s2[mt].y));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m_run, mx);
            const bool grow = m_new > m_run;
            if (__any_sync(0xffffffffu, grow)) {
              const float corr = grow ? ((m_run == -INFINITY) ? 0.f : ex2_approx((m_run - m_new) * f_h)) : 1.f;
              l_run *= corr;
              // accumulator columns are heads 2 tig, 2 tig + 1: lanes 2 tig, 2 tig + 1 hold them
              const float2 cc = make_float2(__shfl_sync(0xffffffffu, corr, 2 * tig),
                                            __shfl_sync(0xffffffffu, corr, 2 * tig + 1));
#pragma unroll
              for (int g = 0; g < NG; ++g) {
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                  float2 a01 = __fmul2_rn(make_float2(acc[g][jj][0], acc[g][jj][1]), cc);
                  float2 a23 = __fmul2_rn(make_float2(acc[g][jj][2], acc[g][jj][3]), cc);
                  acc[g][jj][0] = a01.x;
                  acc[g][jj][1] = a01.y;
                  acc[g][jj][2] = a23.x;
                  acc[g][jj][3] = a23.y;
                }
              }
              m_run = m_new;
            }
            const float mb = (m_run == -INFINITY) ? 0.f : m_run * f_h;
            float2 lsum = make_float2(0.f, 0.f);
            // p of token r of m-tile ks, head j, lives in lane 4 (r mod 8) + j, element r / 8
            const int src0 = 8 * tig + gid, src1 = src0 + 4;
            const bool head_ok = gid < G;  // G <= 4 here
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              const float2 z = __ffma2_rn(s2[mt], make_float2(f_h, f_h), make_float2(-mb, -mb));
              float2 pp = make_float2(ex2_approx(z.x), ex2_approx(z.y));
              lsum = __fadd2_rn(lsum, pp);
              if constexpr (sparse) {  // the V term only: the sum above keeps the token
                if (z.x < p.sparse_lt) pp.x = 0.f;
                if (z.y < p.sparse_lt) pp.y = 0.f;
              }
              const float x0 = __shfl_sync(0xffffffffu, pp.x, src0 & 31);
              const float x1 = __shfl_sync(0xffffffffu, pp.x, src1 & 31);
              const float y0 = __shfl_sync(0xffffffffu, pp.y, src0 & 31);
              const float y1 = __shfl_sync(0xffffffffu, pp.y, src1 & 31);
              pb[mt][0] = head_ok ? make_float2(x0, x1) : make_float2(0.f, 0.f);
              pb[mt][1] = head_ok ? make_float2(y0, y1) : make_float2(0.f, 0.f);
            }
            l_run += lsum.x + lsum.y;
            if constexpr (sparse) {
              bool nz = false;
#pragma unroll
              for (int mt = 0; mt < MT; ++mt)
                nz = nz || pb[mt][0].x != 0.f || pb[mt][0].y != 0.f || pb[mt][1].x != 0.f || pb[mt][1].y != 0.f;
              pv_live = __any_sync(0xffffffffu, nz);
            }
          } else {
            // --- scores S[head gid][token nt*8 + 2*tig + e], per group g
            float2 s2[NT], s2b[NT];  // even and odd groups: two independent chains
  #pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              s2[nt] = make_float2(0.f, 0.f);
              s2b[nt] = make_float2(0.f, 0.f);
            }
            if constexpr (KF16) {
              // B = binary16 K (8 tokens x 16 dims per n-tile and k-step) straight from
              // ldmatrix; one accumulator per n-tile over all k-steps; no scales
              static_assert(NT % 2 == 0, "binary16 K row layout: n-tile pairs");
              float c[NT][4];
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.f;
#pragma unroll
              for (int kk = 0; kk < 2 * NG; ++kk) {
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                  uint32_t kw[4];
                  ldmatrix_x4(kw, kc + (r0 + 16 * np) * C::KLINE + k16_off[kk]);
                  mma_f16_16816_acc(c[2 * np], qA[kk / 2][kk % 2], kw[0], kw[1]);
                  mma_f16_16816_acc(c[2 * np + 1], qA[kk / 2][kk % 2], kw[2], kw[3]);
                }
              }
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)  // hi + lo rows
                s2[nt] = __fadd2_rn(make_float2(c[nt][0], c[nt][1]), make_float2(c[nt][2], c[nt][3]));
            } else {
    #pragma unroll
              for (int g4 = 0; g4 < NG * NT; g4 += 4) {
                uint32_t kw[4];
                ldmatrix_x4(kw, kc + r0 * RB + k_off[g4 / 4]);
                // this lane's K scales for the groups of this batch: (n-tile, e) pairs
                float skv[4 / NT > 0 ? 4 / NT : 1][2 * NT];
    #pragma unroll
                for (int gi = 0; gi < (4 / NT > 0 ? 4 / NT : 1); ++gi) {
                  const int g = g4 / NT + gi;
                  const uint32_t a0 = sck + 4 * (((uu * NG + g) * 4 + tig) * (2 * NT));
    #pragma unroll
                  for (int q4 = 0; q4 < 2 * NT; q4 += 4) {
                    const float4 v = lds_f4(a0 + 4 * q4);
                    skv[gi][q4] = v.x;
                    skv[gi][q4 + 1] = v.y;
                    skv[gi][q4 + 2] = v.z;
                    skv[gi][q4 + 3] = v.w;
                  }
                }
    #pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int g = (g4 + i) / NT, nt = (g4 + i) % NT;
                  const int gi = g - g4 / NT;
                  const float2 sk = make_float2(skv[gi][2 * nt], skv[gi][2 * nt + 1]);
                  float c[4];
                  const uint32_t w = kw[i];
                  mma_f16_16816_c(c, qA[g][0], and_xor(w, 0x000F000Fu, 0x00080008u),
                                  and_xor(w, 0x00F000F0u, 0x00800080u), 0.f, 0.f, 0.f, 0.f);
                  const uint32_t w8 = w >> 8;
                  mma_f16_16816_acc(c, qA[g][1], and_xor(w8, 0x000F000Fu, 0x00080008u),
                                    and_xor(w8, 0x00F000F0u, 0x00800080u));
                  // hi + lo rows, plus the offset term -8 * sum(q) of the offset-binary code
                  const float2 x = __fadd2_rn(__fadd2_rn(make_float2(c[0], c[1]), make_float2(c[2], c[3])),
                                              make_float2(biasK[g], biasK[g]));
                  if (g & 1)
                    s2b[nt] = __ffma2_rn(sk, x, s2b[nt]);
                  else
                    s2[nt] = __ffma2_rn(sk, x, s2[nt]);
                }
              }
            }
  #pragma unroll
            for (int nt = 0; nt < NT; ++nt) s2[nt] = __fadd2_rn(s2[nt], s2b[nt]);
            if (nv < UNIT) {
  #pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                if (nt * 8 + 2 * tig >= nv) s2[nt].x = -INFINITY;
                if (nt * 8 + 2 * tig + 1 >= nv) s2[nt].y = -INFINITY;
              }
            }

            // --- online softmax (head gid; the quad's lanes share a head)
            float mx = fmaxf(s2[0].x, s2[0].y);
  #pragma unroll
            for (int nt = 1; nt < NT; ++nt) mx = fmaxf(mx, fmaxf(s2[nt].x, s2[nt].y));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run, mx);
            const bool grow = m_new > m_run;
            if (__any_sync(0xffffffffu, grow)) {
              const float corr = grow ? ((m_run == -INFINITY) ? 0.f : ex2_approx((m_run - m_new) * f_h)) : 1.f;
              l_run *= corr;
              const float2 cc = make_float2(__shfl_sync(0xffffffffu, corr, 8 * tig),
                                            __shfl_sync(0xffffffffu, corr, 8 * tig + 4));
  #pragma unroll
              for (int g = 0; g < NG; ++g) {
  #pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                  float2 a01 = __fmul2_rn(make_float2(acc[g][jj][0], acc[g][jj][1]), cc);
                  float2 a23 = __fmul2_rn(make_float2(acc[g][jj][2], acc[g][jj][3]), cc);
                  acc[g][jj][0] = a01.x;
                  acc[g][jj][1] = a01.y;
                  acc[g][jj][2] = a23.x;
                  acc[g][jj][3] = a23.y;
                }
              }
              m_run = m_new;
            }
            const float mb = (m_run == -INFINITY) ? 0.f : m_run * f_h;
            float2 p2[NT];
            float2 lsum = make_float2(0.f, 0.f);
  #pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const float2 z = __ffma2_rn(s2[nt], make_float2(f_h, f_h), make_float2(-mb, -mb));
              p2[nt] = make_float2(ex2_approx(z.x), ex2_approx(z.y));
              lsum = __fadd2_rn(lsum, p2[nt]);
              if constexpr (sparse) {  // the V term only: the sum above keeps the token
                if (z.x < p.sparse_lt) p2[nt].x = 0.f;
                if (z.y < p.sparse_lt) p2[nt].y = 0.f;
              }
            }
            l_run += lsum.x + lsum.y;
            if constexpr (sparse) {
              bool nz = false;
  #pragma unroll
              for (int nt = 0; nt < NT; ++nt) nz = nz || p2[nt].x != 0.f || p2[nt].y != 0.f;
              pv_live = __any_sync(0xffffffffu, nz);
            }
  #pragma unroll
            for (int ks = 0; ks < KSP; ++ks) {
              pb[ks][0] = p2[2 * ks];
              pb[ks][1] = p2[2 * ks + 1];
            }

          }

          // --- P.V: acc[d][head] += sum_t (c_t,d * 2^-24) * (p_t * sigmaV_t,g). The signed code
          //     enters exactly: u = code + 8 from the lop3, then one binary16 subtract per pair
          //     (8 * 2^-24 at the low nibble position, 128 * 2^-24 = 16 * 8 * 2^-24 at the high
          //     one, whose rows therefore carry x16). A biased offset must not reach the
          //     accumulator: the tensor core rounds its fp32 sums toward zero, so an all-positive
          //     operand would drift over a long context.
          const __half2 k8 = __ushort_as_half2_pair(0x0008u);
          const __half2 k128 = __ushort_as_half2_pair(0x0080u);
#pragma unroll
          for (int g4 = 0; g4 < NG * NT; g4 += 4) {
            if constexpr (sparse) {
              if (!pv_live) break;  // sparse-V: every weight of this unit fell below the threshold
            }
            uint32_t vw[4];
            ldmatrix_x4_trans(vw, vc + r0 * RB + v_off[g4 / 4]);
#pragma unroll
            for (int i = 0; i < 4; i += 2) {
              const int g = (g4 + i) / NT, tb = (g4 + i) % NT;  // token blocks tb, tb + 1 = one k-step
              const int ks = tb >> 1;
              const float4 sv = lds_f4(scv + 4 * (((uu * NG + g) * 4 + tig) * (2 * NT) + ks * 4));
              const uint32_t b0 = pack_half2_f2(__fmul2_rn(pb[ks][0], make_float2(sv.x, sv.y)));
              const uint32_t b1 = pack_half2_f2(__fmul2_rn(pb[ks][1], make_float2(sv.z, sv.w)));
              const uint32_t va = vw[i], vb = vw[i + 1];
#pragma unroll
              for (int jj = 0; jj < 2; ++jj) {
                const uint32_t xa = jj ? (va >> 8) : va, xb = jj ? (vb >> 8) : vb;
                uint32_t a[4];
                a[0] = h2_sub_u32(and_xor(xa, 0x000F000Fu, 0x00080008u), k8);
                a[1] = h2_sub_u32(and_xor(xa, 0x00F000F0u, 0x00800080u), k128);
                a[2] = h2_sub_u32(and_xor(xb, 0x000F000Fu, 0x00080008u), k8);
                a[3] = h2_sub_u32(and_xor(xb, 0x00F000F0u, 0x00800080u), k128);
                mma_f16_16816_acc(acc[g][jj], a, b0, b1);
              }
            }
          }
          (void)KSP;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      ++tile_i;
      seg_end = walk.advance<T_TILE>();
    }

    // ---------------- segment end: write this (sequence, CTA) partial
    const int slot = b + (int)blockIdx.x;
    float l_tot = l_run;
    if constexpr (TOK_M) {  // head tig: sum over gid
      l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 4);
      l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 8);
      l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 16);
    } else {  // head gid: sum over tig
      l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 1);
      l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 2);
    }
    // the lane that reports (m, l) of head hm
    const int hm = TOK_M ? tig : gid;
    const bool reports = TOK_M ? (gid == 0 && tig < 4) : (tig == 0);
    const float m_real = (m_run == -INFINITY) ? -INFINITY : m_run * f_h;
    constexpr float kTwo24 = 16777216.f;
    // rotated-domain accumulator of head 2*tig + e at d = 32g + 4*gid + {0, 1, 2, 3};
    // rows of the high nibble position carry x16.
    auto final4 = [&](int g, int e) {
      return make_float4(acc[g][0][e] * kTwo24, acc[g][0][2 + e] * (0.0625f * kTwo24), acc[g][1][e] * kTwo24,
                         acc[g][1][2 + e] * (0.0625f * kTwo24));
    };
    if constexpr (C::WPH == 1) {
      if (!dead) {
        if (reports && hm < G) {
          float* ml = p.ws_ml + (((int64_t)slot * p.n_q + h * G + hm) * 2) + 2 * (p.batch + 2);
          ml[0] = m_real;
          ml[1] = l_tot;
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int hh = 2 * tig + e;
          if (hh < G) {
            float* dst = p.ws_acc + ((int64_t)slot * p.n_q + h * G + hh) * D;
#pragma unroll
            for (int g = 0; g < NG; ++g) *reinterpret_cast<float4*>(dst + 32 * g + 4 * gid) = final4(g, e);
          }
        }
      }
    } else {
      // several warps share a KV head: combine their states through shared memory
      float* mls = scratch + 8 * D;  // [8][2]
      if (reports) {
        mls[2 * hm] = dead ? -INFINITY : m_real;
        mls[2 * hm + 1] = dead ? 0.f : l_tot;
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int hh = 2 * tig + e;
#pragma unroll
        for (int g = 0; g < NG; ++g)
          *reinterpret_cast<float4*>(scratch + hh * D + 32 * g + 4 * gid) =
              dead ? make_float4(0.f, 0.f, 0.f, 0.f) : final4(g, e);
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
      // one thread per (kv head, q head): the weights 2^(m_w - m*) of the WPH partials
      // replace their m words, and (m*, sum of weighted l) goes out
      for (int pr = tid; pr < HKV * G; pr += kConsumerWarps * 32) {
        const int hk = pr / G, j = pr % G;
        float mstar = -INFINITY;
        for (int sb = 0; sb < C::WPH; ++sb) {
          const float* sm = reinterpret_cast<const float*>(smem + C::OFF_SCRATCH + (hk + sb * HKV) * C::SCRATCH);
          mstar = fmaxf(mstar, sm[8 * D + 2 * j]);
        }
        float lsum = 0.f;
        for (int sb = 0; sb < C::WPH; ++sb) {
          float* sm = reinterpret_cast<float*>(smem + C::OFF_SCRATCH + (hk + sb * HKV) * C::SCRATCH);
          const float mw = sm[8 * D + 2 * j];
          const float wgt = (mw == -INFINITY) ? 0.f : exp2f(mw - mstar);
          lsum += wgt * sm[8 * D + 2 * j + 1];
          sm[8 * D + 2 * j] = wgt;
        }
        float* ml = p.ws_ml + ((int64_t)slot * p.n_q + hk * G + j) * 2 + 2 * (p.batch + 2);
        ml[0] = mstar;
        ml[1] = lsum;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
      const int items = HKV * G * D;
      for (int it = tid; it < items; it += kConsumerWarps * 32) {
        const int hk = it / (G * D), j = (it / D) % G, d = it % D;
        float asum = 0.f;
#pragma unroll
        for (int sb = 0; sb < C::WPH; ++sb) {
          const float* sm = reinterpret_cast<const float*>(smem + C::OFF_SCRATCH + (hk + sb * HKV) * C::SCRATCH);
          asum = fmaf(sm[8 * D + 2 * j], sm[j * D + d], asum);
        }
        p.ws_acc[((int64_t)slot * p.n_q + hk * G + j) * D + d] = asum;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
    }
  }
}

// Combine the partials of one (sequence, q head), normalise, inverse SRHT.
// Launched as a programmatic dependent of the split-K kernel: blocks may start
// early and wait at griddepcontrol.wait until every split-K block has finished
// and its writes are visible; before the wait they prefetch the lines of their
// partials into L2 (the address translations are then warm). Phase 1 stages
// the weights 2^(m_c - m*) of all partials in shared memory; phase 2 streams
// the accumulators with PF independent loads in flight per thread; one warp
// then sums the slot phases and runs the inverse transform with shuffles.
// NTH = 128 threads (8 blocks per SM) when there are many (sequence, head)
// pairs, 512 when there are fewer than twice the SMs: a long sequence then has
// up to one partial per SM, and its loads (10 per thread, 160 partials at
// head_dim 128) should all be in flight at once.
// Kernel 1b (decode_tail_kernel, delegated cache only): attention partials over
// the hot tail (mlxcel guide, delegated cache variant: the recent tokens keep
// binary16 K and V). One block per (sequence, kv head, chunk of kTailTokens hot
// tokens) computes the partial (running max in log2 units, sum, accumulator) of
// every q head of the group, so each binary16 K and V row is read once per kv
// head: the chunk's K and V rows are staged in shared memory by cp.async (all
// copies in flight together, 16-byte pieces XOR-swizzled by row so that
// ldmatrix is conflict-free), then each of the 4 warps takes 16 tokens on the
// tensor cores (mma.m16n8k16, f16 in, f32 accumulate), as in the split-K kernel:
//   Q.K^T  A rows 0-7 = the binary16 hi piece of q head 0-7 (scaled by 2^sh so
//          that its largest element is below 2^14), rows 8-15 = the lo piece;
//          B = K rows (exact); the score is the sum of the two rows times 2^-sh;
//   P.V    A rows 0-7 = binary16 of the weights p = 2^(s - m), rows 8-15 = the
//          binary16 of their residual; B = V rows through a transposing ldmatrix.
// The warps' partials share the block's running max and are summed in shared
// memory. The accumulator is mapped into the rotated domain by the forward SRHT
// (c_D H (s o x); the transform is linear), so the merge kernel combines it like
// any split-K partial and its single inverse SRHT brings the output back.
// Chunks past a sequence's hot tokens write empty partials (m = -inf, l = 0).
// The inputs were complete before the split-K grid started, so the work runs
// before the dependency wait; the wait comes last, so that this grid completes
// only after the split-K grid, and the merge kernel's wait covers both.
constexpr int kTailTokens = 64;  // tail_chunk_count() in tq_kernels.h uses the same 64
constexpr int kTailThreads = 128;
constexpr int kMaxTailChunks = 16;  // tail windows up to 1024 tokens

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// 16-byte piece c of row j of a [rows][D] binary16 tile, XOR-swizzled so that 8
// consecutive rows at one piece index fall in 8 different bank groups.
template <int D>
__device__ __forceinline__ int tile_piece(int j, int c) {
  return (D >= 64) ? (c ^ (j & 7)) : (c ^ ((j >> 1) & 3));
}

template <int D>
__global__ void __launch_bounds__(kTailThreads) decode_tail_kernel(const __grid_constant__ DecodeParams p) {
  static_assert(D <= 128, "binary16 K rows up to head_dim 128");
  constexpr int CPR = D / 8;  // 16-byte pieces per row
  constexpr int KS = D / 16;  // k-steps of the scores
  constexpr int NT = D / 8;   // n-tiles (8 dims) of P.V
  constexpr int NW = kTailThreads / 32;
  constexpr int PP = D + 8;   // padded row of the warp partials (floats)
  __shared__ __align__(128) uint16_t tiles[2 * kTailTokens * D];  // K rows, then V rows
  __shared__ float mred[NW][8];
  __shared__ float lred[NW][8];
  uint16_t* ks = tiles;
  uint16_t* vsm = tiles + kTailTokens * D;
  float* part = reinterpret_cast<float*>(tiles);  // [NW][8][PP] after P.V
  static_assert(NW * 8 * PP * 4 <= (int)sizeof(tiles), "warp partials fit in the K and V tiles");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int nch = p.tail_chunks;
  const int chunk = blockIdx.x % nch;
  const int bh = blockIdx.x / nch;
  const int kvh = bh % p.n_kv, b = bh / p.n_kv;
  const int G = p.group, W = p.tail_window;
  int len = p.seq_lens[b];
  if (len < 0 || len > p.max_seq) len = 0;
  const int t_lo = (int)cold_tokens(len, W, p.fold_chunk) + chunk * kTailTokens;
  const int n = max(0, min(len, t_lo + kTailTokens) - t_lo);
  const int64_t slot = (int64_t)p.tail_slot0 + (int64_t)b * nch + chunk;
  float* ml = p.ws_ml + 2 * (p.batch + 2) + (slot * p.n_q + (int64_t)kvh * G) * 2;
  float* acc_out = p.ws_acc + (slot * p.n_q + (int64_t)kvh * G) * D;
  if (n == 0) {
    for (int i = tid; i < G; i += kTailThreads) {
      ml[2 * i] = -INFINITY;
      ml[2 * i + 1] = 0.f;
    }
    for (int i = tid; i < G * D; i += kTailThreads) acc_out[i] = 0.f;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  // stage the chunk's K rows and V tail rows; V rows past n are zeroed (their
  // weights are 0, but 0 * NaN would not be)
  {
    const int64_t rstride = (int64_t)p.n_kv * D;  // binary16 elements between tokens (K) or slots (V)
    const uint16_t* kg = p.k16 + (((int64_t)b * p.max_seq + t_lo) * p.n_kv + kvh) * D;
    const uint16_t* vg = p.v_tail + ((int64_t)b * W * p.n_kv + kvh) * D;
    // a thread copies piece c of rows j0, j0 + RSTEP, ...; RSTEP is a multiple of 8
    // (of 32 at D = 32), so the swizzled piece is the same in every row it copies
    const int c = tid % CPR;
    constexpr int RSTEP = kTailThreads / CPR;
    static_assert(RSTEP % 8 == 0, "one swizzle phase per thread");
    const int j0 = tid / CPR;
    const int pc = tile_piece<D>(j0, c);
    uint32_t ks_dst = smem_u32(&ks[j0 * D + pc * 8]);
    uint32_t vs_dst = smem_u32(&vsm[j0 * D + pc * 8]);
    const uint16_t* ksrc = kg + (int64_t)j0 * rstride + c * 8;
    const uint16_t* vcol = vg + c * 8;
    int slot_v = (t_lo + j0) % W;
    for (int j = j0; j < kTailTokens; j += RSTEP) {
      if (j < n) {
        cp_async16(ks_dst, ksrc);
        cp_async16(vs_dst, vcol + (int64_t)slot_v * rstride);
      } else {
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vs_dst), "r"(0u) : "memory");
      }
      ks_dst += RSTEP * D * 2;
      vs_dst += RSTEP * D * 2;
      ksrc += RSTEP * rstride;
      slot_v += RSTEP;
      while (slot_v >= W) slot_v -= W;
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  // A fragments of the scores: head gid's hi (rows 0-7) and lo (rows 8-15) pieces,
  // dims 16 kk + 2 tig + {0, 1} (a0, a1) and 16 kk + 8 + 2 tig + {0, 1} (a2, a3)
  uint32_t qa[KS][4];
  float f_h = 1.f;
  {
    float x[KS][4];
    const int64_t qoff = ((int64_t)b * p.n_q + (int64_t)kvh * G + (gid < G ? gid : 0)) * D + 2 * tig;
    // pairs (d, d + 1), d = 16 kk + 2 tig (+ 8): one 8- or 4-byte load each
    if (p.q_dtype == TQ_F32) {
      const float* qp = reinterpret_cast<const float*>(p.q) + qoff;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 v = *reinterpret_cast<const float2*>(qp + 16 * kk + 8 * h);
          x[kk][2 * h] = v.x;
          x[kk][2 * h + 1] = v.y;
        }
    } else {
      const uint16_t* qp = reinterpret_cast<const uint16_t*>(p.q) + qoff;
      const bool bf = p.q_dtype == TQ_BF16;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t w = *reinterpret_cast<const uint32_t*>(qp + 16 * kk + 8 * h);
          if (bf) {
            x[kk][2 * h] = __uint_as_float(w << 16);
            x[kk][2 * h + 1] = __uint_as_float(w & 0xffff0000u);
          } else {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
            x[kk][2 * h] = f.x;
            x[kk][2 * h + 1] = f.y;
          }
        }
    }
    float mx = 0.f;
    const float qsc = gid < G ? p.sm_scale_log2 : 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[kk][e] *= qsc;
        mx = fmaxf(mx, fabsf(x[kk][e]));
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    int ex = 0;
    if (mx > 0.f) (void)frexpf(mx, &ex);
    const int sh = min(100, max(-100, 14 - ex));  // scaled max < 2^14
    const float sc = __int_as_float((127 + sh) << 23);
    f_h = __int_as_float((127 - sh) << 23);
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 v = make_float2(x[kk][2 * h] * sc, x[kk][2 * h + 1] * sc);
        const __half2 hi = __float22half2_rn(v);
        const float2 hf = __half22float2(hi);
        const __half2 lo = __float22half2_rn(make_float2(v.x - hf.x, v.y - hf.y));
        qa[kk][2 * h] = *reinterpret_cast<const uint32_t*>(&hi);
        qa[kk][2 * h + 1] = *reinterpret_cast<const uint32_t*>(&lo);
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  // scores of this warp's 16 tokens: two n-tiles of 8
  const int tok0 = wp * 16;
  float c[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) c[nt][e] = 0.f;
  {
    const int mi = lane >> 3, r = lane & 7;
    const int row = tok0 + 8 * (mi >> 1) + r;  // matrices: (n-tile 0, piece 2kk), (0, 2kk+1), (1, 2kk), (1, 2kk+1)
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t bf[4];
      ldmatrix_x4(bf, smem_u32(&ks[row * D + tile_piece<D>(row, 2 * kk + (mi & 1)) * 8]));
      mma_f16_16816_acc(c[0], qa[kk], bf[0], bf[1]);
      mma_f16_16816_acc(c[1], qa[kk], bf[2], bf[3]);
    }
  }
  // s for head gid at tokens tok0 + 8 nt + 2 tig + e; masked past n
  float sv[2][2];
  float mloc = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = tok0 + 8 * nt + 2 * tig + e;
      const float v = (c[nt][e] + c[nt][2 + e]) * f_h;
      sv[nt][e] = t < n ? v : -INFINITY;
      mloc = fmaxf(mloc, sv[nt][e]);
    }
  mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
  mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
  if (tig == 0) mred[wp][gid] = mloc;
  __syncthreads();
  float m = mred[0][gid];
#pragma unroll
  for (int w = 1; w < NW; ++w) m = fmaxf(m, mred[w][gid]);
  // weights, their sum, and the A fragments (hi rows 0-7, residual rows 8-15)
  float lsum = 0.f;
  uint32_t pa[4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const float p0 = (sv[nt][0] == -INFINITY) ? 0.f : exp2f(sv[nt][0] - m);
    const float p1 = (sv[nt][1] == -INFINITY) ? 0.f : exp2f(sv[nt][1] - m);
    lsum += p0 + p1;
    const __half2 hi = __float22half2_rn(make_float2(p0, p1));
    const float2 hf = __half22float2(hi);
    const __half2 lo = __float22half2_rn(make_float2(p0 - hf.x, p1 - hf.y));
    pa[2 * nt] = *reinterpret_cast<const uint32_t*>(&hi);
    pa[2 * nt + 1] = *reinterpret_cast<const uint32_t*>(&lo);
  }
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
  lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
  if (tig == 0) lred[wp][gid] = lsum;
  // P.V over this warp's 16 tokens: B = V rows (k = tokens, n = dims) via ldmatrix.trans
  float o[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
  {
    const int mi = lane >> 3, r = lane & 7;
    const int row = tok0 + 8 * (mi & 1) + r;  // matrices: (tokens 0-7, piece dn), (8-15, dn), (0-7, dn+1), (8-15, dn+1)
#pragma unroll
    for (int dn = 0; dn < NT; dn += 2) {
      uint32_t bf[4];
      ldmatrix_x4_trans(bf, smem_u32(&vsm[row * D + tile_piece<D>(row, dn + (mi >> 1)) * 8]));
      mma_f16_16816_acc(o[dn], pa, bf[0], bf[1]);
      mma_f16_16816_acc(o[dn + 1], pa, bf[2], bf[3]);
    }
  }
  __syncthreads();  // every warp is done with the K and V tiles: part[] may overwrite them
  // head gid, dims 8 dn + 2 tig + {0, 1}: hi row plus residual row
#pragma unroll
  for (int dn = 0; dn < NT; ++dn)
    *reinterpret_cast<float2*>(part + (wp * 8 + gid) * PP + 8 * dn + 2 * tig) =
        make_float2(o[dn][0] + o[dn][2], o[dn][1] + o[dn][3]);
  __syncthreads();
  // sum the warps and apply the signs (in place in warp 0's rows)
  for (int i = tid; i < G * D; i += kTailThreads) {
    const int g = i / D, d = i % D;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) sum += part[(w * 8 + g) * PP + d];
    part[g * PP + d] = apply_sign(sum, p.sign_bits, d);
  }
  if (tid < G) {
    float mt = mred[0][tid], l = 0.f;
#pragma unroll
    for (int w = 1; w < NW; ++w) mt = fmaxf(mt, mred[w][tid]);
#pragma unroll
    for (int w = 0; w < NW; ++w) l += lred[w][tid];
    ml[2 * tid] = mt;
    ml[2 * tid + 1] = l;
  }
  __syncthreads();
  // forward SRHT, one warp per q head
  constexpr int EPL = D / 32;  // elements per lane, consecutive
  for (int g = wp; g < G; g += NW) {
    float u[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) u[i] = part[g * PP + lane * EPL + i];
    // butterflies of stride < EPL inside the lane, then across lanes
#pragma unroll
    for (int h = 1; h < EPL; h <<= 1) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        if ((i & h) == 0) {
          const float a = u[i], bb = u[i + h];
          u[i] = a + bb;
          u[i + h] = a - bb;
        }
      }
    }
#pragma unroll
    for (int lm = 1; lm < 32; lm <<= 1) {
      const bool upper = (lane & lm) != 0;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, u[i], lm);
        u[i] = upper ? other - u[i] : u[i] + other;
      }
    }
    float* dst = acc_out + (int64_t)g * D + lane * EPL;
#pragma unroll
    for (int i = 0; i < EPL; ++i) dst[i] = u[i] * p.c_d;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int D>
static cudaError_t launch_tail(const DecodeParams& p, cudaStream_t s, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.batch * p.n_kv * p.tail_chunks));
  cfg.blockDim = dim3(kTailThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, decode_tail_kernel<D>, p);
}

template <int D, int NTH>
__global__ void __launch_bounds__(NTH, NTH >= 512 ? 1 : 1024 / NTH)
    decode_merge_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int F4 = D / 4;            // float4 columns
  constexpr int PH = NTH / F4;         // slot phases
  constexpr int PF = NTH >= 512 ? 10 : 8;  // loads in flight per thread
  constexpr int E = D / 32;            // elements per lane in the closing transform
  constexpr int MAX_SLOTS = 1024;      // a sequence meets at most one partial per split-K CTA
  static_assert(PH >= 1 && PH * F4 == NTH, "whole float4 rows per slot phase");
  __shared__ float wts[MAX_SLOTS + kMaxTailChunks];
  __shared__ float lsv[MAX_SLOTS + kMaxTailChunks];
  __shared__ float red[NTH / 32];
  __shared__ __align__(16) float accs[PH][D];
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int b = blockIdx.x / p.n_q, hq = blockIdx.x % p.n_q;
  // The range of this sequence's partials follows from the lengths alone, with the
  // split-K kernel's rules (lengths outside [0, max_seq] count as 0). The lengths are
  // read before the dependency wait: this grid is launched only once every split-K
  // block has passed its own wait, so whatever wrote them has completed.
  // With a hot tail (delegated cache) the split-K kernel covered only each sequence's
  // cold tokens, and so do these ranges.
  __shared__ long long red64[2][NTH / 32];
  long long before = 0, total = 0;
  for (int i = tid; i < p.batch; i += NTH) {
    int x = p.seq_lens[i];
    if (x < 0 || x > p.max_seq) x = 0;
    long long c = cold_tokens(x, p.tail_window, p.fold_chunk);
    c = (c + p.len_align - 1) & ~(long long)(p.len_align - 1);  // the split-K kernel's padded lengths
    total += c;
    if (i < b) before += c;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    total += __shfl_xor_sync(0xffffffffu, total, o);
  }
  if (lane == 0) {
    red64[0][wp] = before;
    red64[1][wp] = total;
  }
  __syncthreads();
  before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < NTH / 32; ++w) {
    before += red64[0][w];
    total += red64[1][w];
  }
  int len_all = p.seq_lens[b];
  if (len_all < 0 || len_all > p.max_seq) len_all = 0;
  const int64_t len_b = cold_tokens(len_all, p.tail_window, p.fold_chunk);
  int64_t R = (total + p.grid - 1) / p.grid;
  if (R < p.min_split) R = p.min_split;
  const int64_t r_align = p.len_align > 16 ? p.len_align : 16;
  R = (R + r_align - 1) & ~(r_align - 1);
  // the last partial is that of the CTA holding the last TRUE token (padding is never read)
  const int64_t P0 = before, P1 = before + len_b;
  // Delegated cache: the hot tail's partials (one per chunk of hot tokens, in the
  // rotated domain like the rest) follow in slots tail_slot0 + b * tail_chunks + k.
  const int n_tail = (p.tail_window > 0 && len_all > 0) ? p.tail_chunks : 0;
  const bool empty = P1 <= P0 && n_tail == 0;
  const float* ml = p.ws_ml + 2 * (p.batch + 2);
  float* out = p.out + ((int64_t)b * p.n_q + hq) * D;
  const int c0 = P1 > P0 ? (int)(P0 / R) : 0, c1 = P1 > P0 ? (int)((P1 - 1) / R) : -1;
  const int ns_cold = min(c1 - c0 + 1, MAX_SLOTS);
  const int ns = ns_cold + n_tail;
  const int64_t tail_first = (int64_t)p.tail_slot0 + (int64_t)b * p.tail_chunks;
  const float* mlb = ml + ((int64_t)(b + c0) * p.n_q + hq) * 2;
  const float* mlt = ml + (tail_first * p.n_q + hq) * 2;
  const int64_t mls = (int64_t)p.n_q * 2;
  const int col = tid % F4, ph = tid / F4;
  const float4* base = reinterpret_cast<const float4*>(p.ws_acc) + ((int64_t)(b + c0) * p.n_q + hq) * F4 + col;
  const float4* tbase = reinterpret_cast<const float4*>(p.ws_acc) + (tail_first * p.n_q + hq) * F4 + col;
  const int64_t stride = (int64_t)p.n_q * F4;
  auto acc_at = [&](int i) {  // partial i: the cold run first, then the tail run
    return i < ns_cold ? base + (int64_t)i * stride : tbase + (int64_t)(i - ns_cold) * stride;
  };
  auto ml_at = [&](int i) {
    return reinterpret_cast<const float2*>(i < ns_cold ? mlb + i * mls : mlt + (i - ns_cold) * mls);
  };
  // While the split-K grid runs, warm the address translation and L2 lines of the
  // partials this thread reads first. Prefetches only: the values are loaded after
  // the wait, from L2, where the split-K blocks' stores land.
  if (!empty) {
    for (int i = tid; i < ns; i += NTH) prefetch_l2(ml_at(i));
    if ((col & 7) == 0) {  // one 128-byte line per 8 float4 columns
#pragma unroll
      for (int k = 0; k < PF; ++k) {
        const int i = ph + k * PH;
        if (i < ns) prefetch_l2(acc_at(i));
      }
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (empty) {  // empty sequence
    for (int d = tid; d < D; d += NTH) out[d] = 0.f;
    return;
  }
  // phase 1: (m, l) of every partial in one pass -> m*, weights, sum of weighted l.
  // The (m, l) loads go first; the accumulator loads of the first chunk, which do not
  // depend on the weights, follow at once and stream in behind them, so the merge
  // costs about one memory round trip.
  float m = -INFINITY;
  float2 e0 = make_float2(-INFINITY, 0.f);
  if (tid < ns) e0 = __ldcg(ml_at(tid));
  float4 v[PF];
#pragma unroll
  for (int k = 0; k < PF; ++k) {
    const int i = ph + k * PH;
    v[k] = i < ns ? __ldcg(acc_at(i)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (tid < ns) {
    wts[tid] = e0.x;
    lsv[tid] = e0.y;
    m = e0.x;
  }
  for (int i = tid + NTH; i < ns; i += NTH) {
    const float2 e = __ldcg(ml_at(i));
    wts[i] = e.x;
    lsv[i] = e.y;
    m = fmaxf(m, e.x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[wp] = m;
  __syncthreads();
  float mstar = red[0];
#pragma unroll
  for (int w = 1; w < NTH / 32; ++w) mstar = fmaxf(mstar, red[w]);
  float lsum = 0.f;
  for (int i = tid; i < ns; i += NTH) {
    const float mi = wts[i];
    const float w = (mi == -INFINITY) ? 0.f : exp2f(mi - mstar);
    wts[i] = w;
    lsum += w * lsv[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  __syncthreads();  // red[] reused, wts[] complete
  if (lane == 0) red[wp] = lsum;
  // phase 2: weighted accumulator sums, PH slot phases x F4 float4 columns
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i0 = ph;; i0 += PH * PF) {
#pragma unroll
    for (int k = 0; k < PF; ++k) {
      const int i = i0 + k * PH;
      const float w = i < ns ? wts[i] : 0.f;
      a.x = fmaf(w, v[k].x, a.x);
      a.y = fmaf(w, v[k].y, a.y);
      a.z = fmaf(w, v[k].z, a.z);
      a.w = fmaf(w, v[k].w, a.w);
    }
    if (i0 + PH * PF >= ns) break;
#pragma unroll
    for (int k = 0; k < PF; ++k) {
      const int i = i0 + PH * PF + k * PH;
      v[k] = i < ns ? __ldcg(acc_at(i)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  reinterpret_cast<float4*>(accs[ph])[col] = a;
  __syncthreads();  // accs[] and the l sums of every warp are complete
  if (wp != 0) return;
  // One warp closes: lane l sums the slot phases of elements l E .. l E + E - 1,
  // normalises, and runs the inverse SRHT (butterflies of stride below E in
  // registers, the wider ones between lanes, in the forward transform's stage
  // order; each stage forms u_i + u_{i+h} and u_i - u_{i+h} with one rounding).
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < NTH / 32; ++w) L += red[w];
  const float inv_l = (L > 0.f) ? 1.f / L : 0.f;
  float u[E];
#pragma unroll
  for (int j = 0; j < E; ++j) u[j] = 0.f;
#pragma unroll
  for (int q = 0; q < PH; ++q) {
#pragma unroll
    for (int j = 0; j < E; ++j) u[j] += accs[q][lane * E + j];
  }
#pragma unroll
  for (int j = 0; j < E; ++j) {
    float o = u[j] * inv_l;
    if (p.lambda_v != nullptr) o = __fdividef(o, __ldg(p.lambda_v + lane * E + j));  // the V codes hold lambda o y
    u[j] = o;
  }
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int j = 0; j < E; ++j) {
      if ((j & h) == 0) {
        const float x = u[j], y = u[j + h];
        u[j] = __fadd_rn(x, y);
        u[j + h] = __fsub_rn(x, y);
      }
    }
  }
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int j = 0; j < E; ++j) {
      const float o = __shfl_xor_sync(0xffffffffu, u[j], h);
      u[j] = (lane & h) ? __fsub_rn(o, u[j]) : __fadd_rn(u[j], o);
    }
  }
#pragma unroll
  for (int j = 0; j < E; ++j) u[j] = apply_sign(u[j] * p.c_d, p.sign_bits, lane * E + j);
  if constexpr (E % 4 == 0) {
#pragma unroll
    for (int j = 0; j < E; j += 4)
      *reinterpret_cast<float4*>(out + lane * E + j) = make_float4(u[j], u[j + 1], u[j + 2], u[j + 3]);
  } else {
#pragma unroll
    for (int j = 0; j < E; ++j) out[lane * E + j] = u[j];
  }
}

template <int D, int HKV, bool TOK_M, bool KF16, bool SPARSE>
static cudaError_t launch_decode_dht(const DecodeParams& p, const TensorMap128& km, const TensorMap128& vm,
                                    cudaStream_t s, cudaEvent_t ev) {
  using C = DecodeCfg<D, HKV, KF16>;
  const int smem = C::OFF_PREFIX + 8 * (p.batch + 1) + 8 * 16;
  static bool attr_set = false;  // per instantiation; the attribute is per function
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, HKV, TOK_M, KF16, SPARSE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_MAX);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const CUtensorMap& kmap = *reinterpret_cast<const CUtensorMap*>(&km);
  const CUtensorMap& vmap = *reinterpret_cast<const CUtensorMap*>(&vm);
  cudaLaunchConfig_t kcfg = {};
  kcfg.gridDim = dim3((unsigned)p.grid);
  kcfg.blockDim = dim3(kThreads);
  kcfg.dynamicSmemBytes = (size_t)smem;
  kcfg.stream = s;
  cudaLaunchAttribute kattr[1];
  kattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  kattr[0].val.programmaticStreamSerializationAllowed = 1;
  kcfg.attrs = kattr;
  kcfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&kcfg, decode_split_kernel<D, HKV, TOK_M, KF16, SPARSE>, p, kmap, vmap);
  if (e != cudaSuccess) return e;
  const bool few = (int64_t)p.batch * p.n_q < 2 * (int64_t)p.grid;  // merge blocks vs SMs
  if (ev != nullptr) {  // timing split: plain stream order between the kernels
    e = cudaEventRecord(ev, s);
    if (e != cudaSuccess) return e;
    if constexpr (D <= 128) {
      if (p.tail_window > 0) {
        e = launch_tail<D>(p, s, false);
        if (e != cudaSuccess) return e;
      }
    }
    if (few)
      decode_merge_kernel<D, kMergeThreadsFew><<<p.batch * p.n_q, kMergeThreadsFew, 0, s>>>(p);
    else
      decode_merge_kernel<D, kMergeThreads><<<p.batch * p.n_q, kMergeThreads, 0, s>>>(p);
    return cudaGetLastError();
  }
  // programmatic dependent launch: the merge grid is set up while the split-K
  // grid drains; griddepcontrol.wait in the merge kernel orders the reads. With a
  // hot tail its kernel sits in between: it starts as split-K blocks finish, and
  // completes only after the split-K grid (its own wait comes last).
  if constexpr (D <= 128) {
    if (p.tail_window > 0) {
      e = launch_tail<D>(p, s, true);
      if (e != cudaSuccess) return e;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.batch * p.n_q));
  cfg.blockDim = dim3(few ? kMergeThreadsFew : kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (few) return cudaLaunchKernelEx(&cfg, decode_merge_kernel<D, kMergeThreadsFew>, p);
  return cudaLaunchKernelEx(&cfg, decode_merge_kernel<D, kMergeThreads>, p);
}

template <int D, int HKV, bool SPARSE>
static cudaError_t launch_decode_dhs(const DecodeParams& p, const TensorMap128& km, const TensorMap128& vm,
                                     cudaStream_t s, cudaEvent_t ev) {
  if constexpr (D <= 128) {
    if (p.k_f16) {
      if (p.group <= 4) return launch_decode_dht<D, HKV, true, true, SPARSE>(p, km, vm, s, ev);
      return launch_decode_dht<D, HKV, false, true, SPARSE>(p, km, vm, s, ev);
    }
  } else {
    if (p.k_f16) return cudaErrorInvalidValue;  // binary16 K tiles: head_dim <= 128
  }
  if (p.group <= 4) return launch_decode_dht<D, HKV, true, false, SPARSE>(p, km, vm, s, ev);
  return launch_decode_dht<D, HKV, false, false, SPARSE>(p, km, vm, s, ev);
}

// The sparse-V rule is a separate instantiation of the split-K kernel (head dims
// 64 and 128), so that the exact kernel carries none of its instructions.
template <int D, int HKV>
static cudaError_t launch_decode_dh(const DecodeParams& p, const TensorMap128& km, const TensorMap128& vm,
                                    cudaStream_t s, cudaEvent_t ev) {
  if (p.sparse_lt > -INFINITY) {
    if constexpr (D == 64 || D == 128) return launch_decode_dhs<D, HKV, true>(p, km, vm, s, ev);
    return cudaErrorNotSupported;
  }
  return launch_decode_dhs<D, HKV, false>(p, km, vm, s, ev);
}

template <int D>
static cudaError_t launch_decode_d(const DecodeParams& p, const TensorMap128& km, const TensorMap128& vm,
                                   cudaStream_t s, cudaEvent_t ev) {
  switch (p.n_kv) {
    case 1: return launch_decode_dh<D, 1>(p, km, vm, s, ev);
    case 2: return launch_decode_dh<D, 2>(p, km, vm, s, ev);
    case 4: return launch_decode_dh<D, 4>(p, km, vm, s, ev);
    case 8: return launch_decode_dh<D, 8>(p, km, vm, s, ev);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const DecodeParams& p, const TensorMap128& km, const TensorMap128& vm, int D,
                          cudaStream_t s, cudaEvent_t ev) {
  switch (D) {
    case 32: return launch_decode_d<32>(p, km, vm, s, ev);
    case 64: return launch_decode_d<64>(p, km, vm, s, ev);
    case 128: return launch_decode_d<128>(p, km, vm, s, ev);
    case 256: return launch_decode_d<256>(p, km, vm, s, ev);
  }
  return cudaErrorInvalidValue;
}

int decode_tile_tokens(int D, int n_kv, int k_f16) {
#define TQ_TT(DD, HH)                                                          \
  if (D == DD && n_kv == HH) {                                                 \
    if (k_f16) return DD <= 128 ? DecodeCfg<(DD <= 128 ? DD : 128), HH, true>::T_TILE : 0; \
    return DecodeCfg<DD, HH>::T_TILE;                                          \
  }
  TQ_TT(32, 1) TQ_TT(32, 2) TQ_TT(32, 4) TQ_TT(32, 8)
  TQ_TT(64, 1) TQ_TT(64, 2) TQ_TT(64, 4) TQ_TT(64, 8)
  TQ_TT(128, 1) TQ_TT(128, 2) TQ_TT(128, 4) TQ_TT(128, 8)
  TQ_TT(256, 1) TQ_TT(256, 2) TQ_TT(256, 4) TQ_TT(256, 8)
#undef TQ_TT
  return 0;
}

int decode_smem_bytes(int D, int n_kv, int k_f16) {
#define TQ_SM(DD, HH)                                                                                     \
  if (D == DD && n_kv == HH) {                                                                            \
    if (k_f16)                                                                                            \
      return DD <= 128 ? DecodeCfg<(DD <= 128 ? DD : 128), HH, true>::OFF_PREFIX + 8 * (kMaxBatch + 1) + 8 * 16 \
                       : 0;                                                                               \
    return DecodeCfg<DD, HH>::OFF_PREFIX + 8 * (kMaxBatch + 1) + 8 * 16;                                  \
  }
  TQ_SM(32, 1) TQ_SM(32, 2) TQ_SM(32, 4) TQ_SM(32, 8)
  TQ_SM(64, 1) TQ_SM(64, 2) TQ_SM(64, 4) TQ_SM(64, 8)
  TQ_SM(128, 1) TQ_SM(128, 2) TQ_SM(128, 4) TQ_SM(128, 8)
  TQ_SM(256, 1) TQ_SM(256, 2) TQ_SM(256, 4) TQ_SM(256, 8)
#undef TQ_SM
  return 0;
}

}  // namespace tqk
