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
//                 (bulk copies) into a 4-stage shared-memory ring guarded by
//                 mbarriers.
//   warps 0..7  : consumers. Warp w owns KV head w % Hkv and 16-token units of
//                 each tile. Scores and P.V run on the tensor cores with
//                 register fragments (mma.m16n8k16, f16 in, f32 accumulate):
//                 * Q.K^T: A = the rotated query of the group's q heads in
//                   two binary16 pieces (hi + lo, rows 0-7 and 8-15), B = K
//                   codes. A code nibble u (offset binary) enters the tensor
//                   core as the exact binary16 subnormal u * 2^-24 (a single
//                   lop3 per pair); the "-8" offset is folded into the
//                   accumulator's initial value, and the per-group scale is
//                   applied in binary32 after each group's two MMAs.
//                 * P.V: A = V codes (pairs of tokens at one channel, from a
//                   transposing ldmatrix), B = P times the per-(token, group)
//                   V scale, rounded once to binary16.
// Kernel 2 (decode_merge_kernel): per (sequence, q head) the partials are
// combined, normalised, and the inverse SRHT maps the result back to the
// original domain.
#include <cuda.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 4;
constexpr int kMaxBatch = 1024;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s bound on every pipeline wait

template <int D, int HKV>
struct DecodeCfg {
  static constexpr int NG = D / 32;                    // groups per head vector
  static constexpr int RB = D / 2;                     // code bytes per (token, head)
  static constexpr int WPH = kConsumerWarps / HKV;     // consumer warps per KV head
  static constexpr int UPW_MAX = 256 / D;              // 16-token units per warp per stage
  static constexpr int UPW = UPW_MAX < 16 / WPH ? UPW_MAX : 16 / WPH;
  static constexpr int T_TILE = 16 * UPW * WPH;        // tokens per stage (<= 256)
  static constexpr int CODE_BYTES = T_TILE * HKV * RB;
  static constexpr int SROW = HKV * NG * 2;            // scale bytes per token (all heads)
  static constexpr int SCALE_SLAB = ((T_TILE * SROW + 15) / 16) * 16 + 16;
  static constexpr int STAGE_BYTES = ((2 * CODE_BYTES + 2 * SCALE_SLAB + 1023) / 1024) * 1024;
  static constexpr uint32_t STAGE_TX = 2 * CODE_BYTES + 2 * SCALE_SLAB;
  static constexpr int QSTRIDE = D + 4;                // floats per staged q row (padded)
  static constexpr int SCRATCH = ((8 * QSTRIDE * 4 + 64 + 127) / 128) * 128;  // per consumer warp
  static constexpr int SWZ = RB == 128 ? 7 : RB == 64 ? 3 : RB == 32 ? 1 : 0;
  static constexpr int OFF_SCRATCH = kStages * STAGE_BYTES;
  static constexpr int OFF_BARS = OFF_SCRATCH + kConsumerWarps * SCRATCH;
  static constexpr int OFF_MISC = OFF_BARS + 2 * kStages * 8;
  static constexpr int OFF_PREFIX = OFF_MISC + 64;
  static_assert(T_TILE <= 256, "tensor-copy box limit");
  static_assert(CODE_BYTES % 1024 == 0, "V block must stay swizzle-aligned");
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
      if (x < 0 || x > p.max_seq) bad = true; else L = x;
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

// Tile walk shared by the producer and the consumers: visits every
// (sequence b, token offset t0, tokens valid in the tile) of this CTA's range.
struct TileWalker {
  const int64_t* prefix;
  int batch;
  int64_t lo, hi;
  int b;
  int64_t seg_lo, seg_hi, t0;

  __device__ void start(const int64_t* pf, int nb, int64_t l, int64_t h) {
    prefix = pf;
    batch = nb;
    lo = l;
    hi = h;
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
      const int64_t s1 = min(hi, prefix[b + 1]) - prefix[b];
      if (s0 < s1) {
        seg_lo = s0;
        seg_hi = s1;
        t0 = s0;
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

template <int D, int HKV>
__global__ void __launch_bounds__(kThreads, 1)
    decode_split_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap) {
  using C = DecodeCfg<D, HKV>;
  constexpr int NG = C::NG, RB = C::RB, T_TILE = C::T_TILE, UPW = C::UPW;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BARS);
  uint64_t* empty = full + kStages;
  int* misc = reinterpret_cast<int*>(smem + C::OFF_MISC);  // [0] abort flag
  int64_t* prefix = reinterpret_cast<int64_t*>(smem + C::OFF_PREFIX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  block_prefix_lengths(p, prefix, prefix + (p.batch + 1));
  const int64_t T_sum = prefix[p.batch];
  int64_t R = (T_sum + p.grid - 1) / p.grid;
  if (R < p.min_split) R = p.min_split;
  R = ((R + 15) / 16) * 16;
  if (blockIdx.x == 0) {  // header for the merge kernel
    int64_t* hdr = ws_header(p.ws_ml);
    for (int i = tid; i <= p.batch; i += kThreads) hdr[i] = prefix[i];
    if (tid == 0) hdr[p.batch + 1] = R;
  }
  const int64_t lo = (int64_t)blockIdx.x * R;
  const int64_t hi = min(lo + R, T_sum);
  if (lo >= hi) return;
  // the swizzle decode below assumes 1024-byte aligned stage buffers
  if ((smem_u32(smem) & 1023u) != 0) {
    if (tid == 0) status_or(p.status, TQ_STATUS_TIMEOUT);
    return;
  }

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    misc[0] = 0;
    fence_mbar_init();
  }
  __syncthreads();

  TileWalker walk;
  walk.start(prefix, p.batch, lo, hi);

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane != 0) return;
    const uint64_t pol = l2_policy_evict_first();
    const uint8_t* ks_base = reinterpret_cast<const uint8_t*>(p.k_scales);
    const uint8_t* vs_base = reinterpret_cast<const uint8_t*>(p.v_scales);
    int issued = 0;
    bool dead = false;
    for (; !walk.done(); walk.advance<T_TILE>()) {
      const int stage = issued % kStages;
      const uint32_t n = (uint32_t)(issued / kStages);
      if (!mbar_wait_bounded(&empty[stage], (n & 1u) ^ 1u, kWaitLimitNs)) {
        dead = true;
        break;
      }
      if (*reinterpret_cast<volatile int*>(&misc[0]) != 0) break;
      uint8_t* sb = smem + stage * C::STAGE_BYTES;
      mbar_arrive_expect_tx(&full[stage], C::STAGE_TX);
      const int row = (int)((int64_t)walk.b * p.max_seq + walk.t0);
      tma_load_3d(sb, &kmap, &full[stage], 0, row, 0, pol);
      tma_load_3d(sb + C::CODE_BYTES, &vmap, &full[stage], 0, row, 0, pol);
      const int64_t soff = (int64_t)row * C::SROW;  // byte offset of the tile's first scale row
      const int64_t salign = soff & ~(int64_t)15;
      bulk_load(sb + 2 * C::CODE_BYTES, ks_base + salign, C::SCALE_SLAB, &full[stage], pol);
      bulk_load(sb + 2 * C::CODE_BYTES + C::SCALE_SLAB, vs_base + salign, C::SCALE_SLAB, &full[stage], pol);
      ++issued;
    }
    if (dead) {
      misc[0] = 1;
      status_or(p.status, TQ_STATUS_TIMEOUT);
    }
    // drain: no copy may still be in flight when this thread exits
    for (int k = max(0, issued - kStages); k < issued; ++k)
      (void)mbar_wait_bounded(&full[k % kStages], (uint32_t)((k / kStages) & 1), kWaitLimitNs);
    return;
  }

  // -------------------------------------------------------------- consumers
  const int h = warp % HKV;
  const int sub = warp / HKV;
  const int gid = lane >> 2, tig = lane & 3;
  const int G = p.group;
  float* scratch = reinterpret_cast<float*>(smem + C::OFF_SCRATCH + warp * C::SCRATCH);
  const uint32_t smem_base = smem_u32(smem);

  uint32_t qA[NG][2][4];
  float biasK[NG];
  float f_h = 1.f;
  float acc[NG][2][4];
  float m_run = -INFINITY, l_run = 0.f;
  bool dead = false;
  int tile_i = 0;

  while (!walk.done()) {
    const int b = walk.b;
    const int64_t seg_hi = walk.seg_hi;
    // ---------------- segment prologue: rotate this warp's q heads, build fragments
    {
      constexpr int HP = 32 / NG;  // heads rotated per pass
      const int part = lane % NG;
      for (int j0 = 0; j0 < 8; j0 += HP) {
        const int j = j0 + lane / NG;
        float u[32];
        if (j < G && j < 8) {
          load32(u, p.q, ((int64_t)b * p.n_q + (int64_t)h * G + j) * D + part * 32, p.q_dtype);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) u[i] = apply_sign(u[i], p.sign_bits, part * 32 + i);
        fwht_group<NG>(u, part);
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          u[i] = __fmul_rn(__fmul_rn(u[i], p.c_d), p.sm_scale_log2);
          mx = fmaxf(mx, fabsf(u[i]));
        }
#pragma unroll
        for (int o = 1; o < NG; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int e = 0;
        if (mx > 0.f) (void)frexpf(mx, &e);
        const int sh = min(100, max(-100, 14 - e));  // scaled max < 2^14
        if (j < 8) {
          float* row = scratch + j * C::QSTRIDE;
#pragma unroll
          for (int i = 0; i < 32; ++i) row[part * 32 + i] = ldexpf(u[i], sh);
          if (part == 0) reinterpret_cast<int*>(scratch + 8 * C::QSTRIDE)[j] = sh;
        }
      }
      __syncwarp();
      const float* row = scratch + gid * C::QSTRIDE;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        float qv[8];
#pragma unroll
        for (int n = 0; n < 8; ++n) qv[n] = (gid < G) ? row[32 * g + 8 * tig + n] : 0.f;
        float bsum = 0.f;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          // ks = 0 covers nibbles {0,4} (low position) and {1,5} (high position);
          // ks = 1 covers nibbles {2,6} and {3,7}.
          const float lo0 = qv[2 * ks], lo1 = qv[2 * ks + 4];
          const float hi0 = qv[2 * ks + 1] * 0.0625f, hi1 = qv[2 * ks + 5] * 0.0625f;
          const __half a0 = __float2half_rn(lo0), a1 = __float2half_rn(lo1);
          const __half c0 = __float2half_rn(hi0), c1 = __float2half_rn(hi1);
          const __half a0l = __float2half_rn(lo0 - __half2float(a0)), a1l = __float2half_rn(lo1 - __half2float(a1));
          const __half c0l = __float2half_rn(hi0 - __half2float(c0)), c1l = __float2half_rn(hi1 - __half2float(c1));
          qA[g][ks][0] = (uint32_t)__half_as_ushort(a0) | ((uint32_t)__half_as_ushort(a1) << 16);
          qA[g][ks][1] = (uint32_t)__half_as_ushort(a0l) | ((uint32_t)__half_as_ushort(a1l) << 16);
          qA[g][ks][2] = (uint32_t)__half_as_ushort(c0) | ((uint32_t)__half_as_ushort(c1) << 16);
          qA[g][ks][3] = (uint32_t)__half_as_ushort(c0l) | ((uint32_t)__half_as_ushort(c1l) << 16);
          bsum += (__half2float(a0) + __half2float(a0l)) + (__half2float(a1) + __half2float(a1l));
          bsum += 16.f * ((__half2float(c0) + __half2float(c0l)) + (__half2float(c1) + __half2float(c1l)));
        }
        bsum += __shfl_xor_sync(0xffffffffu, bsum, 1);
        bsum += __shfl_xor_sync(0xffffffffu, bsum, 2);
        biasK[g] = -bsum * (8.0f * 5.9604644775390625e-08f);  // 8 * 2^-24
      }
      const int sh = (gid < G) ? reinterpret_cast<const int*>(scratch + 8 * C::QSTRIDE)[gid] : 0;
      f_h = __int_as_float((127 + 24 - sh) << 23);  // 2^(24 - sh): MMA units -> log2 units
      __syncwarp();
#pragma unroll
      for (int g = 0; g < NG; ++g)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[g][jj][r] = 0.f;
      m_run = -INFINITY;
      l_run = 0.f;
    }

    // ---------------- token tiles of this segment
    bool seg_end = false;
    while (!seg_end) {
      const int stage = tile_i % kStages;
      const uint32_t par = (uint32_t)((tile_i / kStages) & 1);
      if (!dead) {
        if (*reinterpret_cast<volatile int*>(&misc[0]) != 0 ||
            !mbar_wait_bounded(&full[stage], par, kWaitLimitNs)) {
          dead = true;
          if (lane == 0) status_or(p.status, TQ_STATUS_TIMEOUT);
        }
      }
      if (!dead) {
        const uint32_t sbase = smem_base + stage * C::STAGE_BYTES;
        const uint32_t kc = sbase + h * T_TILE * RB;
        const uint32_t vc = sbase + C::CODE_BYTES + h * T_TILE * RB;
        const int64_t row0 = (int64_t)b * p.max_seq + walk.t0;
        const int soff = (int)((row0 * C::SROW) & 15);
        const uint8_t* ksr = smem + stage * C::STAGE_BYTES + 2 * C::CODE_BYTES + soff;
        const uint8_t* vsr = ksr + C::SCALE_SLAB;
#pragma unroll 1
        for (int u = 0; u < UPW; ++u) {
          const int r0 = (sub * UPW + u) * 16;  // first tile row of this unit
          const int64_t tok0 = walk.t0 + r0;
          if (tok0 >= seg_hi) break;
          const int nv = (int)min((int64_t)16, seg_hi - tok0);

          // --- K and V code fragments
          uint32_t kw[2][NG], vw[NG][2];
          {
            const int rr = lane & 7, mi = lane >> 3;
            if constexpr (NG == 1) {
              uint32_t t2[2];
              const int row = r0 + (mi & 1) * 8 + rr;
              ldmatrix_x2(t2, kc + row * RB);
              kw[0][0] = t2[0];
              kw[1][0] = t2[1];
              ldmatrix_x2_trans(t2, vc + row * RB);
              vw[0][0] = t2[0];
              vw[0][1] = t2[1];
            } else {
#pragma unroll
              for (int m4 = 0; m4 < 2 * NG; m4 += 4) {
                const int m = m4 + mi;
                {  // K: matrix m = (n-tile m / NG, group m % NG)
                  const int row = r0 + (m / NG) * 8 + rr;
                  const int grp = m % NG;
                  const int roff = (h * T_TILE + row) * RB;
                  const uint32_t addr = kc + row * RB + ((grp ^ ((roff >> 7) & C::SWZ)) << 4);
                  uint32_t t4[4];
                  ldmatrix_x4(t4, addr);
#pragma unroll
                  for (int i = 0; i < 4; ++i) kw[(m4 + i) / NG][(m4 + i) % NG] = t4[i];
                }
                {  // V: matrix m = (group m / 2, token half m % 2)
                  const int row = r0 + (m & 1) * 8 + rr;
                  const int grp = m >> 1;
                  const int roff = (h * T_TILE + row) * RB;
                  const uint32_t addr = vc + row * RB + ((grp ^ ((roff >> 7) & C::SWZ)) << 4);
                  uint32_t t4[4];
                  ldmatrix_x4_trans(t4, addr);
#pragma unroll
                  for (int i = 0; i < 4; ++i) vw[(m4 + i) >> 1][(m4 + i) & 1] = t4[i];
                }
              }
            }
          }

          // --- binary16 scales of this unit -> binary32 (masked tokens -> 0)
          float* sc = scratch;  // [2][16][NG]
          {
            constexpr int HPL = NG >= 2 ? NG / 2 : 1;      // halves per lane
            constexpr int LPT = NG / HPL;                  // lanes per token
            constexpr int USED = 16 * LPT;
            if (lane < USED) {
              const int tk = lane / LPT, first = (lane % LPT) * HPL;
              const int so = ((r0 + tk) * HKV + h) * NG * 2 + first * 2;
#pragma unroll
              for (int i = 0; i < HPL; ++i) {
                const bool ok = tk < nv;
                const float sk = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(ksr + so + 2 * i)));
                const float sv = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(vsr + so + 2 * i)));
                sc[tk * NG + first + i] = ok ? sk : 0.f;
                sc[16 * NG + tk * NG + first + i] = ok ? sv : 0.f;
              }
            }
          }
          __syncwarp();

          // --- scores S[head gid][token] for tokens nt*8 + 2*tig + e
          float s[2][2];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            s[nt][0] = 0.f;
            s[nt][1] = 0.f;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
              float c[4] = {biasK[g], biasK[g], 0.f, 0.f};
              const uint32_t w = kw[nt][g];
              mma_f16_16816(c, qA[g][0], and_xor(w, 0x000F000Fu, 0x00080008u), and_xor(w, 0x00F000F0u, 0x00800080u));
              const uint32_t w8 = w >> 8;
              mma_f16_16816(c, qA[g][1], and_xor(w8, 0x000F000Fu, 0x00080008u), and_xor(w8, 0x00F000F0u, 0x00800080u));
              const int t0i = nt * 8 + 2 * tig;
              s[nt][0] = fmaf(sc[t0i * NG + g], c[0] + c[2], s[nt][0]);
              s[nt][1] = fmaf(sc[(t0i + 1) * NG + g], c[1] + c[3], s[nt][1]);
            }
#pragma unroll
            for (int e = 0; e < 2; ++e)
              if (nt * 8 + 2 * tig + e >= nv) s[nt][e] = -INFINITY;
          }

          // --- online softmax (head gid; quad lanes share a head)
          float mx = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          const float m_new = fmaxf(m_run, mx);
          const bool grow = m_new > m_run;
          if (__any_sync(0xffffffffu, grow)) {
            const float corr = grow ? ((m_run == -INFINITY) ? 0.f : exp2f((m_run - m_new) * f_h)) : 1.f;
            l_run *= corr;
            const float c0 = __shfl_sync(0xffffffffu, corr, 8 * tig);
            const float c1 = __shfl_sync(0xffffffffu, corr, 8 * tig + 4);
#pragma unroll
            for (int g = 0; g < NG; ++g)
#pragma unroll
              for (int jj = 0; jj < 2; ++jj) {
                acc[g][jj][0] *= c0;
                acc[g][jj][1] *= c1;
                acc[g][jj][2] *= c0;
                acc[g][jj][3] *= c1;
              }
            m_run = m_new;
          }
          const float mb = (m_run == -INFINITY) ? 0.f : m_run * f_h;
          float pr[2][2];
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              pr[nt][e] = exp2f(fmaf(s[nt][e], f_h, -mb));
              l_run += pr[nt][e];
            }

          // --- P.V: acc[d][head] += sum_t v[t][d] * (p[t] * sigmaV[t][g])
          const float* sv = sc + 16 * NG;
          const uint32_t K8 = 0x00080008u;       // binary16 pair (8 * 2^-24, 8 * 2^-24)
          const uint32_t NEG8 = 0x80088008u;     // (-8 * 2^-24, -8 * 2^-24)
          const uint32_t SIXTEENTH = 0x2C002C00u;  // (1/16, 1/16)
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            const int t0i = 2 * tig;
            const uint32_t b0 = pack_half2(pr[0][0] * sv[t0i * NG + g], pr[0][1] * sv[(t0i + 1) * NG + g]);
            const uint32_t b1 = pack_half2(pr[1][0] * sv[(t0i + 8) * NG + g], pr[1][1] * sv[(t0i + 9) * NG + g]);
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
              const uint32_t va = jj ? (vw[g][0] >> 8) : vw[g][0];
              const uint32_t vb = jj ? (vw[g][1] >> 8) : vw[g][1];
              uint32_t a[4];
              const uint32_t lo_a = and_xor(va, 0x000F000Fu, K8);
              const uint32_t hi_a = and_xor(va, 0x00F000F0u, 0x00800080u);
              const uint32_t lo_b = and_xor(vb, 0x000F000Fu, K8);
              const uint32_t hi_b = and_xor(vb, 0x00F000F0u, 0x00800080u);
              const __half2 k8 = *reinterpret_cast<const __half2*>(&K8);
              const __half2 n8 = *reinterpret_cast<const __half2*>(&NEG8);
              const __half2 s16 = *reinterpret_cast<const __half2*>(&SIXTEENTH);
              __half2 r;
              r = __hsub2(*reinterpret_cast<const __half2*>(&lo_a), k8);
              a[0] = *reinterpret_cast<uint32_t*>(&r);
              r = __hfma2(*reinterpret_cast<const __half2*>(&hi_a), s16, n8);
              a[1] = *reinterpret_cast<uint32_t*>(&r);
              r = __hsub2(*reinterpret_cast<const __half2*>(&lo_b), k8);
              a[2] = *reinterpret_cast<uint32_t*>(&r);
              r = __hfma2(*reinterpret_cast<const __half2*>(&hi_b), s16, n8);
              a[3] = *reinterpret_cast<uint32_t*>(&r);
              mma_f16_16816(acc[g][jj], a, b0, b1);
            }
          }
          __syncwarp();  // scale scratch is rewritten by the next unit
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
    l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 1);
    l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 2);
    const float m_real = (m_run == -INFINITY) ? -INFINITY : m_run * f_h;
    constexpr float kTwo24 = 16777216.f;
    if constexpr (C::WPH == 1) {
      if (!dead) {
        if (tig == 0 && gid < G) {
          float* ml = p.ws_ml + (((int64_t)slot * p.n_q + h * G + gid) * 2) + 2 * (p.batch + 2);
          ml[0] = m_real;
          ml[1] = l_tot;
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int hh = 2 * tig + e;
          if (hh < G) {
            float* dst = p.ws_acc + ((int64_t)slot * p.n_q + h * G + hh) * D;
#pragma unroll
            for (int g = 0; g < NG; ++g)
              *reinterpret_cast<float4*>(dst + 32 * g + 4 * gid) =
                  make_float4(acc[g][0][e] * kTwo24, acc[g][0][2 + e] * kTwo24, acc[g][1][e] * kTwo24,
                              acc[g][1][2 + e] * kTwo24);
          }
        }
      }
    } else {
      // several warps share a KV head: combine their states through shared memory
      float* mls = scratch + 8 * D;  // [8][2]
      if (tig == 0 && gid < 8) {
        mls[2 * gid] = dead ? -INFINITY : m_real;
        mls[2 * gid + 1] = dead ? 0.f : l_tot;
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int hh = 2 * tig + e;
#pragma unroll
        for (int g = 0; g < NG; ++g)
          *reinterpret_cast<float4*>(scratch + hh * D + 32 * g + 4 * gid) =
              dead ? make_float4(0.f, 0.f, 0.f, 0.f)
                   : make_float4(acc[g][0][e] * kTwo24, acc[g][0][2 + e] * kTwo24, acc[g][1][e] * kTwo24,
                                 acc[g][1][2 + e] * kTwo24);
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
      const int ctid = tid;  // 0 .. 255
      const int items = HKV * G * D;
      for (int it = ctid; it < items; it += kConsumerWarps * 32) {
        const int hk = it / (G * D), j = (it / D) % G, d = it % D;
        float mstar = -INFINITY;
        for (int sb = 0; sb < C::WPH; ++sb) {
          const float* sm = reinterpret_cast<const float*>(smem + C::OFF_SCRATCH + (hk + sb * HKV) * C::SCRATCH);
          mstar = fmaxf(mstar, sm[8 * D + 2 * j]);
        }
        float lsum = 0.f, asum = 0.f;
        if (mstar != -INFINITY) {
          for (int sb = 0; sb < C::WPH; ++sb) {
            const float* sm = reinterpret_cast<const float*>(smem + C::OFF_SCRATCH + (hk + sb * HKV) * C::SCRATCH);
            const float mw = sm[8 * D + 2 * j];
            if (mw == -INFINITY) continue;
            const float wgt = exp2f(mw - mstar);
            lsum += wgt * sm[8 * D + 2 * j + 1];
            asum += wgt * sm[j * D + d];
          }
        }
        const int64_t qh = (int64_t)slot * p.n_q + hk * G + j;
        p.ws_acc[qh * D + d] = asum;
        if (d == 0) {
          float* ml = p.ws_ml + qh * 2 + 2 * (p.batch + 2);
          ml[0] = mstar;
          ml[1] = lsum;
        }
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kConsumerWarps * 32) : "memory");
    }
  }
}

// Combine the partials of one (sequence, q head), normalise, inverse SRHT.
template <int D>
__global__ void __launch_bounds__(128) decode_merge_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int NG = D / 32;
  constexpr int F4 = D / 4;            // float4 columns
  constexpr int PH = 128 / F4;         // slot phases
  __shared__ float red[128];
  __shared__ __align__(16) float accs[PH][D];
  __shared__ float bc[2];
  const int tid = threadIdx.x;
  const int b = blockIdx.x / p.n_q, hq = blockIdx.x % p.n_q;
  const int64_t* hdr = ws_header(p.ws_ml);
  const int64_t P0 = hdr[b], P1 = hdr[b + 1], R = hdr[p.batch + 1];
  const float* ml = p.ws_ml + 2 * (p.batch + 2);
  float* out = p.out + ((int64_t)b * p.n_q + hq) * D;
  if (P1 <= P0) {  // empty sequence
    for (int d = tid; d < D; d += 128) out[d] = 0.f;
    return;
  }
  const int c0 = (int)(P0 / R), c1 = (int)((P1 - 1) / R);
  const int ns = c1 - c0 + 1;
  // pass 1: global max
  float m = -INFINITY;
  for (int i = tid; i < ns; i += 128) m = fmaxf(m, ml[((int64_t)(b + c0 + i) * p.n_q + hq) * 2]);
  red[tid] = m;
  __syncthreads();
  for (int o = 64; o > 0; o >>= 1) {
    if (tid < o) red[tid] = fmaxf(red[tid], red[tid + o]);
    __syncthreads();
  }
  const float mstar = red[0];
  __syncthreads();
  // pass 2: weighted sums
  float lsum = 0.f;
  for (int i = tid; i < ns; i += 128) {
    const float* e = ml + ((int64_t)(b + c0 + i) * p.n_q + hq) * 2;
    if (e[0] != -INFINITY) lsum += exp2f(e[0] - mstar) * e[1];
  }
  red[tid] = lsum;
  const int col = tid % F4, ph = tid / F4;
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
  if (ph < PH) {
    for (int i = ph; i < ns; i += PH) {
      const int64_t qh = (int64_t)(b + c0 + i) * p.n_q + hq;
      const float mw = ml[qh * 2];
      if (mw == -INFINITY) continue;
      const float w = exp2f(mw - mstar);
      const float4 v = reinterpret_cast<const float4*>(p.ws_acc + qh * D)[col];
      a.x = fmaf(w, v.x, a.x);
      a.y = fmaf(w, v.y, a.y);
      a.z = fmaf(w, v.z, a.z);
      a.w = fmaf(w, v.w, a.w);
    }
    reinterpret_cast<float4*>(accs[ph])[col] = a;
  }
  __syncthreads();
  for (int o = 64; o > 0; o >>= 1) {
    if (tid < o) red[tid] += red[tid + o];
    __syncthreads();
  }
  if (tid == 0) bc[0] = red[0];
  __syncthreads();
  const float L = bc[0];
  // inverse SRHT on the normalised rotated-domain output: first warp, NG lanes
  if (tid < 32) {
    const int part = tid % NG;
    float u[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float s = 0.f;
      for (int q = 0; q < PH; ++q) s += accs[q][part * 32 + i];
      u[i] = (L > 0.f) ? s / L : 0.f;
    }
    fwht_group<NG>(u, part);
    if (tid < NG) {
#pragma unroll
      for (int i = 0; i < 32; ++i) out[part * 32 + i] = apply_sign(u[i] * p.c_d, p.sign_bits, part * 32 + i);
    }
  }
}

template <int D, int HKV>
static cudaError_t launch_decode_dh(const DecodeParams& p, const TensorMap128& km, const TensorMap128& vm,
                                    cudaStream_t s, cudaEvent_t ev) {
  using C = DecodeCfg<D, HKV>;
  const int smem = C::OFF_PREFIX + 8 * (p.batch + 1) + 8 * 16;
  static bool attr_set = false;  // per instantiation; the attribute is per function
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, HKV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::OFF_PREFIX + 8 * (kMaxBatch + 1) + 8 * 16);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const CUtensorMap& kmap = *reinterpret_cast<const CUtensorMap*>(&km);
  const CUtensorMap& vmap = *reinterpret_cast<const CUtensorMap*>(&vm);
  decode_split_kernel<D, HKV><<<p.grid, kThreads, smem, s>>>(p, kmap, vmap);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (ev != nullptr) {
    e = cudaEventRecord(ev, s);
    if (e != cudaSuccess) return e;
  }
  decode_merge_kernel<D><<<p.batch * p.n_q, 128, 0, s>>>(p);
  return cudaGetLastError();
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

int decode_tile_tokens(int D, int n_kv) {
#define TQ_TT(DD, HH) \
  if (D == DD && n_kv == HH) return DecodeCfg<DD, HH>::T_TILE;
  TQ_TT(32, 1) TQ_TT(32, 2) TQ_TT(32, 4) TQ_TT(32, 8)
  TQ_TT(64, 1) TQ_TT(64, 2) TQ_TT(64, 4) TQ_TT(64, 8)
  TQ_TT(128, 1) TQ_TT(128, 2) TQ_TT(128, 4) TQ_TT(128, 8)
  TQ_TT(256, 1) TQ_TT(256, 2) TQ_TT(256, 4) TQ_TT(256, 8)
#undef TQ_TT
  return 0;
}

int decode_smem_bytes(int D, int n_kv) {
#define TQ_SM(DD, HH) \
  if (D == DD && n_kv == HH) return DecodeCfg<DD, HH>::OFF_PREFIX + 8 * (kMaxBatch + 1) + 8 * 16;
  TQ_SM(32, 1) TQ_SM(32, 2) TQ_SM(32, 4) TQ_SM(32, 8)
  TQ_SM(64, 1) TQ_SM(64, 2) TQ_SM(64, 4) TQ_SM(64, 8)
  TQ_SM(128, 1) TQ_SM(128, 2) TQ_SM(128, 4) TQ_SM(128, 8)
  TQ_SM(256, 1) TQ_SM(256, 2) TQ_SM(256, 4) TQ_SM(256, 8)
#undef TQ_SM
  return 0;
}

}  // namespace tqk
