// Grouped NVFP4 expert GEMMs of the MoE layer (w13 with the SwiGLU + h
// re-quantization epilogue, w2 with the routing-weighted fp32 epilogue) on
// CTA pairs.
//
// "DeepSeek-V4.1-Flash-NVFP4", §二: per expert e, h = SwiGLU(x W13_e^T) and
// y = w_slot * (h W2_e^T), both products W4A4 with E4M3 scales per 16
// elements; the arithmetic is that of gemm.cu's grouped path.  What differs
// is how the work is laid on the tensor cores:
//
//   * The expert's WEIGHT rows are the MMA's M side and its routed TOKENS the
//     N side (D^T = W . X^T).  A tile is 256 weight rows x up to 256 tokens;
//     the weight side is always full (2I and H are multiples of 256) and the
//     token side is rounded up only to the next multiple of 16, so an
//     expert's last tile computes at most 15 padding tokens (a 128-row token
//     tile pads up to 127).
//   * Each tile runs on a cluster of two CTAs with one tcgen05.mma
//     cta_group::2 of M = 256: each CTA stages 128 weight rows and half of
//     the tile's tokens, so an SM loads 38 KB per 256-deep K stage for the
//     same MMA time that a 1-CTA 128 x 256 tile needs 55 KB for.  That keeps
//     five stages in shared memory and halves the token (B) traffic per SM.
//
// Roles per CTA (352 threads), mirroring gemm.cu:
//   warp 0      TMA producer (both CTAs): per K stage, 128 weight rows, the
//               CTA's half of the token rows (32-row boxes), and the scale
//               tiles (2 KB boxes of the tiled layout: the CTA's 128 weight
//               rows, all of the tile's token rows); every copy completes on
//               the LEADER's "full" barrier, which the leader primes with the
//               bytes of both CTAs.
//   warp 2      scale copier (leader): tcgen05.cp cta_group::2 of the stage's
//               scale tiles into both CTAs' TMEM, commit to "sf_full".
//   warp 1      TMEM allocation (both CTAs, one pair allocation); on the
//               leader one lane issues the stage's 4 MMAs (K = 64 each) and
//               commits to "empty" in both CTAs, and to "acc_full" in both
//               after the tile's last stage.
//   warps 3-10  epilogue (both CTAs): tcgen05.ld of the CTA's 128 weight rows
//               x the tile's tokens, arrive on the leader's "acc_empty", then
//                 w13  lanes 0-15 / 16-31 of a 32-lane quarter hold the gate /
//                      up rows of one 16-feature block of h: exchange halves
//                      by shuffle, SwiGLU, transpose to token rows through
//                      shared memory, NVFP4-quantize each token's block with
//                      the expert's static h scale
//                 w2   alpha * routing weight * acc, 32 consecutive outputs of
//                      one token per warp store
//
// Tiles walk (expert, 256-token chunk, 256-row weight tile) with the weight
// tile innermost, so clusters running at the same time share the chunk's
// tokens and the expert's weights in L2.  Every mbarrier wait is bounded as
// in gemm.cu; both CTAs meet at a cluster barrier before freeing TMEM.
//
// Opt-in (FP4_MOE_PAIR_TILES): measured on B200 it is slower than gemm.cu's
// 1-CTA row tiles on every MoE shape tried.  Each 256-deep K stage still
// needs 12 scale copies (4 x 4 columns of weight scales, 4 x 8 of token
// scales; about 45 cycles each in the tensor pipe), an expert's last chunk
// pays all of them for as few as 16 tokens, and a pair's stage waits on the
// loads of both CTAs (about 3500 cycles from issue to arrival under load).
#include "host.cuh"

namespace fp4 {
namespace {

constexpr int kFirstEpiWarp = 3;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
constexpr int kStages = 5;
constexpr int A_BYTES = 128 * 128;     // 128 weight rows x 256 FP4 (128-byte swizzled rows)
constexpr int B_BYTES = 128 * 128;     // up to 128 token rows (half of the tile's N)
constexpr int B_BOX_ROWS = 32;
constexpr int B_BOX_BYTES = B_BOX_ROWS * 128;
constexpr int SF_BOX_BYTES = 2048;     // one 128-row slab x 4 K steps of the tiled scale layout
constexpr int SFA_BYTES = SF_BOX_BYTES;
constexpr int SFB_BYTES = 2 * SF_BOX_BYTES;  // up to 256 token rows
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int STG_STRIDE = 17;         // floats per token row of the w13 transpose buffer (bank-conflict free)
constexpr int STG_WARP_FLOATS = 32 * STG_STRIDE;
constexpr int TMEM_COLS = 512;
constexpr int SF_COL0 = 256;           // accumulator in columns 0-255, scale slots after it
constexpr int SF_SLOT_COLS = 16 + 32;  // SFA: 4 K steps x 4 columns; SFB: 4 x 8 (two 128-row groups)
constexpr int kBarriers = 3 * kStages + 4;
static_assert(STAGE_BYTES % 1024 == 0, "stage buffers stay 1024-byte aligned");
static_assert(SF_COL0 + kStages * SF_SLOT_COLS <= TMEM_COLS, "tmem");
static_assert(kBarriers * 8 <= 256, "barriers");

enum PairEpi { PAIR_W13 = 0, PAIR_W2 = 1 };

constexpr int stg_bytes(int epi) { return epi == PAIR_W13 ? kEpiWarps * STG_WARP_FLOATS * 4 : 0; }
inline int scan_bytes(int E) { return ((E + 1) * 4 + 15) & ~15; }
inline int smem_bytes(int epi, int E) {
  return 1024 /*align*/ + kStages * STAGE_BYTES + stg_bytes(epi) + scan_bytes(E) + 256 /*barriers*/;
}

struct PairParams {
  int E;
  int MT;          // 256-row weight tiles per expert (2I / 256 or H / 256)
  int w_rows;      // weight rows per expert (2I or H)
  int k_stages;    // K / 256
  int kw;          // K / 64: scale words per row (tiled-layout K steps)
  const int32_t *counts;
  const int32_t *offsets;
  const int32_t *tile_offsets;
  const float *a_g;   // w13: activation tensor scale (device scalar)
  const float *w_g;   // per-expert weight tensor scale
  const float *h_g;   // per-expert static h scale
  uint8_t *h_codes;
  uint8_t *h_sf;
  float *h_dump;
  int I;
  const int32_t *perm;
  const float *topk_w;
  float *y;
  int H;
  unsigned int *status;
  uint64_t wait_limit;
};

struct PairTile {
  int e;         // expert
  int m;         // 256-row weight tile within the expert
  int n;         // tokens of the chunk
  int N;         // n rounded up to 16 (MMA N)
  int row0;      // first padded routed row of the chunk (gathered-buffer row)
  int out_row0;  // first unpadded routed row of the chunk (y row)
};

__device__ __forceinline__ PairTile pair_tile(const PairParams &p, const int32_t *scan, int t) {
  PairTile ti;
  const int u = t / p.MT;  // chunk index over all experts
  ti.m = t - u * p.MT;
  int lo = 0, hi = p.E + 1;  // first index with scan[i] > u
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (scan[mid] <= u) lo = mid + 1; else hi = mid;
  }
  ti.e = lo - 1;
  const int j = u - scan[ti.e];
  ti.n = min(256, p.counts[ti.e] - 256 * j);
  ti.N = (ti.n + 15) & ~15;
  ti.row0 = p.tile_offsets[ti.e] * 128 + 256 * j;
  ti.out_row0 = p.offsets[ti.e] + 256 * j;
  return ti;
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    moe_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                    const PairParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *smA = smem;
  uint8_t *smB = smA + kStages * A_BYTES;
  uint8_t *smSFA = smB + kStages * B_BYTES;
  uint8_t *smSFB = smSFA + kStages * SFA_BYTES;
  float *stg = reinterpret_cast<float *>(smSFB + kStages * SFB_BYTES);
  int32_t *scan = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(stg) + stg_bytes(EPI));
  uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(scan) + (((p.E + 1) * 4 + 15) & ~15));
  uint64_t *full = bars;                       // leader: both CTAs' TMA data landed (count 1 + tx)
  uint64_t *empty = bars + kStages;            // both: the pair's MMAs are done with a stage
  uint64_t *sf_full = bars + 2 * kStages;      // leader: stage scales in both TMEMs
  uint64_t *acc_full = bars + 3 * kStages;     // both: tile accumulated
  uint64_t *acc_empty = acc_full + 1;          // leader: both CTAs' epilogue warps read the accumulator
  uint64_t *drain_mma = acc_full + 2;
  uint64_t *drain_sf = acc_full + 3;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: leader
  const bool leader = rank == 0;
  const int pair = (int)cluster_id_x(), npairs = (int)nclusters_x();

  // per-expert 256-token chunk counts, exclusive prefix in scan[0..E]
  for (int e = threadIdx.x; e < p.E; e += kThreads) scan[e + 1] = (p.counts[e] + 255) >> 8;
  if (threadIdx.x == 0) {
    scan[0] = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kEpiWarps);
    mbar_init(drain_mma, 1);
    mbar_init(drain_sf, 1);
    fence_barrier_init();
    s_abort = 0;
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSA);
    prefetch_tmap(&tmSB);
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < p.E; base += 32) {
      const int i = base + lane;
      int v = (i < p.E) ? scan[i + 1] : 0;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += o;
      }
      if (i < p.E) scan[i + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&s_tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = s_tmem_base;
  const int total = scan[p.E] * p.MT;
  const uint64_t lim = p.wait_limit;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
      int stage = 0;
      uint32_t phase = 0;
      int issued[kStages];
      uint32_t issued_par[kStages];
      for (int s = 0; s < kStages; ++s) issued[s] = 0;
      bool ok = true;
      for (int t = pair; ok && t < total; t += npairs) {
        const PairTile ti = pair_tile(p, scan, t);
        const int half_n = ti.N >> 1;  // token rows staged by each CTA (a multiple of 8)
        const int nb = (half_n + B_BOX_ROWS - 1) / B_BOX_ROWS;
        const int nsl = ti.N > 128 ? 2 : 1;  // 128-row scale slabs of the tile's tokens
        const uint32_t cta_bytes = (uint32_t)(A_BYTES + nb * B_BOX_BYTES + SFA_BYTES + nsl * SF_BOX_BYTES);
        const int a_row = ti.e * p.w_rows + ti.m * 256 + (int)rank * 128;
        const int b_row = ti.row0 + (int)rank * half_n;
        const int a_slab = a_row >> 7;
        const int b_slab = ti.row0 >> 7;
        for (int kt = 0; kt < p.k_stages; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, &s_abort, p.status, lim)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2u * cta_bytes);
          const uint32_t fb = full_leader + 8u * (uint32_t)stage;
          tma_load_2d_pair(smA + stage * A_BYTES, &tmA, fb, kt * 128, a_row);
          for (int b = 0; b < nb; ++b)
            tma_load_2d_pair(smB + stage * B_BYTES + b * B_BOX_BYTES, &tmB, fb, kt * 128, b_row + b * B_BOX_ROWS);
          tma_load_2d_pair(smSFA + stage * SFA_BYTES, &tmSA, fb, 0, (a_slab * p.kw + kt * 4) * 2);
          for (int h = 0; h < nsl; ++h)
            tma_load_2d_pair(smSFB + stage * SFB_BYTES + h * SF_BOX_BYTES, &tmSB, fb, 0,
                             ((b_slab + h) * p.kw + kt * 4) * 2);
          issued[stage] = 1;
          issued_par[stage] = phase;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (ok) {
        // every stage's last release (the leader's commits into this CTA's
        // "empty" barriers) has landed before the CTA can leave
        for (int s = 0; s < kStages; ++s) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, &s_abort, p.status, lim)) break;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      } else if (leader) {  // copies in flight land before the CTA exits
        for (int s = 0; s < kStages; ++s)
          if (issued[s]) mbar_drain(&full[s], issued_par[s], 1000000000ull);
      } else {  // the follower cannot observe the leader's barrier: give its copies time to land
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale copier (leader)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, any = false;
      for (int t = pair; ok && t < total; t += npairs) {
        const PairTile ti = pair_tile(p, scan, t);
        const int nsl = ti.N > 128 ? 2 : 1;
        for (int kt = 0; kt < p.k_stages; ++kt) {
          if (!mbar_wait(&full[stage], phase, &s_abort, p.status, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ta = tmem + SF_COL0 + stage * SF_SLOT_COLS;
          const uint32_t tb = ta + 16;
          const uint64_t da = smem_desc(smem_u32(smSFA + stage * SFA_BYTES), 0, 128, 0);
          const uint64_t db = smem_desc(smem_u32(smSFB + stage * SFB_BYTES), 0, 128, 0);
#pragma unroll
          for (int w = 0; w < 4; ++w) {  // 512-byte tile w = K step w (+32 in 16-byte units)
            tmem_cp_sf_pair(ta + w * 4, da + (uint64_t)(w * 32));
            for (int h = 0; h < nsl; ++h) tmem_cp_sf_pair(tb + w * 8 + h * 4, db + (uint64_t)((h * 4 + w) * 32));
          }
          any = true;
          tc_commit_pair(&sf_full[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && any) {
        tc_commit_pair(drain_sf);
        mbar_drain(drain_sf, 0, 1000000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, any_mma = false;
      for (int t = pair; ok && t < total; t += npairs) {
        const PairTile ti = pair_tile(p, scan, t);
        const uint32_t idesc = idesc_mxf4nvf4(256, (uint32_t)ti.N);
        if (!mbar_wait_cluster(acc_empty, acc_phase ^ 1u, &s_abort, p.status, lim)) { ok = false; break; }
        tc_fence_after();
        for (int kt = 0; kt < p.k_stages; ++kt) {
          if (!mbar_wait(&full[stage], phase, &s_abort, p.status, lim)) { ok = false; break; }
          if (!mbar_wait(&sf_full[stage], phase, &s_abort, p.status, lim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ta = tmem + SF_COL0 + stage * SF_SLOT_COLS;
          const uint32_t tb = ta + 16;
          const uint64_t ad = smem_desc(smem_u32(smA + stage * A_BYTES), 16, 1024, 2);
          const uint64_t bd = smem_desc(smem_u32(smB + stage * B_BYTES), 16, 1024, 2);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_nvf4_pair(tmem, ad + (uint64_t)(j * 2), bd + (uint64_t)(j * 2), idesc, ta + j * 4, tb + j * 8,
                          (kt > 0 || j > 0) ? 1u : 0u);
          any_mma = true;
          tc_commit_pair_both(&empty[stage], 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_both(acc_full, 0x3);
        acc_phase ^= 1u;
      }
      if (!ok && any_mma) {
        tc_commit_pair(drain_mma);
        mbar_drain(drain_mma, 0, 1000000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;                        // TMEM lane quarter this warp may access
    const int half = (warp - kFirstEpiWarp) >> 2;  // which 128 token columns of the tile
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    float *wstg = stg + (warp - kFirstEpiWarp) * STG_WARP_FLOATS;
    uint32_t acc_phase = 0;
    for (int t = pair; t < total; t += npairs) {
      const PairTile ti = pair_tile(p, scan, t);
      if (!mbar_wait(acc_full, acc_phase, &s_abort, p.status, lim)) break;
      tc_fence_after();
      float v[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (half * 128 + c * 32 < ti.N) {
          __syncwarp();
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + half * 128 + c * 32, v + 32 * c);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty_leader);  // the accumulator is in registers now
      acc_phase ^= 1u;

      if constexpr (EPI == PAIR_W13) {
        const float alpha = __fmul_rn(*p.a_g, p.w_g[ti.e]);
        const float hg = p.h_g[ti.e];
        // this quarter's 32 weight rows = gate (lanes 0-15) and up (16-31)
        // rows of h block kb, features 16 kb .. 16 kb + 15
        const int kb = ti.m * 8 + (int)rank * 4 + q;
        const bool lower = lane < 16;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col0 = half * 128 + c * 32;
          if (col0 >= ti.N) break;
          const float *w = v + 32 * c;
          // lower lane f: tokens col0 .. col0+15; upper lane 16+f: col0+16 .. col0+31
          float h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float r = __shfl_xor_sync(0xffffffffu, lower ? w[16 + i] : w[i], 16);
            const float gte = __fmul_rn(lower ? w[i] : r, alpha);
            const float up = __fmul_rn(lower ? r : w[16 + i], alpha);
            h[i] = __fmul_rn(silu_f32(gte), up);
          }
          const int f = lane & 15, tok0 = lower ? 0 : 16;
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 16; ++i) wstg[(tok0 + i) * STG_STRIDE + f] = h[i];
          __syncwarp();
          float x[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) x[i] = wstg[lane * STG_STRIDE + i];
          const int tk = col0 + lane;  // token of this lane within the chunk
          if (tk < ti.N) {
            const int64_t row = (int64_t)ti.row0 + tk;
            uint32_t lo = 0, hi = 0, sf = 0;  // padding tokens (n <= tk < N) get zero codes and scales
            if (tk < ti.n) sf = nvfp4_block16(x, hg, &lo, &hi);
            *reinterpret_cast<uint2 *>(p.h_codes + row * (p.I / 2) + kb * 8) = make_uint2(lo, hi);
            p.h_sf[sf_tiled_offset(row, kb, p.I / 64)] = (uint8_t)sf;
            if (p.h_dump && tk < ti.n) {
              float4 *d = reinterpret_cast<float4 *>(p.h_dump + row * p.I + kb * 16);
#pragma unroll
              for (int i = 0; i < 4; ++i) d[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
            }
          }
        }
      } else {
        const float alpha = __fmul_rn(p.h_g[ti.e], p.w_g[ti.e]);
        const int o = ti.m * 256 + (int)rank * 128 + q * 32 + lane;  // output feature of this lane
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col0 = half * 128 + c * 32;
          if (col0 >= ti.n) break;
          const int tk = col0 + lane;
          float sc = alpha;
          if (p.topk_w && tk < ti.n) sc = __fmul_rn(alpha, p.topk_w[p.perm[ti.out_row0 + tk]]);
          const int nv = min(32, ti.n - col0);
          float *dst = p.y + (int64_t)(ti.out_row0 + col0) * p.H + o;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float s = __shfl_sync(0xffffffffu, sc, i);
            if (i < nv) dst[(int64_t)i * p.H] = __fmul_rn(v[32 * c + i], s);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the pair's MMAs, copies and TMEM reads are over in both CTAs
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// Largest number of co-resident CTA pairs for a kernel and shared-memory
// size, cached per device.
template <int EPI>
int max_pairs(int smem) {
  static std::mutex mu;
  static int cached_dev[16] = {-1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1};
  static int cached_smem[16], cached_val[16];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  std::lock_guard<std::mutex> g(mu);
  const int slot = dev & 15;
  if (cached_dev[slot] == dev && cached_smem[slot] == smem) return cached_val[slot];
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, moe_pair_kernel<EPI>, &cfg) != cudaSuccess) n = 0;
  n = n < sm_count() / 2 ? n : sm_count() / 2;
  cached_dev[slot] = dev;
  cached_smem[slot] = smem;
  cached_val[slot] = n;
  return n;
}

template <int EPI>
fp4_status launch_pair(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tsa, const CUtensorMap &tsb,
                       const PairParams &p, cudaStream_t s) {
  const int smem = smem_bytes(EPI, p.E);
  if (smem > 232448) return FP4_ERR_UNSUPPORTED_SHAPE;
  FP4_HOST_CHECK(cudaFuncSetAttribute(moe_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const int pairs = max_pairs<EPI>(smem);
  if (pairs < 1) return FP4_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  FP4_HOST_CHECK(cudaLaunchKernelEx(&cfg, moe_pair_kernel<EPI>, ta, tb, tsa, tsb, p));
  return FP4_OK;
}

}  // namespace

fp4_status moe_pair_w13(const uint8_t *a_codes, const uint8_t *a_sf, const float *a_g, const fp4_moe_weights *w,
                        int64_t H, int64_t I, int32_t E, const int32_t *counts, const int32_t *tile_offsets,
                        int64_t rows_cap, uint8_t *h_codes, uint8_t *h_sf, float *h_dump, cudaStream_t stream) {
  const DeviceCtx *ctx = device_ctx();
  if (!ctx) return FP4_ERR_CUDA;
  const uint64_t cap_pad = (uint64_t)((rows_cap + 127) / 128) * 128;
  CUtensorMap ta, tb, tsa, tsb;
  if (!make_code_map(&ta, w->w13_codes, (uint64_t)E * 2 * I, (uint64_t)H / 2, 128)) return FP4_ERR_CUDA;
  if (!make_code_map(&tb, a_codes, (uint64_t)rows_cap, (uint64_t)H / 2, B_BOX_ROWS)) return FP4_ERR_CUDA;
  if (!make_sf_map(&tsa, w->w13_sf, (uint64_t)E * 2 * I * (uint64_t)(H / 16))) return FP4_ERR_CUDA;
  if (!make_sf_map(&tsb, a_sf, cap_pad * (uint64_t)(H / 16))) return FP4_ERR_CUDA;
  PairParams p = {};
  p.E = E;
  p.MT = (int)(2 * I / 256);
  p.w_rows = (int)(2 * I);
  p.k_stages = (int)(H / 256);
  p.kw = (int)(H / 64);
  p.counts = counts;
  p.tile_offsets = tile_offsets;
  p.offsets = nullptr;
  p.a_g = a_g;
  p.w_g = w->w13_g;
  p.h_g = w->h_g;
  p.h_codes = h_codes;
  p.h_sf = h_sf;
  p.h_dump = h_dump;
  p.I = (int)I;
  p.H = (int)H;
  p.status = ctx->status;
  p.wait_limit = ctx->wait_limit_ns;
  return launch_pair<PAIR_W13>(ta, tb, tsa, tsb, p, stream);
}

fp4_status moe_pair_w2(const uint8_t *h_codes, const uint8_t *h_sf, const fp4_moe_weights *w, int64_t H, int64_t I,
                       int32_t E, const int32_t *counts, const int32_t *offsets, const int32_t *tile_offsets,
                       const int32_t *perm, const float *topk_weights, int64_t rows_cap, float *y,
                       cudaStream_t stream) {
  const DeviceCtx *ctx = device_ctx();
  if (!ctx) return FP4_ERR_CUDA;
  const uint64_t cap_pad = (uint64_t)((rows_cap + 127) / 128) * 128;
  CUtensorMap ta, tb, tsa, tsb;
  if (!make_code_map(&ta, w->w2_codes, (uint64_t)E * H, (uint64_t)I / 2, 128)) return FP4_ERR_CUDA;
  if (!make_code_map(&tb, h_codes, (uint64_t)rows_cap, (uint64_t)I / 2, B_BOX_ROWS)) return FP4_ERR_CUDA;
  if (!make_sf_map(&tsa, w->w2_sf, (uint64_t)E * H * (uint64_t)(I / 16))) return FP4_ERR_CUDA;
  if (!make_sf_map(&tsb, h_sf, cap_pad * (uint64_t)(I / 16))) return FP4_ERR_CUDA;
  PairParams p = {};
  p.E = E;
  p.MT = (int)(H / 256);
  p.w_rows = (int)H;
  p.k_stages = (int)(I / 256);
  p.kw = (int)(I / 64);
  p.counts = counts;
  p.offsets = offsets;
  p.tile_offsets = tile_offsets;
  p.w_g = w->w2_g;
  p.h_g = w->h_g;
  p.I = (int)I;
  p.H = (int)H;
  p.perm = perm;
  p.topk_w = topk_weights;
  p.y = y;
  p.status = ctx->status;
  p.wait_limit = ctx->wait_limit_ns;
  return launch_pair<PAIR_W2>(ta, tb, tsa, tsb, p, stream);
}

}  // namespace fp4
