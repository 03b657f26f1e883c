// tcgen05 split-KV latent attention for MLA with at most 32 heads (sm_100a).
//
// Method: yololab.net, "超越 GQA 的推理革命…", section "矩陣吸收": with W_UK
// folded into the query, every head scores the cached latent c_KV directly,
// plus the decoupled RoPE key (section "2. 解耦旋轉位置編碼"), and the value
// side is the same latent, so all heads of a sequence share one cache tile:
//   S[h, t] = q_lat[h] . c[t] + q_rot[h] . k[t]      (QK^T, K = 512 + 64)
//   O[h, :] += softmax_t(scale * S)[h, t] . c[t, :]  (PV, over the 512 dims)
//
// Design (B200, H <= 32), next to the full-head kernel of attn_tc.cu:
//   * A worker is a pair of CTAs (a cluster of 2).  CTA r owns latent dims
//     [256r, 256r + 256) and rope dims [32r, 32r + 32) of every page.
//   * The query (this CTA's 288 dims) lives in TMEM, copied into all four
//     32-lane quarters: lane 32q + h holds head h.  QK^T (M = 128, N = 64
//     tokens, A from TMEM) then leaves every head's scores in every lane
//     quarter, so the four softmax warps (one per quarter) each take the
//     16-token slice q of all heads: 16 scores per thread instead of 64.
//   * The exchange warp of quarter q sends slice q of this CTA's partial
//     scores to the peer as fp32 (64 bytes per thread, two buffers deep).
//     Both CTAs add the same two fp32 partials (in the other order), so they
//     hold the same bits and no score is rounded on the way.
//   * The slice warps agree on each page's row maximum through shared memory
//     (one mbarrier per page), take the rare rescale factors of all heads from
//     each other's lanes by shuffle, and write P (bf16) into a shared-memory
//     P^T tile.
//   * PV runs with the operands swapped: O^T[dims, heads] += C^T . P^T, with
//     M = 128 latent dims (the cache tile read MN-major), N = 32 heads and
//     K = 64 tokens; O^T takes 64 TMEM columns.
//   * QK^T and PV are issued by two warps: issuing a page's 18 QK^T MMAs
//     blocks behind the in-order tensor pipe for most of a microsecond, and a
//     PV whose P is ready must not wait behind it (the PV frees the stage the
//     next load needs).  The two write disjoint TMEM, and PV(g) cannot start
//     before QK^T(g) has completed (it needs P(g)), so a stage is free once
//     PV(g) completes.
//   * No query in shared memory, so the stage ring holds five pages of 36 KB
//     (four 64-dim latent blocks and the CTA's 32-dim rope block).  The
//     producer streams pages across sequence changes; the exchange warps load
//     each piece's query into TMEM once its previous query is no longer read.
//   * Rows past the sequence end in the last page are zeroed in shared memory
//     before the MMAs read them (a NaN there would poison P.V even at P = 0).
//   * Every wait is bounded; a wait that runs out sets the CTA's abort flag and
//     records MLRA_ERR_TIMEOUT with its site, and every role then leaves.
// The split plan and the partial-result layout are those of the other
// attention kernels (slot c + b, running max in log2 units, o_part[slot][H][d_c]).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "attn_common.cuh"
#include "attn_tc.h"
#include "host_cache.h"
#include "ptx.cuh"

namespace mlra {
namespace {

using namespace ptx;

// warp 0 TMA, warp 1 QK^T issue, warps 2-5 softmax, warps 6-9 exchange, warp 10 PV issue
constexpr int kSmThreads = 352;
constexpr int kSmSB = 4;                 // S buffers (TMEM) and P^T buffers (shared memory)
constexpr int kSmLat = 4;                // 64-dim latent blocks of this CTA's 256 dims
constexpr int kSmSlot = 64 * 128;        // 64 tokens x 64 bf16, 128-byte swizzle
constexpr int kSmRope = 64 * 64;         // 64 tokens x 32 bf16, 64-byte swizzle
constexpr int kSmStage = kSmLat * kSmSlot + kSmRope;  // one page: 36 KB
constexpr int kSmX = 4 * 32 * 64;        // one page of the peer's partial scores (fp32)
constexpr int kSmP = 32 * 128;           // P^T of one page: 32 heads x 64 tokens bf16
constexpr int kSmMaxStages = 6;
constexpr uint32_t kSmTmemCols = 512;
// TMEM columns: O^T (two accumulators of 32 heads: dims 0-127 and 128-255 of
// this CTA), the S ring, the query's latent half (256 bf16 = 128 columns) and
// rope half (32 bf16 = 16 columns)
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 64;
constexpr uint32_t kColQ = kColS + 64 * kSmSB;
constexpr uint32_t kColQR = kColQ + 128;
static_assert(kColQR + 16 <= kSmTmemCols, "TMEM columns");

struct SmBars {
  uint64_t stage_full[kSmMaxStages], stage_empty[kSmMaxStages];
  uint64_t s_full[kSmSB], s_free[kSmSB], p_full[kSmSB], pv_done[kSmSB];
  uint64_t q_full, q_empty, o_free;
  uint64_t x_full[2][4], x_empty[2][4];  // exchange buffers, per lane quarter
  uint64_t red_full[2], l_full;
  float red[2][4][32];  // per-page maxima of each slice
  float lsum[4][32];    // per-slice softmax sums at the end of a piece
  WorkerPlan plan;
  int page_ids[kIdRing];
  uint32_t tmem_base;
  int abort_flag;
};

// Shared memory: [exchange buffers 2 x 8 KB][P^T buffers 4 x 4 KB][stages][barriers]
struct SmLayout {
  static constexpr int kCap = 232448;
  static constexpr int kX = 0;
  static constexpr int kP = kX + 2 * kSmX;
  static constexpr int kTile = kP + kSmSB * kSmP;
  static constexpr int kFixed = kTile + (int)sizeof(SmBars) + 1024;  // + alignment slack
  static constexpr int kStages = (kCap - kFixed) / kSmStage < kSmMaxStages ? (kCap - kFixed) / kSmStage
                                                                            : kSmMaxStages;
  static constexpr int kBars = kTile + kStages * kSmStage;
  static constexpr int kBytes = kBars + (int)sizeof(SmBars) + 1024;
  static_assert(kP % 1024 == 0 && kTile % 1024 == 0 && kSmStage % 1024 == 0, "swizzle atoms stay aligned");
  static_assert(kStages >= 3 && kBytes <= kCap, "shared memory");
};

// Optional pipeline trace (builds with -DMLRA_TRACE only): globaltimer stamps
// of each role's events for the first kSmTracePages pages of CTAs 0 and 1.
#ifdef MLRA_TRACE
constexpr int kSmTracePages = 64;
constexpr int kSmTraceEvents = 16;
__device__ unsigned long long g_strace[2][kSmTracePages][kSmTraceEvents];
enum { kTvTma = 0, kTvStageSeen, kTvQkIssued, kTvXLoaded, kTvXSent, kTvSLoaded, kTvXRecv, kTvRedDone, kTvPReady,
       kTvPSeen, kTvPvIssued, kTvStageFree, kTvQLoaded, kTvEpilogue };
#define SM_TRACE(gg, ev)                                                                                   \
  do {                                                                                                     \
    if (blockIdx.x < 2 && (gg) < (uint32_t)kSmTracePages) g_strace[blockIdx.x][gg][ev] = globaltimer_ns(); \
  } while (0)
#else
#define SM_TRACE(gg, ev) \
  do {                   \
  } while (0)
#endif

enum { kSiteQEmpty = 1, kSiteStageEmpty, kSiteQFull, kSiteMma, kSiteOFree, kSiteSFull, kSiteXEmpty, kSiteXFull,
       kSitePvDone, kSiteRed, kSiteL, kSitePFull };

// This piece's query rows into TMEM lanes 32q + h (h = lane, the head), by one
// warp of lane quarter q: the CTA's 256 latent dims as 128 packed bf16x2
// columns and its 32 rope dims as 16 (the layout a TMEM A operand takes).
// Heads >= H get zero rows.
__device__ __forceinline__ void load_query(uint32_t taddr_q, uint32_t taddr_qr, const __nv_bfloat16* q_ws, int b,
                                           const AttnArgs& a, uint32_t rank) {
  const int lane = threadIdx.x & 31;
  const bool real = lane < a.H;
  const __nv_bfloat16* src = q_ws + ((size_t)b * a.H + (real ? lane : 0)) * (a.d_c + a.d_r);
  const uint4* lat = reinterpret_cast<const uint4*>(src + 256 * rank);
  const uint4* rop = reinterpret_cast<const uint4*>(src + a.d_c + 32 * rank);
  const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int half = 0; half < 2; ++half) {  // two rounds of 16 loads (64 columns each)
    uint4 u[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) u[i] = real ? __ldg(lat + 16 * half + i) : z;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t r[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        r[4 * i] = u[8 * c + i].x;
        r[4 * i + 1] = u[8 * c + i].y;
        r[4 * i + 2] = u[8 * c + i].z;
        r[4 * i + 3] = u[8 * c + i].w;
      }
      tmem_st32(taddr_q + (uint32_t)(64 * half + 32 * c), r);
    }
  }
  uint32_t r[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = real ? __ldg(rop + i) : z;
    r[4 * i] = v.x;
    r[4 * i + 1] = v.y;
    r[4 * i + 2] = v.z;
    r[4 * i + 3] = v.w;
  }
  tmem_st16(taddr_qr, r);
}

__global__ void __launch_bounds__(kSmThreads, 1)
    attend_tc_small_kernel(const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_rope,
                           const __nv_bfloat16* __restrict__ q_ws, const int* __restrict__ page_table,
                           const int* __restrict__ seq_lens, float* __restrict__ o_part,
                           float* __restrict__ ml_part, int* __restrict__ err, AttnArgs a) {
  using L = SmLayout;
  constexpr int kStages = L::kStages;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 32, true, false);  // A = tile read MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sX = reinterpret_cast<float*>(smem + L::kX);
  uint8_t* sP = smem + L::kP;
  uint8_t* sTile = smem + L::kTile;
  SmBars* bars = reinterpret_cast<SmBars*>(smem + L::kBars);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dep_launch();  // the combine kernel may set up (and load its weights) as this grid retires
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int c = blockIdx.x / 2;
  const int maxL = a.maxp * kPage;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bars->stage_full[s]), 1);
      mbar_init(smem_u32(&bars->stage_empty[s]), 1);
    }
    for (int k = 0; k < kSmSB; ++k) {
      mbar_init(smem_u32(&bars->s_full[k]), 1);
      mbar_init(smem_u32(&bars->s_free[k]), 8);  // the four softmax and four exchange warps read S
      mbar_init(smem_u32(&bars->p_full[k]), 4);
      mbar_init(smem_u32(&bars->pv_done[k]), 1);
    }
    mbar_init(smem_u32(&bars->q_full), 4);
    mbar_init(smem_u32(&bars->q_empty), 1);
    mbar_init(smem_u32(&bars->o_free), 4);
    for (int b = 0; b < 2; ++b)
      for (int q = 0; q < 4; ++q) {
        mbar_init(smem_u32(&bars->x_full[b][q]), 1);
        mbar_init(smem_u32(&bars->x_empty[b][q]), 1);
      }
    mbar_init(smem_u32(&bars->red_full[0]), 4);
    mbar_init(smem_u32(&bars->red_full[1]), 4);
    mbar_init(smem_u32(&bars->l_full), 4);
    // the peer's scores of pages 0 and 1 are expected in phase 0 of the two buffers
    for (int b = 0; b < 2; ++b)
      for (int q = 0; q < 4; ++q) mbar_expect_tx(smem_u32(&bars->x_full[b][q]), 32u * 64u);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kSmTmemCols);
    tmem_relinquish();
  }
  if (warp == 0) {
    WorkerPlan p = plan_worker(seq_lens, a.B, a.G, c, maxL);
    if (lane == 0) bars->plan = p;
  }
  if (warp == 2 && c == 0 && rank == 0) {
    for (int b = lane; b < a.B; b += 32) {
      const int Lb = __ldg(seq_lens + b);
      if (Lb < 0 || Lb > maxL) report_error(err, kErrDeviceCheck, b, Lb);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // the peer's barriers exist before anyone arrives on them
  const uint32_t tmem = bars->tmem_base;
  const WorkerPlan plan = bars->plan;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    // Pages stream through the stage ring in walk order, across pieces (the
    // cache does not depend on the query).  Page ids are read kIdAhead pages
    // before their tile and parked in a small ring.
    IdFetch ids(plan, a.B, maxL, seq_lens);
    {
      int my_b = -1, my_p = 0;
      for (int k = 0; k < kIdAhead && ids.live; ++k) {
        if (lane == k) {
          my_b = ids.w.b;
          my_p = ids.p;
        }
        ids.step(seq_lens);
      }
      if (my_b >= 0) bars->page_ids[lane] = __ldg(page_table + (size_t)my_b * a.maxp + my_p);
      __syncwarp();
    }
    if (lane == 0) {
      tma_prefetch_desc(&tm_lat);
      tma_prefetch_desc(&tm_rope);
      SegWalk walk(plan, a.B, maxL);
      int* id_ring = bars->page_ids;
      int pend = 0;
      bool has_pend = false;
      uint32_t g = 0;
      bool ok = true;
      while (ok && walk.next(seq_lens)) {
        for (int p = walk.pg0; p < walk.pg1; ++p, ++g) {
          if (has_pend) id_ring[(g - 1 + kIdAhead) % kIdRing] = pend;
          has_pend = ids.live;
          if (has_pend) pend = ids.fetch(seq_lens, page_table, a.maxp);  // the id of page g + kIdAhead
          const uint32_t st = g % kStages, use = g / kStages;
          if (use > 0 && !mbar_wait(smem_u32(&bars->stage_empty[st]), (use - 1) & 1, abort_flag, err,
                                    kSiteStageEmpty)) {
            ok = false;
            break;
          }
          SM_TRACE(g, kTvStageFree);
          int pg = id_ring[g % kIdRing];
          if (pg < 0 || pg >= a.num_pages) {  // reported, and replaced by page 0 so that no load leaves the pool
            report_error(err, kErrDeviceCheck, walk.b, p * kPage);
            pg = 0;
          }
          const uint32_t fb = smem_u32(&bars->stage_full[st]);
          uint8_t* tile = sTile + st * kSmStage;
          mbar_expect_tx(fb, kSmStage);
          for (int s = 0; s < kSmLat; ++s)
            tma_load_2d(smem_u32(tile + s * kSmSlot), &tm_lat, fb, 64 * (kSmLat * (int)rank + s), pg * kPage);
          tma_load_2d(smem_u32(tile + kSmLat * kSmSlot), &tm_rope, fb, 32 * (int)rank, pg * kPage);
          SM_TRACE(g, kTvTma);
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- QK^T
    // QK^T of every page in walk order, as soon as it has landed and its S
    // buffer has been read out (by the four softmax and four exchange warps).
    SegWalk walk(plan, a.B, maxL);
    int seg = 0;
    uint32_t g = 0;
    bool ok = true;
    while (ok && walk.next(seq_lens)) {
      if (!mbar_wait_warp(smem_u32(&bars->q_full), seg & 1, abort_flag, err, kSiteQFull)) break;
      tc_fence_after();
      const uint32_t g0 = g, g_end = g + (uint32_t)(walk.pg1 - walk.pg0);
      for (; g < g_end; ++g) {
        const uint32_t st = g % kStages;
        if (!mbar_wait_warp(smem_u32(&bars->stage_full[st]), (g / kStages) & 1, abort_flag, err, kSiteMma) ||
            (g >= (uint32_t)kSmSB && !mbar_wait_warp(smem_u32(&bars->s_free[g % kSmSB]), ((g / kSmSB) - 1) & 1,
                                                      abort_flag, err, kSiteSFull))) {
          ok = false;
          break;
        }
        SM_TRACE(g, kTvStageSeen);
        uint8_t* tile = sTile + st * kSmStage;
        const int p = walk.pg0 + (int)(g - g0);
        const int valid = min(kPage, walk.L - p * kPage);
        if (valid < kPage) {  // zero the rows past the end of the sequence
          const int nrow = kPage - valid;
          const uint4 z = make_uint4(0, 0, 0, 0);
          for (int idx = lane; idx < nrow * 8 * kSmLat; idx += 32) {
            const int s2 = idx / (nrow * 8), rem = idx % (nrow * 8);
            *reinterpret_cast<uint4*>(tile + s2 * kSmSlot + (valid + rem / 8) * 128 + (rem % 8) * 16) = z;
          }
          for (int idx = lane; idx < nrow * 4; idx += 32)
            *reinterpret_cast<uint4*>(tile + kSmLat * kSmSlot + (valid + idx / 4) * 64 + (idx % 4) * 16) = z;
          fence_proxy_async_smem();
        }
        __syncwarp();
        tc_fence_after();
        if (lane == 0) {
          const uint64_t td = sdesc_sw128(smem_u32(tile), 16, 1024);
          const uint32_t s_col = tmem + kColS + (g % kSmSB) * 64u;
#pragma unroll
          for (int s2 = 0; s2 < kSmLat; ++s2)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_ts(s_col, tmem + kColQ + 32u * s2 + 8u * ks, td + (uint64_t)((s2 * kSmSlot + ks * 32) >> 4),
                     kIdescQK, (s2 | ks) ? 1u : 0u);
          const uint64_t rd = sdesc_sw64(smem_u32(tile + kSmLat * kSmSlot), 512);
#pragma unroll
          for (int ks = 0; ks < 2; ++ks)
            mma_ts(s_col, tmem + kColQR + 8u * ks, rd + (uint64_t)(ks * 2), kIdescQK, 1u);
          mma_commit(smem_u32(&bars->s_full[g % kSmSB]));
          if (g + 1 == g_end) mma_commit(smem_u32(&bars->q_empty));  // the last read of this query
          SM_TRACE(g, kTvQkIssued);
        }
        __syncwarp();
      }
      ++seg;
    }
  } else if (warp == 10) {
    // ----------------------------------------------------------------- PV
    // PV of every page in walk order, as soon as its P^T is written; the
    // commit frees the page's stage and P^T buffer.
    SegWalk walk(plan, a.B, maxL);
    int seg = 0;
    uint32_t g = 0;
    bool ok = true;
    while (ok && walk.next(seq_lens)) {
      // the previous piece's O^T must be read out before the first PV overwrites it
      if (seg > 0 && !mbar_wait_warp(smem_u32(&bars->o_free), (seg - 1) & 1, abort_flag, err, kSiteOFree)) break;
      const uint32_t g0 = g, g_end = g + (uint32_t)(walk.pg1 - walk.pg0);
      for (; g < g_end; ++g) {
        if (!mbar_wait_warp(smem_u32(&bars->p_full[g % kSmSB]), (g / kSmSB) & 1, abort_flag, err, kSitePFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          SM_TRACE(g, kTvPSeen);
          const uint32_t first = g == g0 ? 1u : 0u;
          uint8_t* tile = sTile + (g % kStages) * kSmStage;
          const uint64_t pd = sdesc_sw128(smem_u32(sP + (g % kSmSB) * kSmP), 16, 1024);
#pragma unroll
          for (int acc = 0; acc < 2; ++acc) {
            // A = latent dims [128 acc, +128) of the page (two 64-dim blocks), MN-major
            const uint64_t vd = sdesc_sw128(smem_u32(tile + 2 * acc * kSmSlot), 8192, 1024);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_ss(tmem + kColO + 32u * acc, vd + (uint64_t)((ks * 2048) >> 4), pd + (uint64_t)(ks * 2), kIdescPV,
                     ks == 0 ? (first ^ 1u) : 1u);
          }
          mma_commit(smem_u32(&bars->stage_empty[g % kStages]));
          mma_commit(smem_u32(&bars->pv_done[g % kSmSB]));
          SM_TRACE(g, kTvPvIssued);
        }
        __syncwarp();
      }
      ++seg;
    }
  } else if (warp >= 6) {  // warps 6-9 (warp 10 is handled above)
    // ------------------------------------------------------------- exchange
    // Quarter q: loads each piece's query into its TMEM lane quarter, then
    // sends slice q (16 tokens) of this CTA's partial scores of every page to
    // the peer, fp32, as soon as QK^T has produced them.
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t xdst = map_to_cta(smem_u32(sX), peer);
    grid_dep_wait();  // the absorbed queries come from the previous kernel
    SegWalk walk(plan, a.B, maxL);
    uint32_t g = 0;
    int seg = 0;
    bool ok = true;
    while (ok && walk.next(seq_lens)) {
      if (seg > 0 && !mbar_wait_warp(smem_u32(&bars->q_empty), (seg - 1) & 1, abort_flag, err, kSiteQEmpty)) break;
      tc_fence_after();
      load_query(tmem + lane_off + kColQ, tmem + lane_off + kColQR, q_ws, walk.b, a, rank);
      if (q == 0 && lane == 0) SM_TRACE(g, kTvQLoaded);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->q_full));
      for (int p = walk.pg0; p < walk.pg1; ++p, ++g) {
        if (!mbar_wait_warp(smem_u32(&bars->s_full[g % kSmSB]), (g / kSmSB) & 1, abort_flag, err, kSiteSFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[16];
        tmem_ld16(tmem + lane_off + kColS + (g % kSmSB) * 64u + 16u * q, v);
        if (q == 0 && lane == 0) SM_TRACE(g, kTvXLoaded);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[g % kSmSB]));
        const int buf = g & 1;
        // the peer's slice warp has consumed what this buffer held (page g - 2)
        if (g >= 2 && !mbar_wait_warp<true>(smem_u32(&bars->x_empty[buf][q]), ((g >> 1) - 1) & 1, abort_flag, err,
                                            kSiteXEmpty)) {
          ok = false;
          break;
        }
        const uint32_t xbar = map_to_cta(smem_u32(&bars->x_full[buf][q]), peer);
        const uint32_t dst = xdst + (uint32_t)(buf * kSmX);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          st_async_v4(dst + (uint32_t)(((q * 4 + ch) * 32 + lane) * 16), v[4 * ch], v[4 * ch + 1], v[4 * ch + 2],
                      v[4 * ch + 3], xbar);
        if (q == 0 && lane == 0) SM_TRACE(g, kTvXSent);
      }
      ++seg;
    }
  } else {
    // -------------------------------------------------------------- softmax
    // Quarter q: tokens [16q, 16q + 16) of every head (lane = head).
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const bool real = lane < a.H;
    const float4* xin = reinterpret_cast<const float4*>(sX);
    SegWalk walk(plan, a.B, maxL);
    uint32_t g = 0;
    int seg = 0;
    bool ok = true;
    while (ok && walk.next(seq_lens)) {
      const uint32_t g0 = g, g_end = g + (uint32_t)(walk.pg1 - walk.pg0);
      float m_run = -INFINITY, l_run = 0.f;
      for (; g < g_end; ++g) {
        const int valid = min(kPage, walk.L - (walk.pg0 + (int)(g - g0)) * kPage);
        if (!mbar_wait_warp(smem_u32(&bars->s_full[g % kSmSB]), (g / kSmSB) & 1, abort_flag, err, kSiteSFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[16];
        tmem_ld16(tmem + lane_off + kColS + (g % kSmSB) * 64u + 16u * q, v);
        if (q == 0 && lane == 0) SM_TRACE(g, kTvSLoaded);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[g % kSmSB]));
        const int buf = g & 1;
        if (!mbar_wait_warp<true>(smem_u32(&bars->x_full[buf][q]), (g >> 1) & 1, abort_flag, err, kSiteXFull)) {
          ok = false;
          break;
        }
        if (q == 0 && lane == 0) SM_TRACE(g, kTvXRecv);
        // s = own partial + peer's partial, fp32: the same two operands on both CTAs
        float s[16];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const float4 t = xin[buf * (kSmX / 16) + (q * 4 + ch) * 32 + lane];
          s[4 * ch] = __uint_as_float(v[4 * ch]) + t.x;
          s[4 * ch + 1] = __uint_as_float(v[4 * ch + 1]) + t.y;
          s[4 * ch + 2] = __uint_as_float(v[4 * ch + 2]) + t.z;
          s[4 * ch + 3] = __uint_as_float(v[4 * ch + 3]) + t.w;
        }
        __syncwarp();
        if (lane == 0) {  // buffer consumed: arm its next phase (page g + 2), hand it back to the peer
          mbar_expect_tx(smem_u32(&bars->x_full[buf][q]), 32u * 64u);
          mbar_arrive_cluster(map_to_cta(smem_u32(&bars->x_empty[buf][q]), peer));
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (16 * q + i >= valid) s[i] = -INFINITY;
        float m4[4];
#pragma unroll
        for (int i = 0; i < 16; ++i) m4[i & 3] = i < 4 ? s[i] : fmaxf(m4[i & 3], s[i]);
        bars->red[buf][q][lane] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->red_full[buf]));
        if (!mbar_wait_warp(smem_u32(&bars->red_full[buf]), (g >> 1) & 1, abort_flag, err, kSiteRed)) {
          ok = false;
          break;
        }
        if (q == 0 && lane == 0) SM_TRACE(g, kTvRedDone);
        // the page's row maximum (at least one token of a page is valid, so it is finite)
        const float M = fmaxf(fmaxf(bars->red[buf][0][lane], bars->red[buf][1][lane]),
                              fmaxf(bars->red[buf][2][lane], bars->red[buf][3][lane]));
        float m_use, corr;
        bool rescale = false;
        if (g == g0) {
          m_use = M;
          corr = 0.f;
        } else if (M > m_run + kRescaleLog2) {
          m_use = M;
          corr = ex2(m_run - M);
          rescale = true;
        } else {
          m_use = m_run;
          corr = 1.f;
        }
        float pv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pv[i] = ex2(s[i] - m_use);
        const float sum = (((pv[0] + pv[1]) + (pv[2] + pv[3])) + ((pv[4] + pv[5]) + (pv[6] + pv[7]))) +
                          (((pv[8] + pv[9]) + (pv[10] + pv[11])) + ((pv[12] + pv[13]) + (pv[14] + pv[15])));
        l_run = l_run * corr + sum;
        m_run = m_use;
        // O^T columns are heads: every lane of this warp needs every head's factor
        // (all four warps decide the same, from the same maxima)
        if (__any_sync(0xffffffffu, rescale)) {
          if (!mbar_wait_warp(smem_u32(&bars->pv_done[(g - 1) % kSmSB]), ((g - 1) / kSmSB) & 1, abort_flag, err,
                              kSitePvDone)) {
            ok = false;
            break;
          }
          tc_fence_after();
          float cf[32];
#pragma unroll
          for (int h = 0; h < 32; ++h) cf[h] = __shfl_sync(0xffffffffu, corr, h);
#pragma unroll
          for (int acc = 0; acc < 2; ++acc) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + kColO + 32u * acc, o);
#pragma unroll
            for (int h = 0; h < 32; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * cf[h]);
            tmem_st32(tmem + lane_off + kColO + 32u * acc, o);
          }
        }
        // P^T buffer g % kSmSB was last read by PV(g - kSmSB)
        if (g >= (uint32_t)kSmSB && !mbar_wait_warp(smem_u32(&bars->pv_done[g % kSmSB]), ((g / kSmSB) - 1) & 1,
                                                    abort_flag, err, kSitePvDone)) {
          ok = false;
          break;
        }
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = real ? pack_bf16x2(pv[2 * i], pv[2 * i + 1]) : 0u;
        // row = head, tokens [16q, 16q + 16) = 16-byte chunks 2q and 2q + 1 of the 128-byte row
        uint8_t* prow = sP + (g % kSmSB) * kSmP + lane * 128;
        *reinterpret_cast<uint4*>(prow + (((2 * q) ^ (lane & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(prow + (((2 * q + 1) ^ (lane & 7)) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[g % kSmSB]));
        if (q == 0 && lane == 0) SM_TRACE(g, kTvPReady);
      }
      if (!ok) break;
      // epilogue: this quarter's 32 + 32 latent dims of O^T, and (m, l) of the piece
      if (!mbar_wait_warp(smem_u32(&bars->pv_done[(g - 1) % kSmSB]), ((g - 1) / kSmSB) & 1, abort_flag, err,
                          kSitePvDone))
        break;
      tc_fence_after();
      const int slot = c + walk.b;
#pragma unroll
      for (int acc = 0; acc < 2; ++acc) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + kColO + 32u * acc, o);
        float* dst = o_part + (size_t)slot * a.H * a.d_c + 256 * (int)rank + 128 * acc + 32 * q + lane;
#pragma unroll
        for (int h = 0; h < 32; ++h)
          if (h < a.H) dst[(size_t)h * a.d_c] = __uint_as_float(o[h]);
      }
      bars->lsum[q][lane] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->l_full));
      if (!mbar_wait_warp(smem_u32(&bars->l_full), seg & 1, abort_flag, err, kSiteL)) break;
      if (q == 0 && rank == 0 && real) {
        const float l = (bars->lsum[0][lane] + bars->lsum[1][lane]) + (bars->lsum[2][lane] + bars->lsum[3][lane]);
        ml_part[((size_t)slot * 2 + 0) * a.H + lane] = m_run;
        ml_part[((size_t)slot * 2 + 1) * a.H + lane] = l;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->o_free));
      ++seg;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kSmTmemCols);
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
}

}  // namespace

#ifdef MLRA_TRACE
// Copies the pipeline trace of the last small-head attention launch (trace builds only).
extern "C" __attribute__((visibility("default"))) int mlra_small_trace_read(unsigned long long* host, size_t n) {
  const size_t bytes =
      sizeof(g_strace) < n * sizeof(unsigned long long) ? sizeof(g_strace) : n * sizeof(unsigned long long);
  return (int)cudaMemcpyFromSymbol(host, g_strace, bytes);
}
#endif

bool tc_small_supported(int H, int n_branch) { return n_branch == 1 && H >= 1 && H <= 32; }

cudaError_t launch_attend_tc_small(const void* q_ws, const void* lat, const void* rop, const int* page_table,
                                   const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                                   cudaStream_t st, bool pdl) {
  if (!tc_small_supported(a.H, a.n_branch) || a.d_c != 512 || a.d_r != 64) return cudaErrorInvalidValue;
  CUtensorMap tl, tr;
  if (!tmap_2d(&tl, lat, (uint64_t)a.d_c, (uint64_t)a.num_pages * kPage, 64, 64) ||
      !tmap_2d_sw64(&tr, rop, (uint64_t)a.d_r, (uint64_t)a.num_pages * kPage, 32, 64))
    return cudaErrorInvalidValue;
  auto kern = attend_tc_small_kernel;
  const int smem = SmLayout::kBytes;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.G, 1, 1);
  cfg.blockDim = dim3(kSmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, tl, tr, static_cast<const __nv_bfloat16*>(q_ws), page_table, seq_lens, o_part,
                            ml_part, err, a);
}

}  // namespace mlra
