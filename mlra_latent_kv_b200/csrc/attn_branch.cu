// tcgen05 split-KV latent attention, one 128-dim branch per CTA (sm_100a):
// the one-branch (MLA) decode of a 128-dim latent that each rank of a
// branch-parallel MLRA group runs (see tc_branch_supported for why MLRA-4 over
// a 512-dim latent is sent to the four-CTA layout instead).
//
// Method: wispaper.ai, "MLRA：突破 MLA 并行瓶颈…", section "2.1 架构拆解":
// each branch br attends with its own softmax over its own block of the
// latent, with the decoupled RoPE score shared by every branch; yololab.net,
// "超越 GQA 的推理革命…", section "矩陣吸收": with W_UK folded into the query
// the scores read the cached latent directly, and the value side is the same
// latent:
//   S_br[h, t] = q_lat_br[h] . c_br[t] + q_rot[h] . k[t]
//   O_br[h, :] += softmax_t(scale * S_br)[h, t] . c_br[t, :]
//
// Design (B200, up to 128 heads):
//   * A CTA takes one branch of one page range; one CTA per SM.  The grid is
//     n_branch x G CTAs: CTA (br, c) attends branch br over worker c's pages.
//   * The branch's query (128 latent dims and the 64 rope dims of every head)
//     lives in TMEM beside O (128 columns) and a ring of four S buffers, so
//     shared memory holds only pages: up to nine stages of 24 KB (the
//     branch's two 64-dim latent blocks and the 64-dim rope block).
//   * QK^T (M = 128 heads, N = 64 tokens, A from TMEM) and PV (A = P in TMEM,
//     B = the page's latent read MN-major, N = 128) are issued by two warps,
//     so a PV whose P is ready never waits behind the next page's QK^T issue.
//   * Four softmax warps per TMEM lane quarter split each page's 64 tokens in
//     16-token slices: 16 scores per thread, and four warps per SM
//     sub-partition to hide each other's latency.  The four agree on each
//     page's row maximum through shared memory (an mbarrier per lane quarter
//     and page), write their slices of P (bf16) over S, and share the rare O
//     rescale.
//   * Four query warps load each piece's query into TMEM once the previous
//     piece's last QK^T has completed.
//   * Rows past the sequence end in the last page are zeroed in shared memory
//     before the MMAs read them (a NaN there would poison P.V even at P = 0).
//   * Every wait is bounded; a wait that runs out sets the CTA's abort flag and
//     records MLRA_ERR_TIMEOUT with its site, and every role then leaves.
// Partials use the layout of the other attention kernels: slot c + b, o_part
// [slot][H][d_c] (this branch's columns), ml_part[slot][n_branch][2][H] with
// the running max in log2 units.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "attn_common.cuh"
#include "attn_tc.h"
#include "host_cache.h"
#include "ptx.cuh"

namespace mlra {
namespace {

using namespace ptx;

// warp 0 TMA, 1 QK^T issue, 2 PV issue, 3 length checks, 4-19 softmax (token
// slice j = (warp - 4) / 4, lane quarter q = warp % 4), 20-23 query loaders
constexpr int kBrSlices = 4;                          // 16-token slices of a page
constexpr int kBrSliceTok = 64 / kBrSlices;
constexpr int kBrSmxWarps = 4 * kBrSlices;
constexpr int kBrQWarp0 = 4 + kBrSmxWarps;
constexpr int kBrThreads = 32 * (kBrQWarp0 + 4);
constexpr int kBrSB = 4;                  // S buffers
constexpr int kBrSlot = 64 * 128;         // 64 tokens x 64 bf16, 128-byte swizzle
constexpr int kBrStage = 3 * kBrSlot;     // two latent blocks and the rope block of a page: 24 KB
constexpr int kBrMaxStages = 9;
constexpr uint32_t kBrTmemCols = 512;
// TMEM columns: O (128 latent dims), the S ring, the branch's query (128 bf16
// = 64 packed columns) and the rope query (64 bf16 = 32 columns)
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 128;
constexpr uint32_t kColQ = kColS + 64 * kBrSB;
constexpr uint32_t kColQR = kColQ + 64;
static_assert(kColQR + 32 <= kBrTmemCols, "TMEM columns");

struct BrBars {
  uint64_t stage_full[kBrMaxStages], stage_empty[kBrMaxStages];
  uint64_t s_full[kBrSB], p_full[kBrSB], pv_done[kBrSB];
  uint64_t q_full, q_empty, o_free;
  uint64_t red_full[2][4], l_full[4];  // per lane quarter: its slice warps meet
  float red[2][kBrSlices][128];        // [page parity][slice][head] maxima
  float lsum[kBrSlices][128];          // [slice][head] softmax sums at the end of a piece
  WorkerPlan plan;
  int page_ids[kIdRing];
  uint32_t tmem_base;
  int abort_flag;
};

struct BrLayout {
  static constexpr int kCap = 232448;
  static constexpr int kTile = 0;
  static constexpr int kFixed = (int)sizeof(BrBars) + 1024;  // + alignment slack
  static constexpr int kStages = (kCap - kFixed) / kBrStage < kBrMaxStages ? (kCap - kFixed) / kBrStage
                                                                          : kBrMaxStages;
  static constexpr int kBars = kTile + kStages * kBrStage;
  static constexpr int kBytes = kBars + (int)sizeof(BrBars) + 1024;
  static_assert(kBrStage % 1024 == 0, "swizzle atoms stay aligned");
  static_assert(kStages >= 4 && kBytes <= kCap, "shared memory");
};

// Optional pipeline trace (builds with -DMLRA_TRACE only): globaltimer stamps
// of each role's events for the first kBrTracePages pages of CTAs 0 and 1.
#ifdef MLRA_TRACE
constexpr int kBrTracePages = 64;
__device__ unsigned long long g_btrace[2][kBrTracePages][16];
enum { kTbTma = 0, kTbStageSeen, kTbQkIssued, kTbSLoaded, kTbRedDone, kTbPReady, kTbPSeen, kTbPvIssued,
       kTbStageFree, kTbSLoaded1, kTbPReady1 };
#define BR_TRACE(gg, ev)                                                                                   \
  do {                                                                                                     \
    if (blockIdx.x < 2 && (gg) < (uint32_t)kBrTracePages) g_btrace[blockIdx.x][gg][ev] = globaltimer_ns(); \
  } while (0)
#else
#define BR_TRACE(gg, ev) \
  do {                   \
  } while (0)
#endif

enum { kSiteQEmpty = 1, kSiteStageEmpty, kSiteQFull, kSiteMma, kSiteOFree, kSiteSFull, kSitePFull, kSitePvDone,
       kSiteRed, kSiteL };

__global__ void __launch_bounds__(kBrThreads, 1)
    attend_tc_branch_kernel(const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_rope,
                            const __nv_bfloat16* __restrict__ q_ws, const int* __restrict__ page_table,
                            const int* __restrict__ seq_lens, float* __restrict__ o_part,
                            float* __restrict__ ml_part, int* __restrict__ err, AttnArgs a) {
  using L = BrLayout;
  constexpr int kStages = L::kStages;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);  // B = page latent read MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sTile = smem + L::kTile;
  BrBars* bars = reinterpret_cast<BrBars*>(smem + L::kBars);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dep_launch();  // the combine kernel may set up (and load its weights) as this grid retires
  const int br = blockIdx.x / a.G;  // branch
  const int c = blockIdx.x % a.G;   // page-range worker
  const int maxL = a.maxp * kPage;
  const int d_cb = a.d_c / a.n_branch;  // 128

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bars->stage_full[s]), 1);
      mbar_init(smem_u32(&bars->stage_empty[s]), 1);
    }
    for (int k = 0; k < kBrSB; ++k) {
      mbar_init(smem_u32(&bars->s_full[k]), 1);
      mbar_init(smem_u32(&bars->p_full[k]), kBrSmxWarps);  // every slice of every lane quarter
      mbar_init(smem_u32(&bars->pv_done[k]), 1);
    }
    mbar_init(smem_u32(&bars->q_full), 4);
    mbar_init(smem_u32(&bars->q_empty), 1);
    mbar_init(smem_u32(&bars->o_free), kBrSmxWarps);
    for (int q = 0; q < 4; ++q) {
      mbar_init(smem_u32(&bars->red_full[0][q]), kBrSlices);
      mbar_init(smem_u32(&bars->red_full[1][q]), kBrSlices);
      mbar_init(smem_u32(&bars->l_full[q]), kBrSlices);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kBrTmemCols);
    tmem_relinquish();
  }
  if (warp == 0) {
    WorkerPlan p = plan_worker(seq_lens, a.B, a.G, c, maxL);
    if (lane == 0) bars->plan = p;
  }
  if (warp == 3 && blockIdx.x == 0) {
    for (int b = lane; b < a.B; b += 32) {
      const int Lb = __ldg(seq_lens + b);
      if (Lb < 0 || Lb > maxL) report_error(err, kErrDeviceCheck, b, Lb);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
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
          BR_TRACE(g, kTbStageFree);
          int pg = id_ring[g % kIdRing];
          if (pg < 0 || pg >= a.num_pages) {  // reported, and replaced by page 0 so that no load leaves the pool
            report_error(err, kErrDeviceCheck, walk.b, p * kPage);
            pg = 0;
          }
          const uint32_t fb = smem_u32(&bars->stage_full[st]);
          uint8_t* tile = sTile + st * kBrStage;
          mbar_expect_tx(fb, kBrStage);
          tma_load_2d(smem_u32(tile), &tm_lat, fb, d_cb * br, pg * kPage);
          tma_load_2d(smem_u32(tile + kBrSlot), &tm_lat, fb, d_cb * br + 64, pg * kPage);
          tma_load_2d(smem_u32(tile + 2 * kBrSlot), &tm_rope, fb, 0, pg * kPage);
          BR_TRACE(g, kTbTma);
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- QK^T
    // QK^T of every page in walk order, as soon as it has landed and PV has
    // consumed the P written over its S buffer (which implies both softmax
    // halves have read the scores it held).
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
        // S buffer g % kBrSB holds P(g - kBrSB) until PV(g - kBrSB) has completed
        if (!mbar_wait_warp(smem_u32(&bars->stage_full[st]), (g / kStages) & 1, abort_flag, err, kSiteMma) ||
            (g >= (uint32_t)kBrSB && !mbar_wait_warp(smem_u32(&bars->pv_done[g % kBrSB]), ((g / kBrSB) - 1) & 1,
                                                      abort_flag, err, kSitePvDone))) {
          ok = false;
          break;
        }
        if (lane == 0) BR_TRACE(g, kTbStageSeen);
        uint8_t* tile = sTile + st * kBrStage;
        const int p = walk.pg0 + (int)(g - g0);
        const int valid = min(kPage, walk.L - p * kPage);
        if (valid < kPage) {  // zero the rows past the end of the sequence (both latent blocks, rope block)
          const int nrow = kPage - valid;
          const uint4 z = make_uint4(0, 0, 0, 0);
          for (int idx = lane; idx < nrow * 8 * 3; idx += 32) {
            const int s2 = idx / (nrow * 8), rem = idx % (nrow * 8);
            *reinterpret_cast<uint4*>(tile + s2 * kBrSlot + (valid + rem / 8) * 128 + (rem % 8) * 16) = z;
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        tc_fence_after();
        if (lane == 0) {
          const uint64_t td = sdesc_sw128(smem_u32(tile), 16, 1024);
          const uint32_t s_col = tmem + kColS + (g % kBrSB) * 64u;
#pragma unroll
          for (int s2 = 0; s2 < 2; ++s2)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_ts(s_col, tmem + kColQ + 32u * s2 + 8u * ks, td + (uint64_t)((s2 * kBrSlot + ks * 32) >> 4),
                     kIdescQK, (s2 | ks) ? 1u : 0u);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ts(s_col, tmem + kColQR + 8u * ks, td + (uint64_t)((2 * kBrSlot + ks * 32) >> 4), kIdescQK, 1u);
          mma_commit(smem_u32(&bars->s_full[g % kBrSB]));
          if (g + 1 == g_end) mma_commit(smem_u32(&bars->q_empty));  // the last read of this query
          BR_TRACE(g, kTbQkIssued);
        }
        __syncwarp();
      }
      ++seg;
    }
  } else if (warp == 2) {
    // ----------------------------------------------------------------- PV
    // PV of every page in walk order, as soon as every slice of its P is in
    // TMEM; the commits free the page's stage and its S buffer.
    SegWalk walk(plan, a.B, maxL);
    int seg = 0;
    uint32_t g = 0;
    bool ok = true;
    while (ok && walk.next(seq_lens)) {
      // the previous piece's O must be read out before the first PV overwrites it
      if (seg > 0 && !mbar_wait_warp(smem_u32(&bars->o_free), (seg - 1) & 1, abort_flag, err, kSiteOFree)) break;
      const uint32_t g0 = g, g_end = g + (uint32_t)(walk.pg1 - walk.pg0);
      for (; g < g_end; ++g) {
        if (!mbar_wait_warp(smem_u32(&bars->p_full[g % kBrSB]), (g / kBrSB) & 1, abort_flag, err, kSitePFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          BR_TRACE(g, kTbPSeen);
          const uint32_t first = g == g0 ? 1u : 0u;
          const uint64_t vd = sdesc_sw128(smem_u32(sTile + (g % kStages) * kBrStage), 8192, 1024);
          const uint32_t p_base = tmem + kColS + (g % kBrSB) * 64u;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ts(tmem + kColO, p_base + 8u * ks, vd + (uint64_t)((ks * 2048) >> 4), kIdescPV,
                   ks == 0 ? (first ^ 1u) : 1u);
          mma_commit(smem_u32(&bars->stage_empty[g % kStages]));
          mma_commit(smem_u32(&bars->pv_done[g % kBrSB]));
          BR_TRACE(g, kTbPvIssued);
        }
        __syncwarp();
      }
      ++seg;
    }
  } else if (warp >= kBrQWarp0) {
    // -------------------------------------------------------------- query
    // Quarter q: the query rows of heads 32q + lane (this branch's 128 latent
    // dims as 64 packed bf16x2 columns, the 64 rope dims as 32) into TMEM for
    // each piece, once the previous piece's last QK^T has completed.
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int head = q * 32 + lane;
    const bool real = head < a.H;
    grid_dep_wait();  // the absorbed queries come from the previous kernel
    SegWalk walk(plan, a.B, maxL);
    int seg = 0;
    const uint4 z = make_uint4(0, 0, 0, 0);
    while (walk.next(seq_lens)) {
      if (seg > 0 && !mbar_wait_warp(smem_u32(&bars->q_empty), (seg - 1) & 1, abort_flag, err, kSiteQEmpty)) break;
      tc_fence_after();
      const __nv_bfloat16* src = q_ws + ((size_t)walk.b * a.H + (real ? head : 0)) * (a.d_c + a.d_r);
      const uint4* lat = reinterpret_cast<const uint4*>(src + d_cb * br);
      const uint4* rop = reinterpret_cast<const uint4*>(src + a.d_c);
#pragma unroll
      for (int blk = 0; blk < 3; ++blk) {  // latent columns 0-31, 32-63, then the rope's 32
        const uint4* from = blk < 2 ? lat + 8 * blk : rop;
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = real ? __ldg(from + i) : z;
          r[4 * i] = v.x;
          r[4 * i + 1] = v.y;
          r[4 * i + 2] = v.z;
          r[4 * i + 3] = v.w;
        }
        tmem_st32(tmem + lane_off + (blk < 2 ? kColQ + 32u * blk : kColQR), r);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->q_full));
      ++seg;
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax
    // Lane quarter q (heads 32q + lane), token slice j of each page.
    const int q = warp & 3;
    const int j = (warp - 4) >> 2;
    const int head = q * 32 + lane;
    const bool real = head < a.H;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    SegWalk walk(plan, a.B, maxL);
    uint32_t g = 0;
    int seg = 0;
    bool ok = true;
    while (ok && walk.next(seq_lens)) {
      const uint32_t g0 = g, g_end = g + (uint32_t)(walk.pg1 - walk.pg0);
      float m_run = -INFINITY, l_run = 0.f;
      for (; g < g_end; ++g) {
        const int valid = min(kPage, walk.L - (walk.pg0 + (int)(g - g0)) * kPage);
        const uint32_t s_col = kColS + (g % kBrSB) * 64u;
        if (!mbar_wait_warp(smem_u32(&bars->s_full[g % kBrSB]), (g / kBrSB) & 1, abort_flag, err, kSiteSFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[kBrSliceTok];
        {
          uint32_t v[16];
          tmem_ld16(tmem + lane_off + s_col + (uint32_t)(kBrSliceTok * j), v);
#pragma unroll
          for (int i = 0; i < kBrSliceTok; ++i)
            s[i] = kBrSliceTok * j + i < valid ? __uint_as_float(v[i]) : -INFINITY;
        }
        if (q == 0 && lane == 0 && j < 2) BR_TRACE(g, j == 0 ? kTbSLoaded : kTbSLoaded1);
        tc_fence_before();  // the scores are read before the barrier below lets the other slices write P
        float m4[4];
#pragma unroll
        for (int i = 0; i < kBrSliceTok; ++i) m4[i & 3] = i < 4 ? s[i] : fmaxf(m4[i & 3], s[i]);
        const int buf = g & 1;
        bars->red[buf][j][head] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->red_full[buf][q]));
        if (!mbar_wait_warp(smem_u32(&bars->red_full[buf][q]), (g >> 1) & 1, abort_flag, err, kSiteRed)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (q == 0 && j == 0 && lane == 0) BR_TRACE(g, kTbRedDone);
        // the page's row maximum (at least one token of a page is valid, so it is finite); the slices
        // of a quarter read the same four values and decide alike
        const float M = fmaxf(fmaxf(bars->red[buf][0][head], bars->red[buf][1][head]),
                              fmaxf(bars->red[buf][2][head], bars->red[buf][3][head]));
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
        float a4[4];
#pragma unroll
        for (int i = 0; i < kBrSliceTok; ++i) {
          s[i] = ex2(s[i] - m_use);
          a4[i & 3] = i < 4 ? s[i] : a4[i & 3] + s[i];
        }
        l_run = l_run * corr + ((a4[0] + a4[1]) + (a4[2] + a4[3]));
        m_run = m_use;
        // O is rescaled only when the running max jumped; slice j takes columns [32j, 32j + 32)
        if (__any_sync(0xffffffffu, rescale)) {
          if (!mbar_wait_warp(smem_u32(&bars->pv_done[(g - 1) % kBrSB]), ((g - 1) / kBrSB) & 1, abort_flag, err,
                              kSitePvDone)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + kColO + 32u * j, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
          tmem_st32(tmem + lane_off + kColO + 32u * j, o);
        }
        // P (bf16) over the S buffer: slice j's 16 tokens are packed columns [8j, 8j + 8).  Every slice
        // loaded its scores before any passed the barrier above, so nothing unread is overwritten.
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(s[2 * i], s[2 * i + 1]);
        tmem_st8(tmem + lane_off + s_col + 8u * j, pk);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[g % kBrSB]));
        if (q == 0 && lane == 0 && j < 2) BR_TRACE(g, j == 0 ? kTbPReady : kTbPReady1);
      }
      if (!ok) break;
      // epilogue: slice j writes O columns [32j, 32j + 32) of its head; (m, l) of the piece
      if (!mbar_wait_warp(smem_u32(&bars->pv_done[(g - 1) % kBrSB]), ((g - 1) / kBrSB) & 1, abort_flag, err,
                          kSitePvDone))
        break;
      tc_fence_after();
      const int slot = c + walk.b;
      {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + kColO + 32u * j, o);
        if (real) {
          float4* dst =
              reinterpret_cast<float4*>(o_part + ((size_t)slot * a.H + head) * a.d_c + d_cb * br + 32 * j);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                 __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
        }
      }
      bars->lsum[j][head] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->l_full[q]));
      if (!mbar_wait_warp(smem_u32(&bars->l_full[q]), seg & 1, abort_flag, err, kSiteL)) break;
      if (j == 0 && real) {
        const float l = (bars->lsum[0][head] + bars->lsum[1][head]) + (bars->lsum[2][head] + bars->lsum[3][head]);
        ml_part[(((size_t)slot * a.n_branch + br) * 2 + 0) * a.H + head] = m_run;
        ml_part[(((size_t)slot * a.n_branch + br) * 2 + 1) * a.H + head] = l;
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
  if (warp == 1) tmem_dealloc(tmem, kBrTmemCols);
}

}  // namespace

#ifdef MLRA_TRACE
// Copies the pipeline trace of the last branch-kernel launch (trace builds only).
extern "C" __attribute__((visibility("default"))) int mlra_branch_trace_read(unsigned long long* host, size_t n) {
  const size_t bytes =
      sizeof(g_btrace) < n * sizeof(unsigned long long) ? sizeof(g_btrace) : n * sizeof(unsigned long long);
  return (int)cudaMemcpyFromSymbol(host, g_btrace, bytes);
}
#endif

// The kernel is written for n 128-dim branches, but the library sends it the
// one-branch decode of a 128-dim latent only (the share of a branch-parallel
// MLRA rank): MLRA-4 over a 512-dim latent ran faster on the four-CTA layout
// of attn_tc.cu (202.8 against 234 us at 32 x 16384 tokens, 128 heads), whose
// two CTAs per SM give two independent page pipelines.
bool tc_branch_supported(int H, int d_c, int d_r, int n_branch) {
  return H > 32 && H <= 128 && d_r == 64 && n_branch == 1 && d_c == 128;
}

int tc_branch_workers(int sms, int n_branch) { return sms / n_branch > 0 ? sms / n_branch : 1; }

cudaError_t launch_attend_tc_branch(const void* q_ws, const void* lat, const void* rop, const int* page_table,
                                    const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                                    cudaStream_t st, bool pdl) {
  if (!tc_branch_supported(a.H, a.d_c, a.d_r, a.n_branch)) return cudaErrorInvalidValue;
  CUtensorMap tl, tr;
  if (!tmap_2d(&tl, lat, (uint64_t)a.d_c, (uint64_t)a.num_pages * kPage, 64, 64) ||
      !tmap_2d(&tr, rop, (uint64_t)a.d_r, (uint64_t)a.num_pages * kPage, 64, 64))
    return cudaErrorInvalidValue;
  auto kern = attend_tc_branch_kernel;
  const int smem = BrLayout::kBytes;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.n_branch * a.G, 1, 1);
  cfg.blockDim = dim3(kBrThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tl, tr, static_cast<const __nv_bfloat16*>(q_ws), page_table, seq_lens, o_part,
                            ml_part, err, a);
}

}  // namespace mlra
