// tcgen05 split-KV latent attention, one 128-dim branch per CTA (sm_100a),
// over units of two pages.
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
//   * Pages go through the CTA in units of two (128 tokens; a piece's last
//     unit may hold one page).  A unit's pages sit next to each other in
//     shared memory, so QK^T is one N = 128 MMA per 16 dims for both pages:
//     a tcgen05 MMA of N <= 64 costs at least ~45 cycles whatever its size,
//     and N = 128 runs at the full rate.  The unit is also the step of every
//     barrier hand-off, which halves them against a page-sized step.
//   * TMEM holds O (128 columns), two S buffers (128 each), one P buffer (64
//     packed columns) and the branch's latent query (64 packed columns); the
//     rope query (16 KB) sits in shared memory beside the unit ring (four
//     units of 48 KB).  P has its own columns, so an S buffer is free again as
//     soon as the softmax has read it: QK^T of unit u + 2 waits for that read,
//     not for PV of unit u, and the softmax waits for PV of unit u - 1 only
//     when it is about to store P.
//   * QK^T (M = 128 heads, N = 128 tokens; the latent part with A = the query
//     in TMEM, the rope part with A = the rope query in shared memory) and PV
//     (A = P in TMEM, B = the unit's latent read MN-major, N = 128 dims) are
//     issued by two warps.
//   * Softmax: per TMEM lane quarter, four warps, one per 32 tokens of the
//     unit; they agree on the unit's row maximum through shared memory.  Past
//     a piece's first unit each warp exponentiates against the running max
//     while that exchange is in flight (capped so nothing overflows) and
//     corrects afterwards when the unit's maximum jumped, so the exchange is
//     off the critical path.  O is rescaled only when the running max grows by
//     more than 2^8.  The first warp of each quarter also loads the query rows
//     per piece.
//   * Producer: the whole TMA warp walks the pages; per unit, lanes fetch the
//     look-ahead page ids and issue the unit's six tile loads at once.
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

// warp 0 TMA, 1 QK^T issue, 2 PV issue (and the length checks), 3-18 softmax:
// token quarter jq = (warp - 3) / 4 of the unit (tokens 32 jq .. 32 jq + 31),
// lane quarter q = warp % 4 (a warp reaches only the TMEM lanes of quarter
// warp % 4); the warps with jq = 0 also load the query.
constexpr int kBrUnitPages = 2;                 // pages of a unit (128 tokens)
constexpr int kBrSlices = 4;                    // 32-token slices of a unit
constexpr int kBrSmxWarps = 4 * kBrSlices;
constexpr int kBrSmxWarp0 = 3;
constexpr int kBrThreads = 32 * (kBrSmxWarp0 + kBrSmxWarps);
constexpr int kBrSB = 2;                        // S buffers: unit u uses u % 2
constexpr int kBrSlot = 64 * 128;               // one page of one 64-dim block: 64 tokens x 64 bf16, 128-byte swizzle
constexpr int kBrUnitSlot = 2 * kBrSlot;        // the same block of a unit's two pages, adjacent: 128 rows
constexpr int kBrMaxUnits = 4;
// Past a piece's first unit, scores are exponentiated against the running max before the unit's maximum
// is known, capped at 2^64 (a sum of 128 such terms stays far inside fp32).
constexpr float kSpecCapLog2 = 64.f;
constexpr uint32_t kBrTmemCols = 512;
// TMEM columns: O (128 latent dims), two S buffers (128 tokens each), P (128
// bf16 = 64 packed columns) and the latent query (128 bf16 = 64)
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 128;
constexpr uint32_t kColP = kColS + 128 * kBrSB;
constexpr uint32_t kColQ = kColP + 64;
static_assert(kColQ + 64 <= kBrTmemCols, "TMEM columns");
constexpr int kBrQRBytes = 128 * 128;  // rope query: 128 heads x 64 bf16, 128-byte swizzle

struct BrBars {
  uint64_t unit_full[kBrMaxUnits], unit_empty[kBrMaxUnits];
  uint64_t s_full[kBrSB], s_free[kBrSB], p_full[kBrSB], pv_done[kBrSB];
  uint64_t q_full, q_empty, o_free;
  uint64_t red_full[4][2];  // per lane quarter, double-buffered: its four slices meet
  uint64_t l_full[4];       // per lane quarter, at the end of a piece
  float red[2][kBrSlices][128];  // [buffer][slice][head] maxima
  float lsum[kBrSlices][128];    // [slice][head] sums at the end of a piece
  WorkerPlan plan;
  int page_ids[kIdRing];
  uint32_t tmem_base;
  int abort_flag;
};

// Shared memory: the unit ring, block-major: block s (latent 0-63, latent
// 64-127, rope) of ring entry k, page j at s * kBlockStride + k * kBrUnitSlot
// + j * kBrSlot, so that a unit's two pages of a block are one 128-row operand;
// then the rope query.
struct BrLayout {
  static constexpr int kCap = 232448;
  static constexpr int kTile = 0;
  static constexpr int kFixed = kBrQRBytes + (int)sizeof(BrBars) + 1024;  // + alignment slack
  static constexpr int kUnits = (kCap - kFixed) / (3 * kBrUnitSlot) < kBrMaxUnits ? (kCap - kFixed) / (3 * kBrUnitSlot)
                                                                                   : kBrMaxUnits;
  static constexpr int kBlockStride = kUnits * kBrUnitSlot;
  static constexpr int kQR = kTile + 3 * kBlockStride;
  static constexpr int kBars = kQR + kBrQRBytes;
  static constexpr int kBytes = kBars + (int)sizeof(BrBars) + 1024;
  static_assert(kBrUnitSlot % 1024 == 0, "swizzle atoms stay aligned");
  static_assert(kUnits == kBrMaxUnits && kBytes <= kCap, "shared memory");
  static_assert((kBlockStride >> 4) < (1 << 14), "the block stride fits the descriptor's leading byte offset");
};

// Optional pipeline trace (builds with -DMLRA_TRACE only): globaltimer stamps
// of each role's events for the first kBrTraceUnits units of CTAs 0 and 1.
#ifdef MLRA_TRACE
constexpr int kBrTraceUnits = 64;
__device__ unsigned long long g_btrace[2][kBrTraceUnits][16];
enum { kTbTma = 0, kTbStageSeen, kTbQkIssued, kTbSLoaded, kTbRedDone, kTbPReady, kTbPSeen, kTbPvIssued,
       kTbStageFree, kTbSLoaded1, kTbPReady1 };
#define BR_TRACE(uu, ev)                                                                                   \
  do {                                                                                                     \
    if (blockIdx.x < 2 && (uu) < (uint32_t)kBrTraceUnits) g_btrace[blockIdx.x][uu][ev] = globaltimer_ns(); \
  } while (0)
#else
#define BR_TRACE(uu, ev) \
  do {                   \
  } while (0)
#endif

enum { kSiteQEmpty = 1, kSiteStageEmpty, kSiteQFull, kSiteMma, kSiteOFree, kSiteSFull, kSitePFull, kSitePvDone,
       kSiteRed, kSiteL };

// The units of a piece: pages [pg0, pg1) of the piece in pairs, numbered
// globally from u0.
struct UnitRange {
  uint32_t u0, u_end;
  int pg0, pg1, L;
  __device__ __forceinline__ int first_page(uint32_t u) const { return pg0 + kBrUnitPages * (int)(u - u0); }
  __device__ __forceinline__ int pages(uint32_t u) const { return min(kBrUnitPages, pg1 - first_page(u)); }
  // tokens of the unit inside the sequence (a piece may end before the sequence does)
  __device__ __forceinline__ int valid(uint32_t u) const { return min(pages(u) * kPage, L - first_page(u) * kPage); }
};
__device__ __forceinline__ UnitRange units_of(const SegWalk& w, uint32_t u0) {
  UnitRange r;
  r.u0 = u0;
  r.u_end = u0 + (uint32_t)((w.pg1 - w.pg0 + kBrUnitPages - 1) / kBrUnitPages);
  r.pg0 = w.pg0;
  r.pg1 = w.pg1;
  r.L = w.L;
  return r;
}

__global__ void __launch_bounds__(kBrThreads, 1)
    attend_tc_branch_kernel(const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_rope,
                            const __nv_bfloat16* __restrict__ q_ws, const int* __restrict__ page_table,
                            const int* __restrict__ seq_lens, float* __restrict__ o_part,
                            float* __restrict__ ml_part, int* __restrict__ err, AttnArgs a) {
  using L = BrLayout;
  constexpr int kUnits = L::kUnits;
  constexpr uint32_t kIdescQK1 = idesc_bf16_f32(128, 64, false, false);   // one page
  constexpr uint32_t kIdescQK2 = idesc_bf16_f32(128, 128, false, false);  // two pages
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);    // B = the latent read MN-major

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sTile = smem + L::kTile;
  uint8_t* sQR = smem + L::kQR;
  BrBars* bars = reinterpret_cast<BrBars*>(smem + L::kBars);
  volatile int* abort_flag = &bars->abort_flag;
  auto block_of = [&](int s2, uint32_t k, int j) { return sTile + s2 * L::kBlockStride + k * kBrUnitSlot + j * kBrSlot; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dep_launch();  // the combine kernel may set up (and load its weights) as this grid retires
  const int br = blockIdx.x / a.G;  // branch
  const int c = blockIdx.x % a.G;   // page-range worker
  const int maxL = a.maxp * kPage;
  const int d_cb = a.d_c / a.n_branch;  // 128

  if (threadIdx.x == 0) {
    for (int k = 0; k < kUnits; ++k) {
      mbar_init(smem_u32(&bars->unit_full[k]), 1);
      mbar_init(smem_u32(&bars->unit_empty[k]), 1);
    }
    for (int k = 0; k < kBrSB; ++k) {
      mbar_init(smem_u32(&bars->s_full[k]), 1);
      mbar_init(smem_u32(&bars->s_free[k]), kBrSmxWarps);
      mbar_init(smem_u32(&bars->p_full[k]), kBrSmxWarps);
      mbar_init(smem_u32(&bars->pv_done[k]), 1);
    }
    mbar_init(smem_u32(&bars->q_full), 4);  // the query loaders, one per lane quarter
    mbar_init(smem_u32(&bars->q_empty), 1);
    mbar_init(smem_u32(&bars->o_free), kBrSmxWarps);
    for (int q = 0; q < 4; ++q) {
      mbar_init(smem_u32(&bars->red_full[q][0]), kBrSlices);
      mbar_init(smem_u32(&bars->red_full[q][1]), kBrSlices);
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
  if (warp == 2 && blockIdx.x == 0) {
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
    // The pages through the unit ring in walk order, across pieces (the
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
    }
    // The whole warp walks the pages (every lane keeps the same cursors); per
    // unit, lane j fetches the id of page g + kIdAhead + j and parks it in the
    // ring at the next unit, and lane 3 j + s issues block s of the unit's
    // page j, so that a unit costs the warp a few instructions, not a few
    // dozen dependent ones on one lane.
    SegWalk walk(plan, a.B, maxL);
    int* id_ring = bars->page_ids;
    int pend = 0;          // this lane's fetched id (of page pend_g + lane), parked at the next unit
    int npend = 0;
    uint32_t pend_g = 0;
    uint32_t g = 0, u_next = 0;
    bool ok = true;
    while (ok && walk.next(seq_lens)) {
      const UnitRange ur = units_of(walk, u_next);
      for (uint32_t u = ur.u0; u < ur.u_end; ++u) {
        const uint32_t k = u % kUnits, use = u / kUnits;
        if (use > 0 && !mbar_wait_warp(smem_u32(&bars->unit_empty[k]), (use - 1) & 1, abort_flag, err, kSiteStageEmpty)) {
          ok = false;
          break;
        }
        if (lane == 0) BR_TRACE(u, kTbStageFree);
        const int np = ur.pages(u);
        if (lane < npend) id_ring[(pend_g + lane) % kIdRing] = pend;
        {
          int my_b = -1, my_p = 0, nf = 0;
#pragma unroll
          for (int j = 0; j < kBrUnitPages; ++j)
            if (j < np && ids.live) {
              if (lane == j) {
                my_b = ids.w.b;
                my_p = ids.p;
              }
              ids.step(seq_lens);
              ++nf;
            }
          if (lane < nf) pend = __ldg(page_table + (size_t)my_b * a.maxp + my_p);
          npend = nf;
          pend_g = g + kIdAhead;
        }
        const uint32_t fb = smem_u32(&bars->unit_full[k]);
        if (lane == 0) mbar_expect_tx(fb, (uint32_t)(np * 3 * kBrSlot));
        __syncwarp();
        if (lane < 3 * np) {
          const int j = lane / 3, s2 = lane % 3;
          int pg = id_ring[(g + (uint32_t)j) % kIdRing];
          if (pg < 0 || pg >= a.num_pages) {  // reported, and replaced by page 0 so that no load leaves the pool
            report_error(err, kErrDeviceCheck, walk.b, (ur.first_page(u) + j) * kPage);
            pg = 0;
          }
          tma_load_2d(smem_u32(block_of(s2, k, j)), s2 < 2 ? &tm_lat : &tm_rope, fb, s2 < 2 ? d_cb * br + 64 * s2 : 0,
                      pg * kPage);
        }
        __syncwarp();
        if (lane == 0) BR_TRACE(u, kTbTma);
        g += (uint32_t)np;
      }
      u_next = ur.u_end;
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- QK^T
    // QK^T a unit at a time (one N = 128 MMA per 16 dims for two pages), as
    // soon as the unit has landed and the softmax has read the scores its S
    // buffer held two units ago.
    SegWalk walk(plan, a.B, maxL);
    int seg = 0;
    uint32_t u_next = 0;
    bool ok = true;
    while (ok && walk.next(seq_lens)) {
      if (!mbar_wait_warp(smem_u32(&bars->q_full), seg & 1, abort_flag, err, kSiteQFull)) break;
      tc_fence_after();
      const UnitRange ur = units_of(walk, u_next);
      for (uint32_t u = ur.u0; u < ur.u_end; ++u) {
        const uint32_t k = u % kUnits;
        if (!mbar_wait_warp(smem_u32(&bars->unit_full[k]), (u / kUnits) & 1, abort_flag, err, kSiteMma) ||
            (u >= (uint32_t)kBrSB && !mbar_wait_warp(smem_u32(&bars->s_free[u % kBrSB]), ((u / kBrSB) - 1) & 1,
                                                      abort_flag, err, kSitePvDone))) {
          ok = false;
          break;
        }
        if (lane == 0) BR_TRACE(u, kTbStageSeen);
        const int np = ur.pages(u);
        const int valid = ur.valid(u);
        if (valid < np * kPage) {  // zero the rows past the end of the sequence in the unit's last page
          const int j = np - 1, v = valid - j * kPage, nrow = kPage - v;
          const uint4 z = make_uint4(0, 0, 0, 0);
          for (int idx = lane; idx < nrow * 8 * 3; idx += 32) {
            const int s2 = idx / (nrow * 8), rem = idx % (nrow * 8);
            *reinterpret_cast<uint4*>(block_of(s2, k, j) + (v + rem / 8) * 128 + (rem % 8) * 16) = z;
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        tc_fence_after();
        if (lane == 0) {
          const uint64_t td = sdesc_sw128(smem_u32(block_of(0, k, 0)), 16, 1024);
          const uint32_t s_col = tmem + kColS + (u % kBrSB) * 128u;
          const uint32_t idesc = np == 2 ? kIdescQK2 : kIdescQK1;
#pragma unroll
          for (int s2 = 0; s2 < 2; ++s2)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_ts(s_col, tmem + kColQ + 32u * s2 + 8u * ks, td + (uint64_t)((s2 * L::kBlockStride + ks * 32) >> 4),
                     idesc, (s2 | ks) ? 1u : 0u);
          const uint64_t qrd = sdesc_sw128(smem_u32(sQR), 16, 1024);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ss(s_col, qrd + (uint64_t)((ks * 32) >> 4), td + (uint64_t)((2 * L::kBlockStride + ks * 32) >> 4), idesc,
                   1u);
          mma_commit(smem_u32(&bars->s_full[u % kBrSB]));
          if (u + 1 == ur.u_end) mma_commit(smem_u32(&bars->q_empty));  // the last read of this query
          BR_TRACE(u, kTbQkIssued);
        }
        __syncwarp();
      }
      u_next = ur.u_end;
      ++seg;
    }
  } else if (warp == 2) {
    // ----------------------------------------------------------------- PV
    // PV a unit at a time into O, as soon as every slice of its P is in
    // TMEM; the commits free the unit's ring entry and the P buffer.
    SegWalk walk(plan, a.B, maxL);
    int seg = 0;
    uint32_t u_next = 0;
    bool ok = true;
    while (ok && walk.next(seq_lens)) {
      // the previous piece's O must be read out before the first PV overwrites it
      if (seg > 0 && !mbar_wait_warp(smem_u32(&bars->o_free), (seg - 1) & 1, abort_flag, err, kSiteOFree)) break;
      const UnitRange ur = units_of(walk, u_next);
      for (uint32_t u = ur.u0; u < ur.u_end; ++u) {
        if (!mbar_wait_warp(smem_u32(&bars->p_full[u % kBrSB]), (u / kBrSB) & 1, abort_flag, err, kSitePFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          BR_TRACE(u, kTbPSeen);
          const uint32_t k = u % kUnits;
          const uint64_t vd = sdesc_sw128(smem_u32(block_of(0, k, 0)), (uint32_t)L::kBlockStride, 1024);
          // P of tokens 16 ks .. 16 ks + 15: packed columns kColP + 8 ks
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ts(tmem + kColO, tmem + kColP + 8u * ks, vd + (uint64_t)((ks * 2048) >> 4), kIdescPV,
                   (u == ur.u0 && ks == 0) ? 0u : 1u);
          if (ur.pages(u) == 2) {
#pragma unroll
            for (int ks = 4; ks < 8; ++ks)
              mma_ts(tmem + kColO, tmem + kColP + 8u * ks, vd + (uint64_t)((ks * 2048) >> 4), kIdescPV, 1u);
          }
          mma_commit(smem_u32(&bars->unit_empty[k]));
          mma_commit(smem_u32(&bars->pv_done[u % kBrSB]));
          BR_TRACE(u, kTbPvIssued);
        }
        __syncwarp();
      }
      u_next = ur.u_end;
      ++seg;
    }
  } else if (warp >= kBrSmxWarp0) {
    // -------------------------------------------------------------- softmax
    // Lane quarter q (heads 32q + lane), token slice jq of each unit.
    const int sw = warp - kBrSmxWarp0;
    const int jq = sw / 4;
    const int q = warp & 3;
    const int head = q * 32 + lane;
    const bool real = head < a.H;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    SegWalk walk(plan, a.B, maxL);
    uint32_t u_next = 0;
    int seg = 0;
    bool ok = true;
    if (jq == 0) grid_dep_wait();  // the absorbed queries come from the previous kernel
    while (ok && walk.next(seq_lens)) {
      if (jq == 0) {
        // the piece's query rows of heads 32q + lane (this branch's 128 latent dims as 64 packed bf16x2
        // TMEM columns; the 64 rope dims into the rope query's swizzled row in shared memory), once the
        // previous piece's last QK^T has completed
        if (seg > 0 && !mbar_wait_warp(smem_u32(&bars->q_empty), (seg - 1) & 1, abort_flag, err, kSiteQEmpty)) break;
        tc_fence_after();
        const __nv_bfloat16* src = q_ws + ((size_t)walk.b * a.H + (real ? head : 0)) * (a.d_c + a.d_r);
        const uint4* lat = reinterpret_cast<const uint4*>(src + d_cb * br);
        const uint4* rop = reinterpret_cast<const uint4*>(src + a.d_c);
        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {  // latent columns 0-31, 32-63
          const uint4* from = lat + 8 * blk;
          uint32_t r[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint4 v = real ? __ldg(from + i) : z;
            r[4 * i] = v.x;
            r[4 * i + 1] = v.y;
            r[4 * i + 2] = v.z;
            r[4 * i + 3] = v.w;
          }
          tmem_st32(tmem + lane_off + kColQ + 32u * blk, r);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)  // 16-byte chunk i of row `head` sits at chunk i ^ (head % 8)
          *reinterpret_cast<uint4*>(sQR + head * 128 + ((i ^ (head & 7)) * 16)) = real ? __ldg(rop + i) : z;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->q_full));
      }
      const UnitRange ur = units_of(walk, u_next);
      float m_run = -INFINITY, l_run = 0.f;
      for (uint32_t u = ur.u0; u < ur.u_end; ++u) {
        const int valid = ur.valid(u) - 32 * jq;  // valid tokens of this slice (<= 0: none)
        // scores of token 32 jq + t at column s_sl + t; its P (bf16) at packed column kColP + 16 jq + t / 2
        const uint32_t s_sl = tmem + lane_off + kColS + (u % kBrSB) * 128u + 32u * (uint32_t)jq;
        if (!mbar_wait_warp(smem_u32(&bars->s_full[u % kBrSB]), (u / kBrSB) & 1, abort_flag, err, kSiteSFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the slice's scores (masked past the end of the sequence)
        float x[32];
        {
          uint32_t vhi[16], vlo[16];
          tmem_ld16(s_sl + 16u, vhi);  // tokens 16-31 of the slice
          tmem_ld16(s_sl, vlo);        // tokens 0-15
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            x[i] = __uint_as_float(vlo[i]);
            x[16 + i] = __uint_as_float(vhi[i]);
          }
        }
        if (valid < 32) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i >= valid) x[i] = -INFINITY;
        }
        float m4[4];
#pragma unroll
        for (int i = 0; i < 32; ++i) m4[i & 3] = i < 4 ? x[i] : fmaxf(m4[i & 3], x[i]);
        if (q == 0 && lane == 0) BR_TRACE(u, jq == 0 ? kTbSLoaded : kTbSLoaded1);
        const int rb = (int)(u & 1u);
        bars->red[rb][jq][head] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->red_full[q][rb]));
        // Past a piece's first unit the running max is known: exponentiate against it (capped at 2^64, so
        // nothing overflows) while the slices exchange their maxima, and correct afterwards in the rare
        // case the unit's maximum jumped.  The first unit waits for the exchange.
        const bool spec = u != ur.u0;
        float a4[4] = {0.f, 0.f, 0.f, 0.f};
        if (spec) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            x[i] = ex2(fminf(x[i] - m_run, kSpecCapLog2));
            a4[i & 3] += x[i];
          }
        }
        if (!mbar_wait_warp(smem_u32(&bars->red_full[q][rb]), (u >> 1) & 1, abort_flag, err, kSiteRed)) {
          ok = false;
          break;
        }
        if (q == 0 && jq == 0 && lane == 0) BR_TRACE(u, kTbRedDone);
        // the unit's row maximum (its first token is valid, so it is finite); the four slices of a quarter
        // read the same four values and decide alike
        const float M = fmaxf(fmaxf(bars->red[rb][0][head], bars->red[rb][1][head]),
                              fmaxf(bars->red[rb][2][head], bars->red[rb][3][head]));
        float m_use = m_run, corr = 1.f;
        bool rescale = false;
        if (!spec) {
          m_use = M;
          corr = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            x[i] = ex2(x[i] - M);
            a4[i & 3] += x[i];
          }
        } else if (__any_sync(0xffffffffu, M > m_run + kSpecCapLog2)) {
          // a jump past the cap (some head of the warp): exponentiate the scores again, read anew from S
          // (the S buffer is released only below), against each head's new reference
          rescale = M > m_run + kRescaleLog2;
          m_use = rescale ? M : m_run;
          corr = rescale ? ex2(m_run - M) : 1.f;
          uint32_t vhi[16], vlo[16];
          tmem_ld16(s_sl + 16u, vhi);
          tmem_ld16(s_sl, vlo);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float sc = __uint_as_float(i < 16 ? vlo[i] : vhi[i - 16]);
            x[i] = i < valid ? ex2(sc - m_use) : 0.f;
            a4[i & 3] = i < 4 ? x[i] : a4[i & 3] + x[i];
          }
        } else if (M > m_run + kRescaleLog2) {
          rescale = true;
          m_use = M;
          corr = ex2(m_run - M);
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] *= corr;
#pragma unroll
          for (int i = 0; i < 4; ++i) a4[i] *= corr;
        }
        tc_fence_before();  // the S buffer is read: QK^T of unit u + 2 may overwrite it
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->s_free[u % kBrSB]));
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
        l_run = l_run * corr + ((a4[0] + a4[1]) + (a4[2] + a4[3]));
        m_run = m_use;
        // the P buffer (and O) are free once PV of the previous unit, of this piece or the last one, is done
        if (u > 0) {
          const uint32_t up = u - 1;
          if (!mbar_wait_warp(smem_u32(&bars->pv_done[up % kBrSB]), (up / kBrSB) & 1, abort_flag, err, kSitePvDone)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        tmem_st16(tmem + lane_off + kColP + 16u * (uint32_t)jq, pk);
        // O is rescaled only when the running max jumped; slice jq takes columns [32 jq, 32 jq + 32)
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t o[16];
            const uint32_t col = tmem + lane_off + kColO + 32u * (uint32_t)jq + 16u * h2;
            tmem_ld16(col, o);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
            tmem_st16(col, o);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[u % kBrSB]));
        if (q == 0 && lane == 0) BR_TRACE(u, jq == 0 ? kTbPReady : kTbPReady1);
      }
      if (!ok) break;
      // epilogue: slice jq writes O columns [32 jq, 32 jq + 32) of its head; (m, l) of the piece.  PV of the
      // piece's last unit completing implies all of its PVs have (one issuing thread, completed in order).
      const uint32_t last = ur.u_end - 1;
      if (!mbar_wait_warp(smem_u32(&bars->pv_done[last % kBrSB]), (last / kBrSB) & 1, abort_flag, err, kSitePvDone))
        break;
      tc_fence_after();
      const int slot = c + walk.b;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t o[16];
        tmem_ld16(tmem + lane_off + kColO + 32u * (uint32_t)jq + 16u * h2, o);
        if (real) {
          float4* dst = reinterpret_cast<float4*>(o_part + ((size_t)slot * a.H + head) * a.d_c + d_cb * br + 32 * jq +
                                                  16 * h2);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                 __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
        }
      }
      bars->lsum[jq][head] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->l_full[q]));
      if (!mbar_wait_warp(smem_u32(&bars->l_full[q]), seg & 1, abort_flag, err, kSiteL)) break;
      if (jq == 0 && real) {
        const float l = (bars->lsum[0][head] + bars->lsum[1][head]) + (bars->lsum[2][head] + bars->lsum[3][head]);
        ml_part[(((size_t)slot * a.n_branch + br) * 2 + 0) * a.H + head] = m_run;
        ml_part[(((size_t)slot * a.n_branch + br) * 2 + 1) * a.H + head] = l;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->o_free));
      u_next = ur.u_end;
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

// Branches of 128 latent dims (MLRA over n_branch x 128 dims, and the
// one-branch decode of a 128-dim latent that a branch-parallel MLRA rank runs),
// 64 rope dims, 33 to 128 heads.
bool tc_branch_supported(int H, int d_c, int d_r, int n_branch) {
  return H > 32 && H <= 128 && d_r == 64 && (n_branch == 1 || n_branch == 2 || n_branch == 4) &&
         d_c == 128 * n_branch;
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
