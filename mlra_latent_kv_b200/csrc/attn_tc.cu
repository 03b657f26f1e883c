// tcgen05 split-KV latent attention for sm_100a (a3 of the decode path).
//
// Method: yololab.net, "超越 GQA 的推理革命…", section "矩陣吸收": with W_UK
// folded into the query, every head scores the cached latent c_KV directly
// (plus the decoupled RoPE key, section "2. 解耦旋轉位置編碼"), and the value
// side is the same latent, so all heads of a sequence share one cache tile:
//   S[h, t] = q_lat[h] . c[t] + q_rot[h] . k[t]      (QK^T, K = 512 + 64)
//   O[h, :] += softmax_t(scale * S)[h, t] . c[t, :]  (PV, N = 512)
// MLRA (wispaper.ai, "MLRA：突破 MLA 并行瓶颈…", section "2.1 架构拆解"): each
// branch runs its own softmax over its own latent block, with the rope score
// shared by all branches.
//
// Design (B200):
//   * A worker is a pair of CTAs (on two SMs).  The fp32 accumulator O of 128
//     heads x 512 latent dims needs all 512 TMEM columns of an SM, so each CTA
//     of the pair owns 256 latent dims of O (and loads only those 256 dims of
//     every cache page); the other 256 TMEM columns hold a ring of S buffers
//     (four with one branch per CTA, two with two).
//   * MLA (one softmax over all 512 dims): CTA r computes the partial scores
//     of its 256 latent dims and of its 32 of the 64 rope dims.  Exchange warps
//     send each page's partial to the peer through distributed shared memory
//     as soon as QK^T has produced it, as the row's maximum r over the page's
//     tokens (fp32) and each score's offset from it, s - r, rounded to fp16.
//     Both CTAs then form (r_0 + r_1) + (f16(s_0 - r_0) + f16(s_1 - r_1)),
//     the offsets added as an fp16 pair: addition commutes, so they hold the
//     same bits and compute identical softmax weights, and the rounding error
//     of a score is a few 2^-11 of its distance below its row's page maximum,
//     however large the logits.
//   * MLRA with 2 or 4 branches: the branches of a CTA are wholly its own, so
//     the CTAs of a worker never talk; each adds the full rope score to its
//     branches.  MLRA-4 with more than 32 heads runs four CTAs per worker, one
//     branch (128 latent dims) each: O then takes 128 TMEM columns and a page
//     24 KB of shared memory, so two CTAs fit on one SM and each SM runs two
//     independent page pipelines.
//   * Per 64-token page: one TMA producer warp loads the page's latent blocks
//     (128-byte swizzle) into a stage ring, reading page ids a few pages ahead
//     of the loads; one MMA warp issues QK^T (A = queries in shared memory, B =
//     tile K-major) into S in TMEM, and PV with A = P in TMEM and B = the same
//     tile read MN-major; four softmax warps per branch (one TMEM lane quarter
//     each, one head per thread) read S, apply the online softmax (rescaling O
//     only when the running max grows by more than 2^8), and write P (bf16)
//     back over S.
//   * Rows past the sequence end in the last page are zeroed in shared memory
//     before the MMAs read them (a NaN there would poison P.V even at P = 0).
//   * With H <= 32 the query and exchange buffers shrink to 32 rows, which
//     makes room for a six-page ring.
//   * Every wait is bounded; a wait that runs out sets the CTA's abort flag and
//     records MLRA_ERR_TIMEOUT with its site, and every role then leaves.
// The split plan and the partial-result layout are those of the CUDA-core
// kernel (slot c + b, running max in log2 units, o_part[slot][H][d_c]).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "attn_common.cuh"
#include "attn_tc.h"
#include "host_cache.h"
#include "ptx.cuh"

namespace mlra {
namespace {

using namespace ptx;

// warp 0: TMA, warp 1: MMA, then 4 softmax warps per branch a CTA owns (one
// warpgroup covers the 128 TMEM lanes = heads)
template <bool kExch, int kBrPerCta>
constexpr int threads_of() { return 64 + 128 * kBrPerCta + (kExch ? 128 : 0); }  // + MLA exchange warps
constexpr int kTileSlotBytes = 64 * 128;  // 64 tokens x 64 bf16
constexpr int kMaxStages = 6;
// The MLRA-4 four-CTA layout holds only two stages per CTA; its producer also
// starts page g + kQuadPrefetch towards L2 when it loads page g, so that the
// load issued when a stage frees mostly hits L2.
constexpr uint32_t kQuadPrefetch = 2;
static_assert(kQuadPrefetch < (uint32_t)kIdAhead, "prefetched page ids are already in the id ring");
// CTAs per worker.  2: a pair on two SMs, each CTA owning 256 latent dims
// (four 64-dim blocks).  4 (MLRA-4): one branch of 128 latent dims per CTA,
// two CTAs resident per SM, each with half of the SM's TMEM and shared memory.
template <int kCtas>
constexpr int lat_slots() { return 8 / kCtas; }  // 64-dim latent blocks per CTA
template <int kCtas>
constexpr uint32_t tmem_cols() { return kCtas == 4 ? 256u : 512u; }
template <int kCtas>
constexpr int min_blocks() { return kCtas == 4 ? 2 : 1; }
// TMEM columns: O [0, 64 * lat_slots), then a ring of S buffers of 64 columns
// per branch the CTA owns (at most four).
template <int kBrPerCta, int kCtas>
constexpr int s_bufs() {
  return ((int)tmem_cols<kCtas>() - 64 * lat_slots<kCtas>()) / (64 * kBrPerCta) < 4
             ? ((int)tmem_cols<kCtas>() - 64 * lat_slots<kCtas>()) / (64 * kBrPerCta)
             : 4;
}

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t stage_full[kMaxStages], stage_empty[kMaxStages];
  uint64_t rope_full[2], rope_empty[2];  // MLA: the rope half has its own two-slot ring
  uint64_t s_full[4], p_full[4], pv_done[4];
  uint64_t o_free;
  uint64_t x_full[4], x_empty[4];  // MLA exchange, per lane quarter (one softmax warp each)
  uint64_t xs_read[4][4];          // MLA: the exchange warp of a quarter has read S buffer k
  WorkerPlan plan;
  int page_ids[16];  // producer's ring of fetched page ids
  uint32_t tmem_base;
  int abort_flag;
};

// Shared-memory layout.
//  MLA (kExch): 4 latent blocks of this CTA's 256 dims per page in a ring of 4
//  stages; the CTA's half of the rope dims (32, 64-byte swizzle) in its own
//  two-slot ring, released as soon as QK^T has read it; one fp16 exchange
//  buffer for the partial scores of one page.
//  MLRA: the CTA's latent blocks + the full rope block (128-byte swizzle) per
//  stage; a ring of 3 stages for a pair (4 blocks), 2 for a quad (2 blocks,
//  two CTAs per SM).
//  Query blocks, the exchange buffer and the rope query take kHq rows: 128,
//  or 32 when H <= 32, which leaves room for two more stages.  The M = 128
//  MMAs read 128 rows from each query block; the rows past kHq fall on the
//  next buffer, feed only MMA rows of absent heads, and are never used.
template <bool kExch, int kHq, int kCtas>
struct Layout {
  static constexpr int kLat = lat_slots<kCtas>();
  // per-CTA shared memory: one CTA per SM, or half of the SM's 228 KB less the
  // 1 KB the hardware reserves per CTA
  static constexpr int kCap = min_blocks<kCtas>() == 1 ? 232448 : 233472 / 2 - 1024;
  static constexpr int kQSlotBytes = kHq * 128;  // kHq query rows x 64 bf16
  static constexpr int kRopeQBytes = kExch ? kHq * 64 : kQSlotBytes;
  static constexpr int kRopeTileBytes = kExch ? 64 * 64 : kTileSlotBytes;
  static constexpr int kRopeRowBytes = kExch ? 64 : 128;
  static constexpr int kXBytes = 64 * kHq * 2;   // one page of fp16 score offsets, kHq rows
  static constexpr int kXRBytes = kHq * 4;       // the fp32 row maxima they are offsets from
  static constexpr int kStageBytes = kLat * kTileSlotBytes + (kExch ? 0 : kRopeTileBytes);
  static constexpr int kQ = 0;
  static constexpr int kQRope = kLat * kQSlotBytes;
  static constexpr int kRope = kQRope + kRopeQBytes;  // MLA rope ring
  static constexpr int kX = kRope + (kExch ? 2 * kRopeTileBytes : 0);
  static constexpr int kXR = kX + (kExch ? kXBytes : 0);
  static constexpr int kTile = (kXR + (kExch ? kXRBytes : 0) + 1023) / 1024 * 1024;
  static constexpr int kFixed = kTile + (int)sizeof(Bars) + 1024;  // + alignment slack
  static constexpr int kStages = (kCap - kFixed) / kStageBytes < kMaxStages ? (kCap - kFixed) / kStageBytes
                                                                              : kMaxStages;
  static constexpr int kBars = kTile + kStages * kStageBytes;
  static constexpr int kBytes = kBars + (int)sizeof(Bars) + 1024;
  static_assert(kStages >= (kCtas == 4 ? 2 : 3), "stage ring");
  static_assert(kStageBytes % 1024 == 0 && kTile % 1024 == 0 && kRope % 512 == 0 && kQRope % 1024 == 0,
                "aligned slots");
  static_assert(kBytes <= kCap, "shared memory");
  // the last query block's 128-row MMA read stays inside the CTA's shared memory
  static_assert((kLat - 1) * kQSlotBytes + 128 * 128 <= kBytes && kQRope + 128 * (kExch ? 64 : 128) <= kBytes,
                "query reads");
};

// Optional pipeline trace (builds with -DMLRA_TRACE only): globaltimer stamps
// of each role's events for the first kTracePages pages of CTAs 0 and 1.
#ifdef MLRA_TRACE
constexpr int kTracePages = 64;
constexpr int kTraceEvents = 16;
__device__ unsigned long long g_trace[2][kTracePages][kTraceEvents];
__device__ unsigned long long g_span[1024][2];  // entry and exit stamp of every CTA
enum { kEvTma = 0, kEvStageSeen, kEvQkIssued, kEvSReady, kEvSent, kEvRecv, kEvPReady, kEvPvIssued, kEvMath,
       kEvSoftmaxDone, kEvQkStart, kEvRecvAdded, kEvXLoaded, kEvXEmptySeen, kEvOwnLoaded, kEvXFullWait };
#define MLRA_TRACE_EV(gg, ev)                                                                  \
  do {                                                                                         \
    if (blockIdx.x < 2 && (gg) < (uint32_t)kTracePages) g_trace[blockIdx.x][gg][ev] = globaltimer_ns(); \
  } while (0)
#else
#define MLRA_TRACE_EV(gg, ev) \
  do {                        \
  } while (0)
#endif

// wait-site codes recorded with a timeout
enum { kSiteQEmpty = 1, kSiteStageEmpty, kSiteQFull, kSiteMma, kSiteOFree, kSiteSFull, kSiteXEmpty, kSiteXFull,
       kSitePvDone };

// One page of online softmax for one row (head) in the log2 domain (the
// queries arrive pre-multiplied by softmax_scale*log2(e), so the scores are
// base-2 logits).  s: scores in, exp2(s - m) out; tokens >= valid are masked.
// Returns whether O must be rescaled by corr (the running max grew by more
// than 2^8); the first page of a piece starts the running state.
__device__ __forceinline__ bool softmax_page(float (&s)[64], int valid, bool first, float& m_run, float& l_run,
                                             float& corr) {
  if (valid < 64) {
#pragma unroll
    for (int n = 0; n < 64; ++n)
      if (n >= valid) s[n] = -INFINITY;
  }
  float m8[8];
#pragma unroll
  for (int n = 0; n < 64; ++n) m8[n & 7] = (n < 8) ? s[n] : fmaxf(m8[n & 7], s[n]);
  const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                         fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
  bool rescale = false;
  float m_use;
  if (first) {
    m_use = mx;
    corr = 0.f;
  } else if (mx > m_run + kRescaleLog2) {
    m_use = mx;
    corr = ex2(m_run - mx);
    rescale = true;
  } else {
    m_use = m_run;
    corr = 1.f;
  }
  float a8[8];
#pragma unroll
  for (int n = 0; n < 64; ++n) {
    s[n] = ex2(s[n] - m_use);
    a8[n & 7] = (n < 8) ? s[n] : a8[n & 7] + s[n];
  }
  const float sum = ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
  l_run = l_run * corr + sum;
  m_run = m_use;
  return rescale;
}

// Maximum of a row's scores over the page's first `valid` tokens (the exact
// value does not depend on the order, so the exchange warp, which holds the
// scores as two 32-column halves, and the softmax warp agree on it).
// (Full pages, all but a sequence's last, take the unmasked branch.)
__device__ __forceinline__ float row_max_valid(const uint32_t (&lo)[32], const uint32_t (&hi)[32], int valid) {
  float m8[8];
  if (valid >= 64) {
#pragma unroll
    for (int n = 0; n < 64; ++n) {
      const float v = __uint_as_float(n < 32 ? lo[n] : hi[n - 32]);
      m8[n & 7] = n < 8 ? v : fmaxf(m8[n & 7], v);
    }
  } else {
#pragma unroll
    for (int n = 0; n < 64; ++n) {
      const float v = n < valid ? __uint_as_float(n < 32 ? lo[n] : hi[n - 32]) : -INFINITY;
      m8[n & 7] = n < 8 ? v : fmaxf(m8[n & 7], v);
    }
  }
  return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
}
__device__ __forceinline__ float row_max_valid(const float (&s)[64], int valid) {
  float m8[8];
  if (valid >= 64) {
#pragma unroll
    for (int n = 0; n < 64; ++n) m8[n & 7] = n < 8 ? s[n] : fmaxf(m8[n & 7], s[n]);
  } else {
#pragma unroll
    for (int n = 0; n < 64; ++n) {
      const float v = n < valid ? s[n] : -INFINITY;
      m8[n & 7] = n < 8 ? v : fmaxf(m8[n & 7], v);
    }
  }
  return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
}

template <bool kExch, int kBrPerCta, int kHq, int kCtas>
__global__ void __launch_bounds__(threads_of<kExch, kBrPerCta>(), min_blocks<kCtas>())
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_q_rope,
                     const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_rope,
                     const int* __restrict__ page_table, const int* __restrict__ seq_lens,
                     float* __restrict__ o_part, float* __restrict__ ml_part, int* __restrict__ err, AttnArgs a) {
  using L = Layout<kExch, kHq, kCtas>;
  constexpr int kQSlotBytes = L::kQSlotBytes;
  constexpr int kLat = L::kLat;                 // latent slots of this CTA
  constexpr int kLatPerBr = kLat / kBrPerCta;   // latent slots per branch
  constexpr int kOCols = 64 * kLat;             // TMEM columns of O
  constexpr int kPvN = kOCols / kBrPerCta;      // PV output columns per branch
  constexpr uint32_t kTmemCols = tmem_cols<kCtas>();
  static_assert(!kExch || kCtas == 2, "the score exchange is between the two CTAs of a pair");
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kPvN, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sQRope = smem + L::kQRope;
  uint8_t* sTile = smem + L::kTile;
  uint8_t* sRope = smem + L::kRope;
  uint8_t* sX = smem + L::kX;
  float* sXR = reinterpret_cast<float*>(smem + L::kXR);
  constexpr int kStages = L::kStages;
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBars);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dep_launch();  // the combine kernel may set up (and load its weights) as this grid retires
#ifdef MLRA_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 1024) g_span[blockIdx.x][0] = globaltimer_ns();
#endif
  const uint32_t rank = kExch ? cluster_ctarank() : (blockIdx.x % (unsigned)kCtas);
  const int c = blockIdx.x / kCtas;
  const int maxL = a.maxp * kPage;
  const int rope_q_bytes = a.H * (kExch ? 64 : 128);  // H query rows of the rope block

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->q_empty), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bars->stage_full[s]), 1);
      mbar_init(smem_u32(&bars->stage_empty[s]), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(smem_u32(&bars->rope_full[k]), 1);
      mbar_init(smem_u32(&bars->rope_empty[k]), 1);
    }
    for (int k = 0; k < 4; ++k) {
      mbar_init(smem_u32(&bars->s_full[k]), 1);
      mbar_init(smem_u32(&bars->p_full[k]), 4 * kBrPerCta);
      mbar_init(smem_u32(&bars->pv_done[k]), 1);
    }
    for (int q = 0; q < 4; ++q) {
      mbar_init(smem_u32(&bars->x_full[q]), 1);
      mbar_init(smem_u32(&bars->x_empty[q]), 1);
      for (int k = 0; k < 4; ++k) mbar_init(smem_u32(&bars->xs_read[q][k]), 1);
    }
    mbar_init(smem_u32(&bars->o_free), 4 * kBrPerCta);
    // MLA: the peer's partial scores of page 0 are expected in phase 0 of x_full
    if (kExch)
      for (int q = 0; q * 32 < a.H; ++q)
        mbar_expect_tx(smem_u32(&bars->x_full[q]), (uint32_t)min(32, a.H - q * 32) * (128u + 4u));
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
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
  if (kExch) cluster_sync();  // the peer's barriers exist before anyone arrives on them
  const uint32_t tmem = bars->tmem_base;
  const WorkerPlan plan = bars->plan;

  // S ring (kSB buffers of 64 columns per branch) after the columns of O
  constexpr int kSB = s_bufs<kBrPerCta, kCtas>();
  auto S_col = [](uint32_t buf, int i) -> uint32_t {
    return (uint32_t)kOCols + buf * (64u * kBrPerCta) + (uint32_t)i * 64u;
  };
  static_assert(kSB >= 2 && kOCols + kSB * 64 * kBrPerCta <= (int)kTmemCols, "TMEM columns overflow");
  auto O_col = [](int i) -> uint32_t { return (uint32_t)i * (uint32_t)kPvN; };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    // Page ids are read kIdAhead pages before their tile is loaded (a second
    // cursor over the same pages) and parked in a small ring, so that no
    // page-table load sits between a freed stage and its refill.  The first
    // kIdAhead ids are read by the lanes in parallel; later a fetched id is
    // written to the ring one page after its load was issued.
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
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_lat);
      tma_prefetch_desc(&tm_rope);
      if (kExch) tma_prefetch_desc(&tm_q_rope);
      grid_dep_wait();  // the absorbed queries come from the previous kernel
      SegWalk walk(plan, a.B, maxL);
      int* id_ring = bars->page_ids;
      int pend = 0;
      bool has_pend = false;
      int seg = 0;
      uint32_t g = 0;
      bool ok = true;
      const uint32_t n_pages = (uint32_t)(plan.end - plan.start);  // pages of this worker
      while (ok && walk.next(seq_lens)) {
        if (seg > 0 && !mbar_wait(smem_u32(&bars->q_empty), (seg - 1) & 1, abort_flag, err, kSiteQEmpty)) break;
        const uint32_t qb = smem_u32(&bars->q_full);
        mbar_expect_tx(qb, kLat * a.H * 128 + rope_q_bytes);
        for (int s = 0; s < kLat; ++s)
          tma_load_2d(smem_u32(sQ + s * kQSlotBytes), &tm_q, qb, 64 * (kLat * (int)rank + s), walk.b * a.H);
        if (kExch)
          tma_load_2d(smem_u32(sQRope), &tm_q_rope, qb, a.d_c + 32 * (int)rank, walk.b * a.H);
        else
          tma_load_2d(smem_u32(sQRope), &tm_q, qb, a.d_c, walk.b * a.H);
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
          if (kExch && g >= 2 &&
              !mbar_wait(smem_u32(&bars->rope_empty[g & 1]), ((g >> 1) - 1) & 1, abort_flag, err, kSiteStageEmpty)) {
            ok = false;
            break;
          }
          int pg = id_ring[g % kIdRing];
          if (pg < 0 || pg >= a.num_pages) {  // reported, and replaced by page 0 so that no load leaves the pool
            report_error(err, kErrDeviceCheck, walk.b, p * kPage);
            pg = 0;
          }
          const uint32_t fb = smem_u32(&bars->stage_full[st]);
          uint8_t* tile = sTile + st * L::kStageBytes;
          mbar_expect_tx(fb, L::kStageBytes);
          for (int s = 0; s < kLat; ++s)
            tma_load_2d(smem_u32(tile + s * kTileSlotBytes), &tm_lat, fb, 64 * (kLat * (int)rank + s), pg * kPage);
          if (kExch) {
            const uint32_t rb = smem_u32(&bars->rope_full[g & 1]);
            mbar_expect_tx(rb, L::kRopeTileBytes);
            tma_load_2d(smem_u32(sRope + (g & 1) * L::kRopeTileBytes), &tm_rope, rb, 32 * (int)rank, pg * kPage);
          } else {
            tma_load_2d(smem_u32(tile + kLat * kTileSlotBytes), &tm_rope, fb, 0, pg * kPage);
          }
          if (kCtas == 4 && g + kQuadPrefetch < n_pages) {
            const int pf = id_ring[(g + kQuadPrefetch) % kIdRing];  // written kIdAhead - 1 pages ago
            if (pf >= 0 && pf < a.num_pages) {
              for (int s = 0; s < kLat; ++s) tma_prefetch_l2_2d(&tm_lat, 64 * (kLat * (int)rank + s), pf * kPage);
              tma_prefetch_l2_2d(&tm_rope, 0, pf * kPage);
            }
          }
          MLRA_TRACE_EV(g, kEvTma);
        }
        ++seg;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    // Event loop: QK^T of the next landed page and PV of the next page whose P
    // is ready are issued in whichever order they become possible (QK(g) may
    // run once PV(g - kSB) is issued: S buffer g % kSB holds P(g - kSB) until then).
    SegWalk walk(plan, a.B, maxL);
    int seg = 0;
    uint32_t g = 0;
    bool ok = true;
    const uint64_t qd = sdesc_sw128(smem_u32(sQ), 16, 1024);  // query latent blocks (when read from smem)
    const uint64_t qrd = kExch ? sdesc_sw64(smem_u32(sQRope), 512) : sdesc_sw128(smem_u32(sQRope), 16, 1024);
    while (ok && walk.next(seq_lens)) {
      if (!mbar_wait_warp(smem_u32(&bars->q_full), seg & 1, abort_flag, err, kSiteQFull)) break;
      tc_fence_after();
      const uint32_t g0 = g, g_end = g + (uint32_t)(walk.pg1 - walk.pg0);
      uint32_t g_qk = g0, g_pv = g0;
      bool o_ready = (seg == 0);
      long long t_idle = 0;
      while (g_pv < g_end) {
        bool progressed = false;
        // MLRA issues the next QK^T before a ready PV (its softmax is the longer
        // wait); MLA issues the ready PV first (it frees the stage the next load needs)
        if constexpr (!kExch) {
          // QK(g) needs S buffer g % kSB, free once PV(g - kSB) is issued; look
          // ahead at most two pages past the next PV so that PVs (which free the
          // stages) are not queued behind a run of QKs
          if (!progressed && g_qk < g_end && g_qk < g_pv + kSB && g_qk <= g_pv + 2) {
            const uint32_t st = g_qk % kStages;
            bool ready = lane == 0 ? mbar_test_wait(smem_u32(&bars->stage_full[st]), (g_qk / kStages) & 1) &&
                                         (!kExch || mbar_test_wait(smem_u32(&bars->rope_full[g_qk & 1]),
                                                                   (g_qk >> 1) & 1))
                                   : false;
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (ready) {
              if (lane == 0) MLRA_TRACE_EV(g_qk, kEvStageSeen);
              uint8_t* tile = sTile + st * L::kStageBytes;
              uint8_t* rope_tile = kExch ? sRope + (g_qk & 1) * L::kRopeTileBytes : tile + kLat * kTileSlotBytes;
              const int p = walk.pg0 + (int)(g_qk - g0);
              const int valid = min(kPage, walk.L - p * kPage);
              if (valid < kPage) {  // zero the rows past the end of the sequence
                const int nrow = kPage - valid;
                const uint4 z = make_uint4(0, 0, 0, 0);
                for (int idx = lane; idx < nrow * 8 * kLat; idx += 32) {
                  const int s = idx / (nrow * 8), rem = idx % (nrow * 8);
                  *reinterpret_cast<uint4*>(tile + s * kTileSlotBytes + (valid + rem / 8) * 128 + (rem % 8) * 16) = z;
                }
                constexpr int kRopeChunks = L::kRopeRowBytes / 16;
                for (int idx = lane; idx < nrow * kRopeChunks; idx += 32)
                  *reinterpret_cast<uint4*>(rope_tile + (valid + idx / kRopeChunks) * L::kRopeRowBytes +
                                            (idx % kRopeChunks) * 16) = z;
                fence_proxy_async_smem();
              }
              __syncwarp();
              tc_fence_after();
              if (lane == 0) {
                MLRA_TRACE_EV(g_qk, kEvQkStart);
                // descriptors = per-stage base + compile-time offsets (no per-MMA rebuild)
                const uint64_t td = sdesc_sw128(smem_u32(tile), 16, 1024);
                const uint32_t s_base = tmem + S_col(g_qk % kSB, 0);
  #pragma unroll
                for (int i = 0; i < kBrPerCta; ++i) {
  #pragma unroll
                  for (int j = 0; j < kLatPerBr; ++j) {
                    const int s = i * kLatPerBr + j;
  #pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                      const uint64_t bd = td + (uint64_t)((s * kTileSlotBytes + ks * 32) >> 4);
                      mma_ss(s_base + 64u * i, qd + (uint64_t)((s * kQSlotBytes + ks * 32) >> 4), bd, kIdescQK,
                             (j | ks) ? 1u : 0u);
                    }
                  }
                  if (kExch) {
                    const uint64_t trd = sdesc_sw64(smem_u32(rope_tile), 512);
  #pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
                      mma_ss(s_base + 64u * i, qrd + (uint64_t)(ks * 2), trd + (uint64_t)(ks * 2), kIdescQK, 1u);
                  } else {
  #pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                      mma_ss(s_base + 64u * i, qrd + (uint64_t)(ks * 2),
                             td + (uint64_t)((kLat * kTileSlotBytes + ks * 32) >> 4), kIdescQK, 1u);
                  }
                }
                mma_commit(smem_u32(&bars->s_full[g_qk % kSB]));
                if (kExch) mma_commit(smem_u32(&bars->rope_empty[g_qk & 1]));
                MLRA_TRACE_EV(g_qk, kEvQkIssued);
                if (g_qk + 1 == g_end) mma_commit(smem_u32(&bars->q_empty));  // last read of this Q
              }
              __syncwarp();
              ++g_qk;
              progressed = true;
            }
          }
        }
        if (!progressed && g_pv < g_qk) {
          if (!o_ready) {  // the previous piece's O must be drained before the first PV overwrites it
            bool r = lane == 0 ? mbar_test_wait(smem_u32(&bars->o_free), (seg - 1) & 1) : false;
            o_ready = __shfl_sync(0xffffffffu, r, 0);
          }
          if (o_ready) {
            bool ready =
                lane == 0 ? mbar_test_wait(smem_u32(&bars->p_full[g_pv % kSB]), (g_pv / kSB) & 1) : false;
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (ready) {
              tc_fence_after();
              if (lane == 0) {
                const uint32_t first = g_pv == g0 ? 1u : 0u;
                // B = the page's latent blocks read MN-major (the value side of the same tile)
                const uint64_t vd = sdesc_sw128(smem_u32(sTile + (g_pv % kStages) * L::kStageBytes), 8192, 1024);
                const uint32_t p_base = tmem + S_col(g_pv % kSB, 0);
#pragma unroll
                for (int i = 0; i < kBrPerCta; ++i) {
#pragma unroll
                  for (int ks = 0; ks < 4; ++ks)
                    mma_ts(tmem + O_col(i), p_base + 64u * i + 8u * ks,
                           vd + (uint64_t)(((i * kLatPerBr) * kTileSlotBytes + ks * 2048) >> 4), kIdescPV,
                           ks == 0 ? (first ^ 1u) : 1u);
                }
                mma_commit(smem_u32(&bars->stage_empty[g_pv % kStages]));
                mma_commit(smem_u32(&bars->pv_done[g_pv % kSB]));
                MLRA_TRACE_EV(g_pv, kEvPvIssued);
              }
              __syncwarp();
              ++g_pv;
              progressed = true;
            }
          }
        }
        if constexpr (kExch) {
          // QK(g) needs S buffer g % kSB, free once PV(g - kSB) is issued; look
          // ahead at most two pages past the next PV so that PVs (which free the
          // stages) are not queued behind a run of QKs
          if (!progressed && g_qk < g_end && g_qk < g_pv + kSB && g_qk <= g_pv + 2) {
            const uint32_t st = g_qk % kStages;
            bool ready = lane == 0 ? mbar_test_wait(smem_u32(&bars->stage_full[st]), (g_qk / kStages) & 1) &&
                                         (!kExch || mbar_test_wait(smem_u32(&bars->rope_full[g_qk & 1]),
                                                                   (g_qk >> 1) & 1))
                                   : false;
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (ready) {
              if (lane == 0) MLRA_TRACE_EV(g_qk, kEvStageSeen);
              uint8_t* tile = sTile + st * L::kStageBytes;
              uint8_t* rope_tile = kExch ? sRope + (g_qk & 1) * L::kRopeTileBytes : tile + kLat * kTileSlotBytes;
              const int p = walk.pg0 + (int)(g_qk - g0);
              const int valid = min(kPage, walk.L - p * kPage);
              if (valid < kPage) {  // zero the rows past the end of the sequence
                const int nrow = kPage - valid;
                const uint4 z = make_uint4(0, 0, 0, 0);
                for (int idx = lane; idx < nrow * 8 * kLat; idx += 32) {
                  const int s = idx / (nrow * 8), rem = idx % (nrow * 8);
                  *reinterpret_cast<uint4*>(tile + s * kTileSlotBytes + (valid + rem / 8) * 128 + (rem % 8) * 16) = z;
                }
                constexpr int kRopeChunks = L::kRopeRowBytes / 16;
                for (int idx = lane; idx < nrow * kRopeChunks; idx += 32)
                  *reinterpret_cast<uint4*>(rope_tile + (valid + idx / kRopeChunks) * L::kRopeRowBytes +
                                            (idx % kRopeChunks) * 16) = z;
                fence_proxy_async_smem();
              }
              __syncwarp();
              tc_fence_after();
              if (lane == 0) {
                MLRA_TRACE_EV(g_qk, kEvQkStart);
                // descriptors = per-stage base + compile-time offsets (no per-MMA rebuild)
                const uint64_t td = sdesc_sw128(smem_u32(tile), 16, 1024);
                const uint32_t s_base = tmem + S_col(g_qk % kSB, 0);
  #pragma unroll
                for (int i = 0; i < kBrPerCta; ++i) {
  #pragma unroll
                  for (int j = 0; j < kLatPerBr; ++j) {
                    const int s = i * kLatPerBr + j;
  #pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                      const uint64_t bd = td + (uint64_t)((s * kTileSlotBytes + ks * 32) >> 4);
                      mma_ss(s_base + 64u * i, qd + (uint64_t)((s * kQSlotBytes + ks * 32) >> 4), bd, kIdescQK,
                             (j | ks) ? 1u : 0u);
                    }
                  }
                  if (kExch) {
                    const uint64_t trd = sdesc_sw64(smem_u32(rope_tile), 512);
  #pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
                      mma_ss(s_base + 64u * i, qrd + (uint64_t)(ks * 2), trd + (uint64_t)(ks * 2), kIdescQK, 1u);
                  } else {
  #pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                      mma_ss(s_base + 64u * i, qrd + (uint64_t)(ks * 2),
                             td + (uint64_t)((kLat * kTileSlotBytes + ks * 32) >> 4), kIdescQK, 1u);
                  }
                }
                mma_commit(smem_u32(&bars->s_full[g_qk % kSB]));
                if (kExch) mma_commit(smem_u32(&bars->rope_empty[g_qk & 1]));
                MLRA_TRACE_EV(g_qk, kEvQkIssued);
                if (g_qk + 1 == g_end) mma_commit(smem_u32(&bars->q_empty));  // last read of this Q
              }
              __syncwarp();
              ++g_qk;
              progressed = true;
            }
          }
        }
        if (progressed) {
          t_idle = 0;
        } else {
          if (*abort_flag) {
            ok = false;
            break;
          }
          if (t_idle == 0) t_idle = clock64();
          if (clock64() - t_idle > kWaitCycles) {
            if (lane == 0) {
              *abort_flag = 1;
              report_error(err, kErrTimeout, kSiteMma, (int)blockIdx.x);
            }
            ok = false;
            break;
          }
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      g = g_end;
      ++seg;
    }
  } else if (kExch && warp >= 6) {
    // ------------------------------------------------------------- exchange
    // MLA: send this CTA's partial scores of every page (fp16, its 32 rows)
    // to the same warp of the peer CTA as soon as QK^T has produced them.
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const bool real = row < a.H;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t peer = rank ^ 1u;
    if (q4 * 32 < a.H) {
      const uint32_t dst = map_to_cta(smem_u32(sX), peer);
      const uint32_t dst_r = map_to_cta(smem_u32(sXR), peer);
      const uint32_t bar = map_to_cta(smem_u32(&bars->x_full[q4]), peer);
      SegWalk walk(plan, a.B, maxL);
      uint32_t g = 0;
      bool ok = true;
      while (ok && walk.next(seq_lens)) {
        for (int p = walk.pg0; p < walk.pg1; ++p, ++g) {
          if (!mbar_wait_warp(smem_u32(&bars->s_full[g % kSB]), (g / kSB) & 1, abort_flag, err, kSiteSFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t lo[32], hi[32];
          tmem_ld32x2(tmem + lane_off + S_col(g % kSB, 0), tmem + lane_off + S_col(g % kSB, 0) + 32u, lo, hi);
          tc_fence_before();
          __syncwarp();
          // S(g) may now be overwritten by P(g).  One barrier per S buffer: the
          // softmax warp's wait for page g then sees at most one phase ahead
          // (page g + kSB needs QK(g + kSB), hence P(g) written).
          if (lane == 0) mbar_arrive(smem_u32(&bars->xs_read[q4][g % kSB]));
          if (row == 0) MLRA_TRACE_EV(g, kEvXLoaded);
          const int valid = min(kPage, walk.L - p * kPage);
          const float r = row_max_valid(lo, hi, valid);
          uint32_t h[32];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            h[j] = pack_f16x2(__uint_as_float(lo[2 * j]) - r, __uint_as_float(lo[2 * j + 1]) - r);
            h[16 + j] = pack_f16x2(__uint_as_float(hi[2 * j]) - r, __uint_as_float(hi[2 * j + 1]) - r);
          }
          // single buffer: the peer warp must have read my page g-1
          if (g > 0 && !mbar_wait_warp<true>(smem_u32(&bars->x_empty[q4]), (g - 1) & 1, abort_flag, err,
                                             kSiteXEmpty)) {
            ok = false;
            break;
          }
          if (row == 0) MLRA_TRACE_EV(g, kEvXEmptySeen);
          if (real) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              st_async_v4(dst + (uint32_t)((q * kHq + row) * 16), h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3],
                          bar);
            st_async_b32(dst_r + (uint32_t)(row * 4), __float_as_uint(r), bar);
          }
          if (row == 0) MLRA_TRACE_EV(g, kEvSent);
        }
      }
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int q4 = warp & 3;
    const int bi = (warp - 2) >> 2;  // branch of this warpgroup (0 unless 2 branches per CTA)
    const int row = q4 * 32 + lane;  // head
    const bool real = row < a.H;
    const bool warp_real = q4 * 32 < a.H;  // warp-uniform: some lane holds a real head
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t peer = rank ^ 1u;
    const int q_rows = a.H - q4 * 32 < 0 ? 0 : (a.H - q4 * 32 > 32 ? 32 : a.H - q4 * 32);
    SegWalk walk(plan, a.B, maxL);
    uint32_t g = 0;
    bool ok = true;

    while (ok && walk.next(seq_lens)) {
      const uint32_t g0 = g, g_end = g + (uint32_t)(walk.pg1 - walk.pg0);
      float m_run = -INFINITY, l_run = 0.f;
      for (; g < g_end; ++g) {
        const int valid = min(kPage, walk.L - (walk.pg0 + (int)(g - g0)) * kPage);
        float cur[64];
        if (!mbar_wait_warp(smem_u32(&bars->s_full[g % kSB]), (g / kSB) & 1, abort_flag, err, kSiteSFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (row == 0) MLRA_TRACE_EV(g, kEvSReady);
        if (warp_real) {
          uint32_t lo[32], hi[32];
          tmem_ld32x2(tmem + lane_off + S_col(g % kSB, bi), tmem + lane_off + S_col(g % kSB, bi) + 32u, lo, hi);
#pragma unroll
          for (int n = 0; n < 32; ++n) {
            cur[n] = __uint_as_float(lo[n]);
            cur[n + 32] = __uint_as_float(hi[n]);
          }
        }
        if (kExch && warp_real) {
          // s = f16(mine) + f16(peer's): the same bits on both CTAs of the pair
          if (row == 0) MLRA_TRACE_EV(g, kEvXFullWait);
          if (!mbar_wait_warp<true>(smem_u32(&bars->x_full[q4]), g & 1, abort_flag, err, kSiteXFull)) {
            ok = false;
            break;
          }
          if (row == 0) MLRA_TRACE_EV(g, kEvRecv);
          if (real) {
            // s = (r_own + r_peer) + (f16(s_own - r_own) + f16(s_peer - r_peer)), the offsets added as an
            // fp16 pair; each sum has the same operands on both CTAs, in the other order, so both get the
            // same bits (the exchange warp packed f16(s_own - r_own) the same way for the peer)
            const float r_own = row_max_valid(cur, valid);
            const float r_sum = r_own + sXR[row];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint4 v = *reinterpret_cast<const uint4*>(sX + (q * kHq + row) * 16);
              const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float2 d = unpack_f16x2(
                    add_f16x2(pack_f16x2(cur[8 * q + 2 * j] - r_own, cur[8 * q + 2 * j + 1] - r_own), w[j]));
                cur[8 * q + 2 * j] = r_sum + d.x;
                cur[8 * q + 2 * j + 1] = r_sum + d.y;
              }
            }
          }
          if (row == 0) MLRA_TRACE_EV(g, kEvRecvAdded);
          // page g consumed: arm the next phase, then let the peer refill the buffer
          __syncwarp();
          if (lane == 0) {
            mbar_expect_tx(smem_u32(&bars->x_full[q4]), (uint32_t)q_rows * (128u + 4u));
            mbar_arrive_cluster(map_to_cta(smem_u32(&bars->x_empty[q4]), peer));
          }
        }
        uint32_t P[32];
        float corr = 1.f;
        bool rescale = false;
        if (warp_real) {
          rescale = softmax_page(cur, valid, g == g0, m_run, l_run, corr);
          if (row == 0) MLRA_TRACE_EV(g, kEvSoftmaxDone);
#pragma unroll
          for (int j = 0; j < 32; ++j) P[j] = pack_bf16x2(cur[2 * j], cur[2 * j + 1]);
        }
        if (row == 0) MLRA_TRACE_EV(g, kEvMath);
        // O is rescaled only when the running max jumped; that needs PV(g-1)
        // complete.  PV(g-1) signals pv_done[(g-1) % kSB]; that barrier is at
        // most one phase from this target (PV(g-1-kSB) finished before QK(g-1),
        // whose scores were read, and PV(g-1+kSB) needs a P not yet written),
        // so its parity identifies PV(g-1) without waiting on every page.
        if (g > g0 && warp_real && __any_sync(0xffffffffu, rescale)) {
          if (!mbar_wait_warp(smem_u32(&bars->pv_done[(g - 1) % kSB]), ((g - 1) / kSB) & 1, abort_flag, err,
                              kSitePvDone)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int cc = 0; cc < kPvN; cc += 32) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + O_col(bi) + cc, o);
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * corr);
            tmem_st32(tmem + lane_off + O_col(bi) + cc, o);
          }
        }
        if (warp_real) {
          // MLA: the exchange warp must have read S(g) before P(g) overwrites it
          if (kExch && !mbar_wait_warp(smem_u32(&bars->xs_read[q4][g % kSB]), (g / kSB) & 1, abort_flag, err,
                                       kSiteSFull)) {
            ok = false;
            break;
          }
          tmem_st32(tmem + lane_off + S_col(g % kSB, bi), P);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[g % kSB]));
        if (row == 0) MLRA_TRACE_EV(g, kEvPReady);
      }
      if (!ok) break;
      // epilogue: O and (m, l) of this piece to its slot
      if (!mbar_wait_warp(smem_u32(&bars->pv_done[(g - 1) % kSB]), ((g - 1) / kSB) & 1, abort_flag, err,
                          kSitePvDone))
        break;
      tc_fence_after();
      const int slot = c + walk.b;
      if (warp_real) {
        for (int cc = 0; cc < kPvN; cc += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + O_col(bi) + cc, o);
          if (real) {
            const int d0 = kOCols * (int)rank + (int)O_col(bi) + cc;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int d = d0 + 8 * q;
              float4* dst = reinterpret_cast<float4*>(o_part + ((size_t)slot * a.H + row) * a.d_c + d);
              dst[0] = make_float4(__uint_as_float(o[8 * q]), __uint_as_float(o[8 * q + 1]),
                                   __uint_as_float(o[8 * q + 2]), __uint_as_float(o[8 * q + 3]));
              dst[1] = make_float4(__uint_as_float(o[8 * q + 4]), __uint_as_float(o[8 * q + 5]),
                                   __uint_as_float(o[8 * q + 6]), __uint_as_float(o[8 * q + 7]));
            }
          }
        }
        if (real && (!kExch || rank == 0)) {
          const int br = kExch ? 0 : (int)rank * kBrPerCta + bi;
          ml_part[(((size_t)slot * a.n_branch + br) * 2 + 0) * a.H + row] = m_run;
          ml_part[(((size_t)slot * a.n_branch + br) * 2 + 1) * a.H + row] = l_run;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->o_free));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (kExch) cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
#ifdef MLRA_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 1024) g_span[blockIdx.x][1] = globaltimer_ns();
#endif
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------
template <bool kExch, int kBrPerCta, int kHq, int kCtas>
cudaError_t launch_variant(const CUtensorMap& tq, const CUtensorMap& tqr, const CUtensorMap& tl, const CUtensorMap& tr,
                           const int* page_table,
                           const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                           cudaStream_t st, bool pdl) {
  auto kern = attend_tc_kernel<kExch, kBrPerCta, kHq, kCtas>;
  const int smem = Layout<kExch, kHq, kCtas>::kBytes;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  if (min_blocks<kCtas>() > 1) {  // the whole unified L1/shared array as shared memory: two CTAs per SM
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributePreferredSharedMemoryCarveout,
                             100);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kCtas * a.G, 1, 1);
  cfg.blockDim = dim3(threads_of<kExch, kBrPerCta>(), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kExch ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, tqr, tl, tr, page_table, seq_lens, o_part, ml_part, err, a);
}

}  // namespace

bool tc_supported(int dtype, int H, int d_c, int d_r, int n_branch, int /*d_h*/, int /*d_v*/) {
  if (dtype != 1) return false;
  if (tc_branch_supported(H, d_c, d_r, n_branch)) return true;
  return d_c == 512 && d_r == 64 && H >= 1 && H <= kTcHeads && (n_branch == 1 || n_branch == 2 || n_branch == 4);
}

cudaError_t launch_attend_tc(const void* q_ws, const void* lat, const void* rop, const int* page_table,
                             const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                             cudaStream_t st, bool pdl) {
  if (tc_small_supported(a.H, a.n_branch))  // MLA with at most 32 heads: attn_small.cu
    return launch_attend_tc_small(q_ws, lat, rop, page_table, seq_lens, o_part, ml_part, err, a, st, pdl);
  if (tc_branch_supported(a.H, a.d_c, a.d_r, a.n_branch))  // 128-dim branches: attn_branch.cu
    return launch_attend_tc_branch(q_ws, lat, rop, page_table, seq_lens, o_part, ml_part, err, a, st, pdl);
  CUtensorMap tq, tqr, tl, tr;
  const bool exch = a.n_branch == 1;
  if (!tmap_2d(&tq, q_ws, (uint64_t)(a.d_c + a.d_r), (uint64_t)a.B * a.H, 64, (uint32_t)a.H) ||
      !tmap_2d(&tl, lat, (uint64_t)a.d_c, (uint64_t)a.num_pages * kPage, 64, 64))
    return cudaErrorInvalidValue;
  if (exch) {  // each CTA of the pair takes half of the rope dims
    if (!tmap_2d_sw64(&tqr, q_ws, (uint64_t)(a.d_c + a.d_r), (uint64_t)a.B * a.H, 32, (uint32_t)a.H) ||
        !tmap_2d_sw64(&tr, rop, (uint64_t)a.d_r, (uint64_t)a.num_pages * kPage, 32, 64))
      return cudaErrorInvalidValue;
  } else {
    tqr = tq;
    if (!tmap_2d(&tr, rop, (uint64_t)a.d_r, (uint64_t)a.num_pages * kPage, 64, 64)) return cudaErrorInvalidValue;
  }
#define MLRA_LAUNCH(E, BR, HQ, CTAS) \
  launch_variant<E, BR, HQ, CTAS>(tq, tqr, tl, tr, page_table, seq_lens, o_part, ml_part, err, a, st, pdl)
  const bool small = a.H <= 32;  // compact query buffers, deeper ring
  switch (a.n_branch) {
    case 1: return MLRA_LAUNCH(true, 1, 128, 2);
    case 2: return small ? MLRA_LAUNCH(false, 1, 32, 2) : MLRA_LAUNCH(false, 1, 128, 2);
    // MLRA-4 at full head count: four one-branch CTAs per worker, two per SM
    case 4: return small ? MLRA_LAUNCH(false, 2, 32, 2) : MLRA_LAUNCH(false, 1, 128, 4);
    default: return cudaErrorInvalidValue;
  }
#undef MLRA_LAUNCH
}

const char* tc_variant_name(int H, int d_c, int n_branch) {
  if (tc_branch_supported(H, d_c, 64, n_branch))
    return n_branch == 1 ? "attend_tc_branch_kernel<mla over a 128-dim latent, two-page units>"
                         : (n_branch == 2 ? "attend_tc_branch_kernel<mlra-2, one branch per cta, two-page units>"
                                          : "attend_tc_branch_kernel<mlra-4, one branch per cta, two-page units>");
  const bool small = H <= 32;
  switch (n_branch) {
    case 1: return small ? "attend_tc_small_kernel<mla, cta pair, head-replicated query>"
                         : "attend_tc_kernel<mla, cta pair>";
    case 2: return small ? "attend_tc_kernel<mlra-2, cta pair, 32 query rows>" : "attend_tc_kernel<mlra-2, cta pair>";
    case 4: return small ? "attend_tc_kernel<mlra-4, cta pair, 32 query rows>"
                         : "attend_tc_kernel<mlra-4, four ctas, two per sm>";
    default: return "none";
  }
}

void tc_shutdown() { host_cache_clear(); }

#ifdef MLRA_TRACE
// Copies the pipeline trace of the last attention launch (trace builds only).
extern "C" __attribute__((visibility("default"))) int mlra_trace_read(unsigned long long* host, size_t n) {
  const size_t bytes = sizeof(g_trace) < n * sizeof(unsigned long long) ? sizeof(g_trace) : n * sizeof(unsigned long long);
  return (int)cudaMemcpyFromSymbol(host, g_trace, bytes);
}
extern "C" __attribute__((visibility("default"))) int mlra_span_read(unsigned long long* host, size_t n) {
  const size_t bytes = sizeof(g_span) < n * sizeof(unsigned long long) ? sizeof(g_span) : n * sizeof(unsigned long long);
  return (int)cudaMemcpyFromSymbol(host, g_span, bytes);
}
#endif

}  // namespace mlra
