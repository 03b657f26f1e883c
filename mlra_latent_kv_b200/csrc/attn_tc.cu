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
//     every cache tile); TMEM then also holds a double-buffered S.
//   * MLA (one softmax over all 512 dims): CTA r computes the partial scores
//     of its 256 dims (CTA 0 adds the rope part) and the two partials are
//     exchanged through distributed shared memory, so both CTAs hold the same
//     full S and compute bit-identical softmax weights.
//   * MLRA with 2 or 4 branches: the branches of a CTA are wholly its own, so
//     the pair never talks; each CTA adds the full rope score to its branches.
//   * Per 64-token page: one TMA producer warp loads the page's latent dims
//     and rope key (128-byte swizzle) into a stage ring; one MMA warp issues
//     QK^T (A = queries in smem, B = tile K-major) into S in TMEM, and PV with
//     A = P in TMEM and B = the same smem tile read MN-major; four softmax
//     warps (one TMEM lane quarter each, one head per thread) read S, apply
//     the online softmax (rescaling O only when the running max grows by more
//     than 2^8), and write P (bf16) back over S.
//   * Rows past the sequence end in the last page are zeroed in shared memory
//     before the MMAs read them (a NaN there would poison P.V even at P = 0).
// The split plan, partial-result layout and combine are those of the CUDA-core
// kernel (slot c + b, running max in log2 units).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "attn_tc.h"
#include "ptx.cuh"

namespace mlra {
namespace {

using namespace ptx;

constexpr int kThreads = 192;             // warp 0: TMA, warp 1: MMA, warps 2-5: softmax
constexpr int kQSlotBytes = 128 * 128;    // 128 query rows x 64 bf16
constexpr int kTileSlotBytes = 64 * 128;  // 64 tokens x 64 bf16
constexpr int kSlots = 5;                 // 4 latent blocks of 64 dims + the rope block
constexpr uint32_t kTmemCols = 512;
constexpr int kXBytes = 64 * 128 * 4;     // one page of fp32 partial scores, 128 rows
constexpr float kRescaleLog2 = 8.f;

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t stage_full[3], stage_empty[3];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, o_free;
  uint64_t x_full, x_empty;
  WorkerPlan plan;
  uint32_t tmem_base;
  int abort_flag;
};

template <bool kExch>
struct Layout {
  static constexpr int kStages = kExch ? 2 : 3;
  static constexpr int kQ = 0;
  static constexpr int kTile = kSlots * kQSlotBytes;
  static constexpr int kX = kTile + kStages * kSlots * kTileSlotBytes;
  static constexpr int kBars = kX + (kExch ? kXBytes : 0);
  static constexpr int kBytes = kBars + (int)sizeof(Bars) + 1024;  // + alignment slack
};

// wait-site codes recorded with a timeout
enum { kSiteQEmpty = 1, kSiteStageEmpty, kSiteQFull, kSiteStageFull, kSitePFull, kSiteOFree, kSiteSFull,
       kSiteXEmpty, kSiteXFull, kSitePvDone };

template <bool kExch, int kBrPerCta>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_lat,
                     const __grid_constant__ CUtensorMap tm_rope, const int* __restrict__ page_table,
                     const int* __restrict__ seq_lens, float* __restrict__ o_part, float* __restrict__ ml_part,
                     int* __restrict__ err, AttnArgs a) {
  using L = Layout<kExch>;
  constexpr int kStages = L::kStages;
  constexpr int kLatPerBr = 4 / kBrPerCta;      // latent slots per branch
  constexpr int kPvN = 256 / kBrPerCta;         // PV output columns per branch
  constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, false, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kPvN, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sTile = smem + L::kTile;
  uint8_t* sX = smem + L::kX;
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBars);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = kExch ? cluster_ctarank() : (blockIdx.x & 1u);
  const int c = blockIdx.x >> 1;
  const bool has_rope = kExch ? (rank == 0) : true;
  const int n_slots = has_rope ? 5 : 4;
  const int maxL = a.maxp * kPage;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->q_empty), 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(smem_u32(&bars->stage_full[s]), 1);
      mbar_init(smem_u32(&bars->stage_empty[s]), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(smem_u32(&bars->s_full[k]), 1);
      mbar_init(smem_u32(&bars->p_full[k]), 4);
    }
    mbar_init(smem_u32(&bars->pv_done), 1);
    mbar_init(smem_u32(&bars->o_free), 4);
    mbar_init(smem_u32(&bars->x_full), 128);
    mbar_init(smem_u32(&bars->x_empty), 128);
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

  auto S_col = [](uint32_t buf, int i) -> uint32_t { return 256u + buf * 128u + (uint32_t)i * 64u; };
  auto O_col = [](int i) -> uint32_t { return (uint32_t)i * (uint32_t)kPvN; };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_lat);
      tma_prefetch_desc(&tm_rope);
      SegWalk walk(plan, a.B, maxL);
      int seg = 0;
      uint32_t g = 0;
      bool ok = true;
      while (ok && walk.next(seq_lens)) {
        if (seg > 0 && !mbar_wait(smem_u32(&bars->q_empty), (seg - 1) & 1, abort_flag, err, kSiteQEmpty)) break;
        const uint32_t qb = smem_u32(&bars->q_full);
        mbar_expect_tx(qb, n_slots * kQSlotBytes);
        for (int s = 0; s < 4; ++s)
          tma_load_2d(smem_u32(sQ + s * kQSlotBytes), &tm_q, qb, 64 * (4 * (int)rank + s), walk.b * 128);
        if (has_rope) tma_load_2d(smem_u32(sQ + 4 * kQSlotBytes), &tm_q, qb, a.d_c, walk.b * 128);
        for (int p = walk.pg0; p < walk.pg1; ++p, ++g) {
          const uint32_t st = g % kStages, use = g / kStages;
          if (use > 0 && !mbar_wait(smem_u32(&bars->stage_empty[st]), (use - 1) & 1, abort_flag, err,
                                    kSiteStageEmpty)) {
            ok = false;
            break;
          }
          const int pg = page_of(page_table, a.maxp, a.num_pages, walk.b, p * kPage, err);
          const uint32_t fb = smem_u32(&bars->stage_full[st]);
          uint8_t* tile = sTile + st * (kSlots * kTileSlotBytes);
          mbar_expect_tx(fb, n_slots * kTileSlotBytes);
          for (int s = 0; s < 4; ++s)
            tma_load_2d(smem_u32(tile + s * kTileSlotBytes), &tm_lat, fb, 64 * (4 * (int)rank + s), pg * kPage);
          if (has_rope) tma_load_2d(smem_u32(tile + 4 * kTileSlotBytes), &tm_rope, fb, 0, pg * kPage);
        }
        ++seg;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    SegWalk walk(plan, a.B, maxL);
    int seg = 0;
    uint32_t g = 0;
    bool ok = true;
    auto issue_pv = [&](uint32_t gg, bool first) -> bool {
      if (first && seg > 0 &&
          !mbar_wait_warp(smem_u32(&bars->o_free), (seg - 1) & 1, abort_flag, err, kSiteOFree))
        return false;
      if (!mbar_wait_warp(smem_u32(&bars->p_full[gg & 1]), (gg >> 1) & 1, abort_flag, err, kSitePFull)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t tile = smem_u32(sTile + (gg % kStages) * (kSlots * kTileSlotBytes));
#pragma unroll
        for (int i = 0; i < kBrPerCta; ++i) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t bd = sdesc_sw128(tile + (i * kLatPerBr) * kTileSlotBytes + ks * 2048, 8192, 1024);
            mma_ts(tmem + O_col(i), tmem + S_col(gg & 1, i) + 8u * ks, bd, kIdescPV, (first && ks == 0) ? 0u : 1u);
          }
        }
        mma_commit(smem_u32(&bars->stage_empty[gg % kStages]));
        mma_commit(smem_u32(&bars->pv_done));
      }
      __syncwarp();
      return true;
    };
    while (ok && walk.next(seq_lens)) {
      if (!mbar_wait_warp(smem_u32(&bars->q_full), seg & 1, abort_flag, err, kSiteQFull)) break;
      tc_fence_after();
      const uint32_t g0 = g;
      for (int p = walk.pg0; p < walk.pg1; ++p, ++g) {
        const uint32_t st = g % kStages, use = g / kStages;
        if (!mbar_wait_warp(smem_u32(&bars->stage_full[st]), use & 1, abort_flag, err, kSiteStageFull)) {
          ok = false;
          break;
        }
        uint8_t* tile = sTile + st * (kSlots * kTileSlotBytes);
        const int valid = min(kPage, walk.L - p * kPage);
        if (valid < kPage) {  // zero the rows past the end of the sequence
          const int nrow = kPage - valid;
          const uint4 z = make_uint4(0, 0, 0, 0);
          for (int idx = lane; idx < nrow * 8 * n_slots; idx += 32) {
            const int s = idx / (nrow * 8), rem = idx % (nrow * 8);
            *reinterpret_cast<uint4*>(tile + s * kTileSlotBytes + (valid + rem / 8) * 128 + (rem % 8) * 16) = z;
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        tc_fence_after();
        if (lane == 0) {
          const uint32_t qa = smem_u32(sQ), ta = smem_u32(tile);
#pragma unroll
          for (int i = 0; i < kBrPerCta; ++i) {
            uint32_t kk = 0;
            for (int j = 0; j < kLatPerBr + (has_rope ? 1 : 0); ++j) {
              const int s = j < kLatPerBr ? i * kLatPerBr + j : 4;
#pragma unroll
              for (int ks = 0; ks < 4; ++ks, ++kk) {
                const uint64_t ad = sdesc_sw128(qa + s * kQSlotBytes + ks * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(ta + s * kTileSlotBytes + ks * 32, 16, 1024);
                mma_ss(tmem + S_col(g & 1, i), ad, bd, kIdescQK, kk > 0 ? 1u : 0u);
              }
            }
          }
          mma_commit(smem_u32(&bars->s_full[g & 1]));
        }
        __syncwarp();
        if (g > g0 && !issue_pv(g - 1, g - 1 == g0)) {
          ok = false;
          break;
        }
      }
      if (!ok || g == g0) break;
      if (!issue_pv(g - 1, g - 1 == g0)) break;
      if (lane == 0) mma_commit(smem_u32(&bars->q_empty));
      __syncwarp();
      ++seg;
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;  // head
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t peer = rank ^ 1u;
    const uint32_t x_remote = kExch ? map_to_cta(smem_u32(sX), peer) : 0u;
    const uint32_t xfull_remote = kExch ? map_to_cta(smem_u32(&bars->x_full), peer) : 0u;
    const uint32_t xempty_remote = kExch ? map_to_cta(smem_u32(&bars->x_empty), peer) : 0u;
    SegWalk walk(plan, a.B, maxL);
    uint32_t g = 0;
    bool ok = true;
    while (ok && walk.next(seq_lens)) {
      const uint32_t g0 = g;
      float m_run[kBrPerCta], l_run[kBrPerCta];
#pragma unroll
      for (int i = 0; i < kBrPerCta; ++i) {
        m_run[i] = -INFINITY;
        l_run[i] = 0.f;
      }
      for (int p = walk.pg0; p < walk.pg1; ++p, ++g) {
        const int valid = min(kPage, walk.L - p * kPage);
        if (!mbar_wait_warp(smem_u32(&bars->s_full[g & 1]), (g >> 1) & 1, abort_flag, err, kSiteSFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t P[kBrPerCta][32];
        float corr[kBrPerCta];
        bool rescale = false;
#pragma unroll
        for (int i = 0; i < kBrPerCta; ++i) {
          uint32_t lo[32], hi[32];
          tmem_ld32(tmem + lane_off + S_col(g & 1, i), lo);
          tmem_ld32(tmem + lane_off + S_col(g & 1, i) + 32u, hi);
          if (kExch) {
            // send my partial scores to the peer, receive and add its partial
            if (g > 0 && !mbar_wait_warp<true>(smem_u32(&bars->x_empty), (g - 1) & 1, abort_flag, err, kSiteXEmpty)) {
              ok = false;
              break;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
              st_cluster_v4(x_remote + (uint32_t)((q * 128 + row) * 16), lo[4 * q], lo[4 * q + 1], lo[4 * q + 2],
                            lo[4 * q + 3]);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              st_cluster_v4(x_remote + (uint32_t)(((8 + q) * 128 + row) * 16), hi[4 * q], hi[4 * q + 1],
                            hi[4 * q + 2], hi[4 * q + 3]);
            mbar_arrive_cluster(xfull_remote);
            if (!mbar_wait_warp<true>(smem_u32(&bars->x_full), g & 1, abort_flag, err, kSiteXFull)) {
              ok = false;
              break;
            }
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float4 v = *reinterpret_cast<const float4*>(sX + (q * 128 + row) * 16);
              uint32_t* d = q < 8 ? &lo[4 * q] : &hi[4 * (q - 8)];
              d[0] = __float_as_uint(__uint_as_float(d[0]) + v.x);
              d[1] = __float_as_uint(__uint_as_float(d[1]) + v.y);
              d[2] = __float_as_uint(__uint_as_float(d[2]) + v.z);
              d[3] = __float_as_uint(__uint_as_float(d[3]) + v.w);
            }
            mbar_arrive_cluster(xempty_remote);
          }
          // online softmax over this page (log2 domain)
          float s[64];
          float mx = -INFINITY;
#pragma unroll
          for (int n = 0; n < 64; ++n) {
            const float raw = __uint_as_float(n < 32 ? lo[n] : hi[n - 32]);
            s[n] = n < valid ? raw * a.scale_log2 : -INFINITY;
            mx = fmaxf(mx, s[n]);
          }
          float m_use;
          if (g == g0) {
            m_use = mx;
            corr[i] = 0.f;
          } else if (mx > m_run[i] + kRescaleLog2) {
            m_use = mx;
            corr[i] = ex2(m_run[i] - mx);
            rescale = true;
          } else {
            m_use = m_run[i];
            corr[i] = 1.f;
          }
          float sum = 0.f;
#pragma unroll
          for (int n = 0; n < 64; ++n) {
            s[n] = ex2(s[n] - m_use);
            sum += s[n];
          }
          l_run[i] = l_run[i] * corr[i] + sum;
          m_run[i] = m_use;
#pragma unroll
          for (int j = 0; j < 32; ++j) P[i][j] = pack_bf16x2(s[2 * j], s[2 * j + 1]);
        }
        if (!ok) break;
        if (g > g0) {
          if (!mbar_wait_warp(smem_u32(&bars->pv_done), (g - 1) & 1, abort_flag, err, kSitePvDone)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
            for (int i = 0; i < kBrPerCta; ++i) {
              for (int cc = 0; cc < kPvN; cc += 32) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + O_col(i) + cc, o);
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * corr[i]);
                tmem_st32(tmem + lane_off + O_col(i) + cc, o);
              }
            }
          }
        }
#pragma unroll
        for (int i = 0; i < kBrPerCta; ++i) tmem_st32(tmem + lane_off + S_col(g & 1, i), P[i]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[g & 1]));
      }
      if (!ok || g == g0) break;
      // epilogue: O and (m, l) of this piece to its slot
      if (!mbar_wait_warp(smem_u32(&bars->pv_done), (g - 1) & 1, abort_flag, err, kSitePvDone)) break;
      tc_fence_after();
      const int slot = c + walk.b;
      const bool real = row < a.H;
#pragma unroll
      for (int i = 0; i < kBrPerCta; ++i) {
        for (int cc = 0; cc < kPvN; cc += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + O_col(i) + cc, o);
          if (real) {
            const int d0 = 256 * (int)rank + (int)O_col(i) + cc;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int d = d0 + 4 * q;
              float4 v = make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                                     __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3]));
              *reinterpret_cast<float4*>(o_part + (((size_t)slot * (a.d_c / 4) + d / 4) * a.H + row) * 4) = v;
            }
          }
        }
        if (real && (!kExch || rank == 0)) {
          const int br = kExch ? 0 : (int)rank * kBrPerCta + i;
          ml_part[(((size_t)slot * a.n_branch + br) * 2 + 0) * a.H + row] = m_run[i];
          ml_part[(((size_t)slot * a.n_branch + br) * 2 + 1) * a.H + row] = l_run[i];
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
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// 2-D bf16 map over rows x cols (cols contiguous), box = box_cols x box_rows, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kExch, int kBrPerCta>
cudaError_t launch_variant(const CUtensorMap& tq, const CUtensorMap& tl, const CUtensorMap& tr, const int* page_table,
                           const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                           cudaStream_t st) {
  auto kern = attend_tc_kernel<kExch, kBrPerCta>;
  const int smem = Layout<kExch>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.G, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kExch ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tq, tl, tr, page_table, seq_lens, o_part, ml_part, err, a);
}

}  // namespace

bool tc_supported(int dtype, int H, int d_c, int d_r, int n_branch, int /*d_h*/, int /*d_v*/) {
  return dtype == 1 && d_c == 512 && d_r == 64 && H >= 1 && H <= kTcHeads &&
         (n_branch == 1 || n_branch == 2 || n_branch == 4);
}

cudaError_t launch_attend_tc(const void* q_ws, const void* lat, const void* rop, const int* page_table,
                             const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                             cudaStream_t st) {
  cudaError_t e = get_encoder();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tl, tr;
  if (!make_map(&tq, q_ws, (uint64_t)(a.d_c + a.d_r), (uint64_t)a.B * kTcHeads, 64, 128) ||
      !make_map(&tl, lat, (uint64_t)a.d_c, (uint64_t)a.num_pages * kPage, 64, 64) ||
      !make_map(&tr, rop, (uint64_t)a.d_r, (uint64_t)a.num_pages * kPage, 64, 64))
    return cudaErrorInvalidValue;
  switch (a.n_branch) {
    case 1: return launch_variant<true, 1>(tq, tl, tr, page_table, seq_lens, o_part, ml_part, err, a, st);
    case 2: return launch_variant<false, 1>(tq, tl, tr, page_table, seq_lens, o_part, ml_part, err, a, st);
    case 4: return launch_variant<false, 2>(tq, tl, tr, page_table, seq_lens, o_part, ml_part, err, a, st);
    default: return cudaErrorInvalidValue;
  }
}

void tc_shutdown() {}

}  // namespace mlra
