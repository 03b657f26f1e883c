// tcgen05 kernels for the two small per-head contractions of the decode step
// (yololab.net, "超越 GQA 的推理革命…", section "矩陣吸收": W_UK is folded into
// the query before attention and W_UV applied after it):
//
//   a2  q_lat[b, h, :] = q_nope[b, h, :] . W_UK[h]        (+ RoPE of q_rope)
//   a4+a5  o_lat[b, h, :] = combine of the split-KV partials of (b, h)
//          out[b, h, :]   = o_lat[b, h, :] . W_UV[h]
//
// Both are weight-bandwidth bound (every weight is read once per step and used
// for B rows), so they run "swap-AB": the weight is the M x K operand (M =
// latent or value dims, MN-major straight from its row-major layout by TMA),
// the batch is N (padded to a multiple of 16 with TMA zero fill), and one CTA
// per (head, 128-row M tile) streams its weight slice once (the up-projection:
// once per block of 16 sequences, the repeats from L2).  The combine is fused
// into the up-projection: the CTA of head h merges the partials of its
// sequences into bf16 rows of the MMA's B operand in shared memory, so o_lat
// never goes to HBM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "gemm_tc.h"
#include "host_cache.h"
#include "ptx.cuh"

namespace mlra {
namespace {

using namespace ptx;

// Optional phase trace (builds with -DMLRA_TRACE only): globaltimer stamps of
// each CTA's phases, [kernel][cta][event].
#ifdef MLRA_TRACE
__device__ unsigned long long g_gtrace[2][1024][8];
#define GEMM_TRACE(k, ev)                                                                      \
  do {                                                                                         \
    const int cta_ = blockIdx.x * gridDim.y + blockIdx.y;                                      \
    if (threadIdx.x == 0 && cta_ < 1024) g_gtrace[k][cta_][ev] = globaltimer_ns();              \
  } while (0)
#else
#define GEMM_TRACE(k, ev) \
  do {                    \
  } while (0)
#endif

// 128-byte-swizzled K-major tile of `rows` rows x 64 bf16: byte offset of the
// 16-byte chunk (row, chunk) -- the layout TMA writes and the MMA reads.
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t tmem_cols_for(int n) {
  uint32_t c = 32;
  while ((int)c < n) c <<= 1;
  return c;
}

// ---------------------------------------------------------------------------
// a2: query absorption.  grid (H, d_c / 128), block 128.
//   A (M = 128 latent dims, K = d_h) = W_UK[h][:, m0:m0+128]   MN-major
//   B (N = Bp batch rows, K = d_h)   = q_nope[:, h, :]          K-major
//   D (TMEM, 128 lanes x Bp)         -> q_ws[b][h][m0 + lane] (bf16)
// Block (h, 0) also rotates q_rope[:, h] into q_ws[b][h][d_c:].
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128, 1)
    absorb_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_q,
                     const __nv_bfloat16* __restrict__ q_rope, const int* __restrict__ q_pos,
                     __nv_bfloat16* __restrict__ q_ws, int* __restrict__ err, GemmArgs a, RopeTable tab) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int a_bytes = 2 * a.K * 128;          // two 64-column M blocks of K rows
  uint8_t* sA = smem;
  uint8_t* sB = smem + a_bytes;               // K/64 blocks of Bp rows
  __shared__ uint64_t full_bar, done_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int h = blockIdx.x, m0 = blockIdx.y * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ncols = tmem_cols_for(a.Bp);
  grid_dep_launch();  // the attention kernel may set up as this grid retires
  GEMM_TRACE(0, 0);
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&full_bar), 1);
    mbar_init(smem_u32(&done_bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base), ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t fb = smem_u32(&full_bar);
  if (threadIdx.x == 0) {  // weights and queries in flight while the RoPE below runs
    mbar_expect_tx(fb, a_bytes + (a.K / 64) * a.Bp * 128);
    for (int mb = 0; mb < 2; ++mb) tma_load_2d(smem_u32(sA + mb * a.K * 128), &tm_w, fb, m0 + 64 * mb, h * a.K);
    for (int kb = 0; kb < a.K / 64; ++kb) tma_load_3d(smem_u32(sB + kb * a.Bp * 128), &tm_q, fb, 64 * kb, h, 0);
  }
  // RoPE of the query (independent of the MMA), spread over the head's
  // d_c/128 blocks; the loads of a thread's pairs are issued before any use
  {
    const int pairs = a.d_r / 2;
    const int n = a.B * pairs, stride = blockDim.x * gridDim.y;
    constexpr int kU = 4;
    for (int base = blockIdx.y * blockDim.x + threadIdx.x; base < n; base += kU * stride) {
      __nv_bfloat162 x[kU];
      int pos[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int idx = base + u * stride;
        if (idx < n) {
          const int b = idx / pairs, i = idx % pairs;
          x[u] = *reinterpret_cast<const __nv_bfloat162*>(q_rope + ((size_t)b * a.H + h) * a.d_r + 2 * i);
          pos[u] = __ldg(q_pos + b);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int idx = base + u * stride;
        if (idx < n) {
          const int b = idx / pairs, i = idx % pairs;
          const float x0 = __low2float(x[u]), x1 = __high2float(x[u]);
          float sn, cs;
          rope_sincos(tab, i, pos[u], &sn, &cs);
          *reinterpret_cast<__nv_bfloat162*>(q_ws + ((size_t)b * a.H + h) * (a.d_c + a.d_r) + a.d_c + 2 * i) =
              __floats2bfloat162_rn((x0 * cs - x1 * sn) * a.q_scale, (x0 * sn + x1 * cs) * a.q_scale);
        }
      }
    }
  }
  if (threadIdx.x == 0 && mbar_wait(fb, 0, &abort_flag, err, 20)) {
    GEMM_TRACE(0, 2);
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(128, a.Bp, true, false);
    const uint64_t ad0 = sdesc_sw128(smem_u32(sA), a.K * 128, 1024);
    const uint64_t bd0 = sdesc_sw128(smem_u32(sB), 16, 1024);
    const uint64_t bkb = (uint64_t)((a.Bp * 128) >> 4);
    for (int kb = 0; kb < a.K / 64; ++kb) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_ss(tmem, ad0 + (uint64_t)(kb * 4 + ks) * 128u, bd0 + kb * bkb + (uint64_t)(ks * 2), idesc,
               (kb | ks) ? 1u : 0u);
    }
    mma_commit(smem_u32(&done_bar));
  }
  GEMM_TRACE(0, 3);
  // epilogue: q_lat rows staged as bf16 in the (now free) operand space, then
  // written to q_ws with 16-byte stores (each row's 128 dims are contiguous)
  __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem);  // [Bp][128]; the launch sizes smem for it
  const bool mma_ok = mbar_wait_warp(smem_u32(&done_bar), 0, &abort_flag, err, 21);
  if (mma_ok) {
    GEMM_TRACE(0, 4);
    tc_fence_after();
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    for (int cc = 0; cc < a.Bp; cc += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + cc, v);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        stage[(size_t)(cc + j) * 128 + warp * 32 + lane] = __float2bfloat16_rn(__uint_as_float(v[j]) * a.q_scale);
    }
  }
  __syncthreads();
  if (mma_ok) {
    for (int idx = threadIdx.x; idx < a.B * 16; idx += blockDim.x) {
      const int b = idx >> 4, ch = idx & 15;
      *reinterpret_cast<uint4*>(q_ws + ((size_t)b * a.H + h) * (a.d_c + a.d_r) + m0 + ch * 8) =
          *reinterpret_cast<const uint4*>(stage + (size_t)b * 128 + ch * 8);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, ncols);
  GEMM_TRACE(0, 5);
}

// ---------------------------------------------------------------------------
// a4 + a5: split combine fused into the output up-projection.
// grid (H, d_v / 128, ceil(B / R)), block 512: a CTA takes one head, 128 value
// dims and a block of R sequences (16, or 32 when the heads alone nearly fill
// the GPU: more CTAs would re-read the weights for no gain), so that a few heads still fill
// the GPU (at H = 32 one CTA per head would leave most SMs idle, each of its
// CTAs streaming a whole head's partials).
//   A (M = 128 value dims, K = d_c)      = W_UV[h][:, m0:m0+128]  MN-major (TMA)
//   B (N = R batch rows, K = d_c)        = o_lat[b0 + n, h, :] built here in smem:
//       o_lat[b, h, br cols] = branch_scale * sum_s 2^(m_s - M) o_s / L
//   D (TMEM, 128 lanes x R)              -> out[b][h][m0 + lane] (bf16)
// ---------------------------------------------------------------------------
constexpr int kCuThreads = 512;
constexpr int kCuRowsMax = 32;   // sequences per CTA at most (the MMA's N)
constexpr int kPieceUnroll = 4;  // partials of a row fetched together

__global__ void __launch_bounds__(kCuThreads, 1)
    combine_upproj_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const float* __restrict__ o_part,
                             const float* __restrict__ ml_part, const int* __restrict__ seq_lens,
                             __nv_bfloat16* __restrict__ out, int* __restrict__ err, GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int a_bytes = 2 * a.K * 128;             // K = d_c rows, two 64-column M blocks
  const int n_ml = (a.G + a.B - 1) * a.n_branch;  // (slot, branch) pairs
  uint8_t* sB = smem + a_bytes;                  // d_c/64 blocks of R rows
  uint8_t* sA = smem;
  float* s_wt = reinterpret_cast<float*>(sB + (a.K / 64) * a.R * 128);  // [slot][n_branch] piece weights
  float* s_m = s_wt + n_ml;                                              // [slot][n_branch] running max
  float* s_l = s_m + n_ml;                                               // [slot][n_branch] sum
  int* s_c0 = reinterpret_cast<int*>(s_l + n_ml);
  int* s_c1 = s_c0 + a.B;
  int* s_ne = s_c1 + a.B;  // [G] worker has pages
  __shared__ uint64_t full_bar, done_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ long long s_T;
  const int h = blockIdx.x, m0 = blockIdx.y * 128, b0 = blockIdx.z * a.R;
  const int nb = min(a.R, a.B - b0);  // sequences of this CTA
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ncols = tmem_cols_for(a.R);
  const int maxL = a.maxp * kPage;
  GEMM_TRACE(1, 0);
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&full_bar), 1);
    mbar_init(smem_u32(&done_bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base), ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  if (threadIdx.x == 0) {  // stream the weight slice while the combine runs
    const uint32_t fb = smem_u32(&full_bar);
    mbar_expect_tx(fb, a_bytes);
    const int box_rows = a.K < 256 ? a.K : 256;
    for (int mb = 0; mb < 2; ++mb)
      for (int r = 0; r < a.K; r += box_rows)
        tma_load_2d(smem_u32(sA + mb * a.K * 128 + r * 128), &tm_w, fb, m0 + 64 * mb, h * a.K + r);
  }
  if (warp == 1) {
    // sequence -> worker range (the split plan of the attention kernel)
    long long T = 0;
    for (int base = 0; base < a.B; base += 32) {
      const int np = base + lane < a.B ? npages_of(seq_len_at(seq_lens, base + lane, maxL)) : 0;
      T += warp_sum_i(np);
    }
    long long prefix = 0;
    for (int base = 0; base < a.B; base += 32) {
      const int b = base + lane;
      const int np = b < a.B ? npages_of(seq_len_at(seq_lens, b, maxL)) : 0;
      const int incl = warp_incl_scan(np);
      if (b < a.B) {
        const long long P = prefix + incl - np;
        s_c0[b] = np > 0 ? worker_of_page(P, T, a.G) : 0;
        s_c1[b] = np > 0 ? worker_of_page(P + np - 1, T, a.G) : -1;
      }
      prefix += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_T = T;
  }
  __syncthreads();
  {
    // workers with an empty page range wrote no partial: flag them once
    const long long T = s_T;
    for (int c = threadIdx.x; c < a.G; c += blockDim.x)
      s_ne[c] = worker_start(c, T, a.G) != worker_start(c + 1, T, a.G) ? 1 : 0;
  }
  grid_dep_wait();  // the partials come from the attention kernel
  // (m, l) of the slots of this CTA's sequences, all loads in flight at once
  // (slot c + b for worker c; the sequences b0 .. b0 + nb - 1 use slots
  // s_c0[b0] + b0 .. s_c1[b0 + nb - 1] + b0 + nb - 1)
  const int slot_lo = nb > 0 ? s_c0[b0] + b0 : 0;
  int slot_hi = slot_lo - 1;
  for (int b = b0; b < b0 + nb; ++b) slot_hi = max(slot_hi, s_c1[b] + b);
  for (int i = slot_lo * a.n_branch + threadIdx.x; i < (slot_hi + 1) * a.n_branch; i += blockDim.x) {
    const size_t base = (size_t)i * 2;
    s_m[i] = ml_part[(base + 0) * a.H + h];
    s_l[i] = ml_part[(base + 1) * a.H + h];
  }
  __syncthreads();
  GEMM_TRACE(1, 1);
  // per (b, branch): weight of each piece, 2^(m_s - M) * branch_scale / L
  for (int idx = threadIdx.x; idx < nb * a.n_branch; idx += blockDim.x) {
    const int b = b0 + idx / a.n_branch, br = idx % a.n_branch;
    const int c0 = s_c0[b], c1 = s_c1[b];
    float M = -INFINITY;
    for (int c = c0; c <= c1; ++c)
      if (s_ne[c]) M = fmaxf(M, s_m[(c + b) * a.n_branch + br]);
    float Lsum = 0.f;
    for (int c = c0; c <= c1; ++c)
      if (s_ne[c]) {
        const int k = (c + b) * a.n_branch + br;
        Lsum += exp2f(s_m[k] - M) * s_l[k];
      }
    const float scale = a.branch_scale / Lsum;
    for (int c = c0; c <= c1; ++c) {
      const int k = (c + b) * a.n_branch + br;
      s_wt[k] = s_ne[c] ? exp2f(s_m[k] - M) * scale : 0.f;
    }
  }
  __syncthreads();
  GEMM_TRACE(1, 2);
  // o_lat rows (bf16) straight into the swizzled B operand; padding rows are
  // zero.  A thread takes two (row, 8-dim chunk) items at a time and fetches
  // the partials of up to kPieceUnroll pieces of both before using any.
  const int chunks = a.K / 8;
  const int d_cb = a.K / a.n_branch;
  const int n_items = a.R * chunks;
  for (int base = threadIdx.x; base < n_items; base += 2 * blockDim.x) {
    int rq[2], bq[2], chq[2], c0q[2], c1q[2], brq[2];  // local row, sequence, chunk, workers, branch
    float acc[2][8];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int idx = base + u * blockDim.x;
      rq[u] = idx < n_items ? idx / chunks : a.R;
      bq[u] = b0 + rq[u];
      chq[u] = idx % chunks;
      const bool row = rq[u] < nb;
      c0q[u] = row ? s_c0[bq[u]] : 0;
      c1q[u] = row ? s_c1[bq[u]] : -1;
      brq[u] = (chq[u] * 8) / d_cb;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[u][j] = 0.f;
    }
    const int np = max(c1q[0] - c0q[0], c1q[1] - c0q[1]) + 1;
    for (int k0 = 0; k0 < np; k0 += kPieceUnroll) {
      float4 uv[2][kPieceUnroll][2];
      float w[2][kPieceUnroll];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int k = 0; k < kPieceUnroll; ++k) {
          const int c = c0q[u] + k0 + k;
          w[u][k] = c <= c1q[u] ? s_wt[(c + bq[u]) * a.n_branch + brq[u]] : 0.f;
          if (w[u][k] != 0.f) {
            const float4* src =
                reinterpret_cast<const float4*>(o_part + ((size_t)(c + bq[u]) * a.H + h) * a.K + chq[u] * 8);
            uv[u][k][0] = src[0];
            uv[u][k][1] = src[1];
          } else {
            uv[u][k][0] = uv[u][k][1] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int k = 0; k < kPieceUnroll; ++k) {
          const float wk = w[u][k];
          acc[u][0] = fmaf(wk, uv[u][k][0].x, acc[u][0]);
          acc[u][1] = fmaf(wk, uv[u][k][0].y, acc[u][1]);
          acc[u][2] = fmaf(wk, uv[u][k][0].z, acc[u][2]);
          acc[u][3] = fmaf(wk, uv[u][k][0].w, acc[u][3]);
          acc[u][4] = fmaf(wk, uv[u][k][1].x, acc[u][4]);
          acc[u][5] = fmaf(wk, uv[u][k][1].y, acc[u][5]);
          acc[u][6] = fmaf(wk, uv[u][k][1].z, acc[u][6]);
          acc[u][7] = fmaf(wk, uv[u][k][1].w, acc[u][7]);
        }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (rq[u] >= a.R) continue;
      uint4 pk;  // rows past the batch are zero (no pieces, weights 0)
      pk.x = pack_bf16x2(acc[u][0], acc[u][1]);
      pk.y = pack_bf16x2(acc[u][2], acc[u][3]);
      pk.z = pack_bf16x2(acc[u][4], acc[u][5]);
      pk.w = pack_bf16x2(acc[u][6], acc[u][7]);
      *reinterpret_cast<uint4*>(sB + (chq[u] / 8) * a.R * 128 + sw128_off(rq[u], chq[u] % 8)) = pk;
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  GEMM_TRACE(1, 3);
  if (threadIdx.x == 0) {
    if (mbar_wait(smem_u32(&full_bar), 0, &abort_flag, err, 22)) {
      GEMM_TRACE(1, 4);
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, a.R, true, false);
      const uint64_t ad0 = sdesc_sw128(smem_u32(sA), a.K * 128, 1024);
      const uint64_t bd0 = sdesc_sw128(smem_u32(sB), 16, 1024);
      const uint64_t bkb = (uint64_t)((a.R * 128) >> 4);
      for (int kb = 0; kb < a.K / 64; ++kb) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_ss(tmem, ad0 + (uint64_t)(kb * 4 + ks) * 128u, bd0 + kb * bkb + (uint64_t)(ks * 2), idesc,
                 (kb | ks) ? 1u : 0u);
      }
      mma_commit(smem_u32(&done_bar));
    }
  }
  if (warp < 4 && mbar_wait_warp(smem_u32(&done_bar), 0, &abort_flag, err, 23)) {
    GEMM_TRACE(1, 5);
    tc_fence_after();
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    for (int cc = 0; cc < a.R; cc += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + lane_off + (uint32_t)cc, v);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (cc + j < nb)
          out[((size_t)(b0 + cc + j) * a.H + h) * a.N_out + m0 + warp * 32 + lane] =
              __float2bfloat16_rn(__uint_as_float(v[j]));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, ncols);
  GEMM_TRACE(1, 6);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
}  // namespace

bool absorb_tc_supported(int dtype, int B, int d_h, int d_c) {
  return dtype == 1 && B >= 1 && B <= 256 && d_h % 64 == 0 && d_h <= 256 && d_c % 128 == 0;
}

int batch_pad(int B) { return B <= 16 ? 16 : (B + 15) / 16 * 16; }

// Sequences per CTA: 16, or up to 32 when the heads and value blocks alone
// give most of a wave of CTAs (then a finer split only re-reads the weights).
static int combine_rows(int B, int H, int d_v) {
  return H * (d_v / 128) >= 96 ? (batch_pad(B) < kCuRowsMax ? batch_pad(B) : kCuRowsMax) : 16;
}

// shared memory: the whole W_UV[h] slice (2 x d_c x 128 B), d_c/64 x R x 128 B
// of o_lat rows (R at most kCuRowsMax), the (m, l, weight) of every slot and
// branch, two ints per sequence, one flag per worker
static size_t upproj_smem_bytes(int B, int d_c, int G, int n_branch) {
  return 1024 + (size_t)2 * d_c * 128 + (size_t)(d_c / 64) * kCuRowsMax * 128 +
         (size_t)3 * (G + B) * n_branch * 4 + (size_t)2 * B * 4 + (size_t)G * 4;
}

bool upproj_tc_supported(int dtype, int B, int d_c, int d_v, int G, int n_branch) {
  return dtype == 1 && B >= 1 && d_c % 64 == 0 && d_c <= 512 && (d_c <= 256 || d_c % 256 == 0) &&
         d_v % 128 == 0 && upproj_smem_bytes(B, d_c, G, n_branch) <= 232448;
}

cudaError_t launch_absorb_tc(const void* q_nope, const void* q_rope, const int* q_pos, const void* W_UK, void* q_ws,
                             int* err, const GemmArgs& a, const RopeTable& tab, cudaStream_t st) {
  CUtensorMap tw, tq;
  if (!tmap_2d(&tw, W_UK, (uint64_t)a.d_c, (uint64_t)a.H * a.K, 64, (uint32_t)a.K) ||
      !tmap_3d_batch(&tq, q_nope, (uint64_t)a.K, (uint64_t)a.H, (uint64_t)a.B, (uint32_t)a.Bp))
    return cudaErrorInvalidValue;
  const int operands = 2 * a.K * 128 + (a.K / 64) * a.Bp * 128;
  const int smem = 1024 + (operands > a.Bp * 256 ? operands : a.Bp * 256);  // operands, later the output stage
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(absorb_tc_kernel), smem);
  if (e != cudaSuccess) return e;
  absorb_tc_kernel<<<dim3(a.H, a.d_c / 128), 128, smem, st>>>(tw, tq, (const __nv_bfloat16*)q_rope, q_pos,
                                                              (__nv_bfloat16*)q_ws, err, a, tab);
  return cudaGetLastError();
}

cudaError_t launch_combine_upproj_tc(const float* o_part, const float* ml_part, const int* seq_lens, const void* W_UV,
                                     void* out, int* err, const GemmArgs& a, cudaStream_t st, bool pdl) {
  CUtensorMap tw;
  if (!tmap_2d(&tw, W_UV, (uint64_t)a.N_out, (uint64_t)a.H * a.K, 64, (uint32_t)(a.K < 256 ? a.K : 256)))
    return cudaErrorInvalidValue;
  GemmArgs g = a;
  g.R = combine_rows(a.B, a.H, a.N_out);
  const int smem = (int)upproj_smem_bytes(a.B, a.K, a.G, a.n_branch);
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(combine_upproj_tc_kernel), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.H, g.N_out / 128, (g.B + g.R - 1) / g.R);
  cfg.blockDim = dim3(kCuThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, combine_upproj_tc_kernel, tw, o_part, ml_part, seq_lens, (__nv_bfloat16*)out, err,
                            g);
}

#ifdef MLRA_TRACE
// Copies the phase trace of the last absorption / combine launches (trace builds only).
extern "C" __attribute__((visibility("default"))) int mlra_gemm_trace_read(unsigned long long* host, size_t n) {
  const size_t bytes =
      sizeof(g_gtrace) < n * sizeof(unsigned long long) ? sizeof(g_gtrace) : n * sizeof(unsigned long long);
  return (int)cudaMemcpyFromSymbol(host, g_gtrace, bytes);
}
#endif

}  // namespace mlra
