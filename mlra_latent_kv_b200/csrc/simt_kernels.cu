// CUDA-core kernels of the decode path: query absorption, split-KV latent
// attention, split combine and output up-projection.  They run every shape
// the ABI accepts (fp32 and bf16) and are the path for shapes the tcgen05
// kernels do not implement.  Arithmetic is fp32 throughout.
#include <cuda_fp8.h>

#include "common.cuh"
#include "fp8_cache.h"
#include "launch.h"

namespace mlra {

// ---------------------------------------------------------------------------
// a2: query absorption and query RoPE
//   q_ws[b, h, 0:d_c]        = q_nope[b, h] . W_UK[h]
//   q_ws[b, h, d_c:d_c+d_r]  = RoPE(q_rope[b, h], q_pos[b])
// Rows h in [H, Hq) are written as zeros (padding rows of the tcgen05 path).
// grid (Hq, ceil(d_c/128) + 1), block 128; the last y-slice does the RoPE.
// ---------------------------------------------------------------------------
constexpr int kAbsorbB = 16;

template <typename T, typename QO>
__global__ void __launch_bounds__(128) absorb_kernel(const T* __restrict__ q_nope, const T* __restrict__ q_rope,
                                                     const int* __restrict__ q_pos, const T* __restrict__ W_UK,
                                                     QO* __restrict__ q_ws, AbsorbArgs a, RopeTable tab) {
  extern __shared__ float qs[];  // [kAbsorbB][d_h]
  const int h = blockIdx.x;
  const int ycols = (a.d_c + 127) / 128;
  const int row = a.d_c + a.d_r;
  if ((int)blockIdx.y == ycols) {  // RoPE slice
    const int pairs = a.d_r / 2;
    for (int idx = threadIdx.x; idx < a.B * pairs; idx += blockDim.x) {
      const int b = idx / pairs, i = idx % pairs;
      QO* dst = q_ws + ((size_t)b * a.Hq + h) * row + a.d_c + 2 * i;
      if (h >= a.H) {
        dst[0] = from_f<QO>(0.f);
        dst[1] = from_f<QO>(0.f);
        continue;
      }
      const T* src = q_rope + ((size_t)b * a.H + h) * a.d_r + 2 * i;
      float x0 = to_f(src[0]), x1 = to_f(src[1]);
      float s, c;
      rope_sincos(tab, i, __ldg(q_pos + b), &s, &c);
      dst[0] = from_f<QO>((x0 * c - x1 * s) * a.q_scale);
      dst[1] = from_f<QO>((x0 * s + x1 * c) * a.q_scale);
    }
    return;
  }
  const int col = blockIdx.y * 128 + threadIdx.x;
  for (int b0 = 0; b0 < a.B; b0 += kAbsorbB) {
    const int nb = min(kAbsorbB, a.B - b0);
    if (h < a.H) {
      for (int e = threadIdx.x; e < nb * a.d_h; e += blockDim.x) {
        const int bi = e / a.d_h, d = e % a.d_h;
        qs[bi * a.d_h + d] = to_f(q_nope[((size_t)(b0 + bi) * a.H + h) * a.d_h + d]);
      }
    }
    __syncthreads();
    if (col < a.d_c) {
      float acc[kAbsorbB];
#pragma unroll
      for (int i = 0; i < kAbsorbB; ++i) acc[i] = 0.f;
      if (h < a.H) {
        const T* w = W_UK + (size_t)h * a.d_h * a.d_c + col;
        for (int d = 0; d < a.d_h; ++d) {
          const float wv = to_f(w[(size_t)d * a.d_c]);
#pragma unroll
          for (int i = 0; i < kAbsorbB; ++i) acc[i] = fmaf(qs[i * a.d_h + d], wv, acc[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < kAbsorbB; ++i)
        if (i < nb) q_ws[((size_t)(b0 + i) * a.Hq + h) * row + col] = from_f<QO>(acc[i] * a.q_scale);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// a3 (CUDA cores): split-KV latent attention, per worker piece and head.
// grid (G, ceil(H/8)), block 256: warp w handles head blockIdx.y*8 + w; the
// block stages kTileTok cache rows (latent | rope) in shared memory as fp32.
// Lane l owns latent dims l + 32k and rope dims l + 32k.
// Writes the unnormalised partial o (relative to the running max m, in log2
// units) and m, l per branch to slot c + b.  Partial layout (shared with the
// tcgen05 kernels): o_part[slot][H][d_c] fp32 (head-major, so the combine of a
// head reads each piece's row contiguously), ml_part[slot][n_branch][2][H] (m, l).
// ---------------------------------------------------------------------------
constexpr int kTileTok = 16;

// Cache element -> fp32.  An FP8 cache (E4M3 codes, one fp32 scale per page
// and tensor) stores uint8_t; its value is decode(code) * scale[page].
__device__ __forceinline__ float cache_f(float x, const float*, int) { return x; }
__device__ __forceinline__ float cache_f(__nv_bfloat16 x, const float*, int) { return __bfloat162float(x); }
__device__ __forceinline__ float cache_f(uint8_t x, const float* scale, int pg) {
  __nv_fp8_e4m3 v;
  v.__x = x;
  return static_cast<float>(v) * __ldg(scale + pg);
}
constexpr int kMaxDpl = 16;  // d_c <= 512
constexpr int kMaxRpl = 2;   // d_r <= 64
constexpr int kMaxBr = 8;

template <typename T>
__global__ void __launch_bounds__(256) attend_simt_kernel(const float* __restrict__ q_ws, const T* __restrict__ lat,
                                                          const T* __restrict__ rop, const int* __restrict__ page_table,
                                                          const int* __restrict__ seq_lens, float* __restrict__ o_part,
                                                          float* __restrict__ ml_part, int* __restrict__ err,
                                                          AttnArgs a, const float* __restrict__ lat_scale = nullptr,
                                                          const float* __restrict__ rop_scale = nullptr) {
  extern __shared__ float tile[];  // [kTileTok][d_c + d_r]
  __shared__ WorkerPlan s_plan;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int h = blockIdx.y * 8 + warp;
  const int W = a.d_c + a.d_r;
  const int dpl = a.d_c / 32;
  const int d_cb = a.d_c / a.n_branch;
  const int maxL = a.maxp * kPage;
  if (c == 0 && blockIdx.y == 0) check_lengths(seq_lens, a.B, maxL, err);
  if (warp == 0) {
    WorkerPlan p = plan_worker(seq_lens, a.B, a.G, c, maxL);
    if (lane == 0) s_plan = p;
  }
  __syncthreads();
  SegWalk walk(s_plan, a.B, maxL);
  while (walk.next(seq_lens)) {
    const int b = walk.b;
    const int t0 = walk.pg0 * kPage;
    const int t1 = min(walk.pg1 * kPage, walk.L);
    float qv[kMaxDpl], qr[kMaxRpl], o[kMaxDpl], m[kMaxBr], l[kMaxBr];
#pragma unroll
    for (int k = 0; k < kMaxDpl; ++k) {
      qv[k] = 0.f;
      o[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < kMaxRpl; ++k) qr[k] = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxBr; ++k) {
      m[k] = -INFINITY;
      l[k] = 0.f;
    }
    if (h < a.H) {
      const float* q = q_ws + ((size_t)b * a.H + h) * W;
#pragma unroll
      for (int k = 0; k < kMaxDpl; ++k)
        if (k < dpl) qv[k] = q[lane + 32 * k];
#pragma unroll
      for (int k = 0; k < kMaxRpl; ++k)
        if (lane + 32 * k < a.d_r) qr[k] = q[a.d_c + lane + 32 * k];
    }
    for (int tt = t0; tt < t1; tt += kTileTok) {
      const int n = min(kTileTok, t1 - tt);
      for (int e = threadIdx.x; e < n * W; e += blockDim.x) {
        const int j = e / W, col = e % W;
        const int t = tt + j;
        const int pg = page_of(page_table, a.maxp, a.num_pages, b, t, err);
        const size_t slot = (size_t)pg * kPage + (t % kPage);
        tile[j * W + col] = col < a.d_c ? cache_f(lat[slot * a.d_c + col], lat_scale, pg)
                                        : cache_f(rop[slot * a.d_r + (col - a.d_c)], rop_scale, pg);
      }
      __syncthreads();
      if (h < a.H) {
        for (int j = 0; j < n; ++j) {
          const float* row = tile + j * W;
          float r = 0.f;
#pragma unroll
          for (int k = 0; k < kMaxRpl; ++k)
            if (lane + 32 * k < a.d_r) r = fmaf(qr[k], row[a.d_c + lane + 32 * k], r);
          r = warp_sum(r);
#pragma unroll
          for (int br = 0; br < kMaxBr; ++br) {
            if (br < a.n_branch) {
              float sb = 0.f;
#pragma unroll
              for (int k = 0; k < kMaxDpl; ++k)
                if (k < dpl && (32 * k) / d_cb == br) sb = fmaf(qv[k], row[lane + 32 * k], sb);
              const float s2 = (warp_sum(sb) + r) * a.scale_log2;
              const float mn = fmaxf(m[br], s2);
              const float corr = exp2f(m[br] - mn);
              const float p = exp2f(s2 - mn);
              l[br] = fmaf(l[br], corr, p);
              m[br] = mn;
#pragma unroll
              for (int k = 0; k < kMaxDpl; ++k)
                if (k < dpl && (32 * k) / d_cb == br) o[k] = fmaf(o[k], corr, p * row[lane + 32 * k]);
            }
          }
        }
      }
      __syncthreads();
    }
    if (h < a.H) {
      const int slot = c + b;
#pragma unroll
      for (int k = 0; k < kMaxDpl; ++k) {
        if (k < dpl) {
          const int d = lane + 32 * k;
          o_part[((size_t)slot * a.H + h) * a.d_c + d] = o[k];
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int br = 0; br < kMaxBr; ++br) {
          if (br < a.n_branch) {
            ml_part[(((size_t)slot * a.n_branch + br) * 2 + 0) * a.H + h] = m[br];
            ml_part[(((size_t)slot * a.n_branch + br) * 2 + 1) * a.H + h] = l[br];
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// a4: split combine.  For sequence b, the pieces are workers
// [worker_of_page(P_b), worker_of_page(P_b + np_b - 1)], at slots c + b.
//   M = max_s m_s;  w_s = 2^(m_s - M);  L = sum_s w_s l_s
//   o_lat[b, h, br cols] = branch_scale * sum_s w_s o_s / L
// grid (B, ceil(H/4)), block 128: one warp per head, lanes over 4-dim groups.
// ---------------------------------------------------------------------------
template <typename OT>
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ o_part, const float* __restrict__ ml_part,
                                                      const int* __restrict__ seq_lens, OT* __restrict__ o_lat,
                                                      CombineArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int h = blockIdx.y * 4 + warp;
  // total pages and this sequence's first page
  const int maxL = a.maxp * kPage;
  long long T = 0, P = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int bb = base + lane;
    const int np = bb < a.B ? npages_of(seq_len_at(seq_lens, bb, maxL)) : 0;
    T += warp_sum_i(np);
    P += warp_sum_i(bb < b ? np : 0);
  }
  if (h >= a.H) return;
  const int L = seq_len_at(seq_lens, b, maxL);
  const int np = npages_of(L);
  const int d_cb = a.d_c / a.n_branch;
  OT* dst = o_lat + ((size_t)b * a.H + h) * a.d_c;
  if (np == 0) {
    for (int d = lane; d < a.d_c; d += 32) dst[d] = from_f<OT>(0.f);
    return;
  }
  // workers c0..c1 hold this sequence's pages; with more workers than pages
  // some in between own no page at all and wrote nothing: skip them
  const int c0 = worker_of_page(P, T, a.G);
  const int c1 = worker_of_page(P + np - 1, T, a.G);
#define MLRA_WORKER_EMPTY(c) (worker_start((c), T, a.G) == worker_start((c) + 1, T, a.G))
  for (int br = 0; br < a.n_branch; ++br) {
    float M = -INFINITY;
    for (int c = c0; c <= c1; ++c)
      if (!MLRA_WORKER_EMPTY(c)) M = fmaxf(M, ml_part[(((size_t)(c + b) * a.n_branch + br) * 2 + 0) * a.H + h]);
    float Lsum = 0.f;
    for (int c = c0; c <= c1; ++c) {
      if (MLRA_WORKER_EMPTY(c)) continue;
      const size_t base = ((size_t)(c + b) * a.n_branch + br) * 2;
      Lsum += exp2f(ml_part[(base + 0) * a.H + h] - M) * ml_part[(base + 1) * a.H + h];
    }
    const float inv = a.branch_scale / Lsum;
    for (int d = br * d_cb + lane; d < (br + 1) * d_cb; d += 32) {
      float acc = 0.f;
      for (int c = c0; c <= c1; ++c) {
        if (MLRA_WORKER_EMPTY(c)) continue;
        const size_t base = ((size_t)(c + b) * a.n_branch + br) * 2;
        const float w = exp2f(ml_part[(base + 0) * a.H + h] - M);
        acc = fmaf(w, o_part[((size_t)(c + b) * a.H + h) * a.d_c + d], acc);
      }
      dst[d] = from_f<OT>(acc * inv);
    }
  }
#undef MLRA_WORKER_EMPTY
}

// ---------------------------------------------------------------------------
// a5: output up-projection  out[b, h] = o_lat[b, h] . W_UV[h]
// grid (H, ceil(d_v/128)), block 128: thread per output column, batch rows
// staged 16 at a time.
// ---------------------------------------------------------------------------
template <typename IT, typename T>
__global__ void __launch_bounds__(128) upproj_kernel(const IT* __restrict__ o_lat, const T* __restrict__ W_UV,
                                                     T* __restrict__ out, UpArgs a) {
  extern __shared__ float os[];  // [kAbsorbB][d_c]
  const int h = blockIdx.x;
  const int v = blockIdx.y * 128 + threadIdx.x;
  for (int b0 = 0; b0 < a.B; b0 += kAbsorbB) {
    const int nb = min(kAbsorbB, a.B - b0);
    for (int e = threadIdx.x; e < nb * a.d_c; e += blockDim.x) {
      const int bi = e / a.d_c, d = e % a.d_c;
      os[bi * a.d_c + d] = to_f(o_lat[((size_t)(b0 + bi) * a.H + h) * a.d_c + d]);
    }
    __syncthreads();
    if (v < a.d_v) {
      float acc[kAbsorbB];
#pragma unroll
      for (int i = 0; i < kAbsorbB; ++i) acc[i] = 0.f;
      const T* w = W_UV + (size_t)h * a.d_c * a.d_v + v;
      for (int d = 0; d < a.d_c; ++d) {
        const float wv = to_f(w[(size_t)d * a.d_v]);
#pragma unroll
        for (int i = 0; i < kAbsorbB; ++i) acc[i] = fmaf(os[i * a.d_c + d], wv, acc[i]);
      }
#pragma unroll
      for (int i = 0; i < kAbsorbB; ++i)
        if (i < nb) out[((size_t)(b0 + i) * a.H + h) * a.d_v + v] = from_f<T>(acc[i]);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <typename T, typename QO>
cudaError_t launch_absorb_t(const void* q_nope, const void* q_rope, const int* q_pos, const void* W_UK, void* q_ws,
                            const AbsorbArgs& a, const RopeTable& tab, cudaStream_t st) {
  dim3 grid(a.Hq, (a.d_c + 127) / 128 + 1);
  size_t smem = (size_t)kAbsorbB * a.d_h * sizeof(float);
  absorb_kernel<T, QO><<<grid, 128, smem, st>>>((const T*)q_nope, (const T*)q_rope, q_pos, (const T*)W_UK,
                                               (QO*)q_ws, a, tab);
  return cudaGetLastError();
}

cudaError_t launch_absorb(int dtype, bool q_bf16, const void* q_nope, const void* q_rope, const int* q_pos,
                          const void* W_UK, void* q_ws, const AbsorbArgs& a, const RopeTable& tab,
                          cudaStream_t st) {
  if (dtype == 1) {
    return q_bf16 ? launch_absorb_t<__nv_bfloat16, __nv_bfloat16>(q_nope, q_rope, q_pos, W_UK, q_ws, a, tab, st)
                  : launch_absorb_t<__nv_bfloat16, float>(q_nope, q_rope, q_pos, W_UK, q_ws, a, tab, st);
  }
  return launch_absorb_t<float, float>(q_nope, q_rope, q_pos, W_UK, q_ws, a, tab, st);
}

cudaError_t launch_attend_simt(int dtype, const float* q_ws, const void* lat, const void* rop, const int* page_table,
                               const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                               cudaStream_t st) {
  dim3 grid(a.G, (a.H + 7) / 8);
  size_t smem = (size_t)kTileTok * (a.d_c + a.d_r) * sizeof(float);
  if (dtype == 1) {
    attend_simt_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(q_ws, (const __nv_bfloat16*)lat,
                                                              (const __nv_bfloat16*)rop, page_table, seq_lens, o_part,
                                                              ml_part, err, a);
  } else {
    attend_simt_kernel<float><<<grid, 256, smem, st>>>(q_ws, (const float*)lat, (const float*)rop, page_table,
                                                      seq_lens, o_part, ml_part, err, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_attend_simt_fp8(const float* q_ws, const uint8_t* lat, const uint8_t* rop, const float* lat_scale,
                                   const float* rop_scale, const int* page_table, const int* seq_lens, float* o_part,
                                   float* ml_part, int* err, const AttnArgs& a, cudaStream_t st) {
  dim3 grid(a.G, (a.H + 7) / 8);
  size_t smem = (size_t)kTileTok * (a.d_c + a.d_r) * sizeof(float);
  attend_simt_kernel<uint8_t><<<grid, 256, smem, st>>>(q_ws, lat, rop, page_table, seq_lens, o_part, ml_part, err, a,
                                                       lat_scale, rop_scale);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// FP8 cache quantizer: one CTA per page of one tensor (latent or rope).
//   scale = (largest finite |x| on the page) / 448, fp32 (1 for a page with no
//   nonzero finite value); code = E4M3 of fl32(x / scale), nearest with ties
//   to even, saturating at 448; NaN stays NaN.
// grid (num_pages), block 256.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) quantize_pages_kernel(const T* __restrict__ pool, int n_per_page,
                                                             uint8_t* __restrict__ codes, float* __restrict__ scales) {
  __shared__ float red[8];
  __shared__ float s_scale;
  const T* src = pool + (size_t)blockIdx.x * n_per_page;
  uint8_t* dst = codes + (size_t)blockIdx.x * n_per_page;
  float amax = 0.f;
  for (int i = threadIdx.x; i < n_per_page; i += blockDim.x) {
    const float v = to_f(src[i]);
    if (isfinite(v)) amax = fmaxf(amax, fabsf(v));
  }
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
    s_scale = m == 0.f ? 1.f : __fdiv_rn(m, 448.f);
    scales[blockIdx.x] = s_scale;
  }
  __syncthreads();
  const float scale = s_scale;
  for (int i = threadIdx.x; i < n_per_page; i += blockDim.x)
    dst[i] = (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(to_f(src[i]), scale), __NV_SATFINITE, __NV_E4M3);
}

cudaError_t launch_quantize_pages(int dtype, const void* pool, int num_pages, int n_per_page, uint8_t* codes,
                                  float* scales, cudaStream_t st) {
  if (dtype == 1)
    quantize_pages_kernel<__nv_bfloat16><<<num_pages, 256, 0, st>>>((const __nv_bfloat16*)pool, n_per_page, codes,
                                                                    scales);
  else
    quantize_pages_kernel<float><<<num_pages, 256, 0, st>>>((const float*)pool, n_per_page, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_combine(bool out_bf16, const float* o_part, const float* ml_part, const int* seq_lens,
                           void* o_lat, const CombineArgs& a, cudaStream_t st) {
  dim3 grid(a.B, (a.H + 3) / 4);
  if (out_bf16)
    combine_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(o_part, ml_part, seq_lens, (__nv_bfloat16*)o_lat, a);
  else
    combine_kernel<float><<<grid, 128, 0, st>>>(o_part, ml_part, seq_lens, (float*)o_lat, a);
  return cudaGetLastError();
}

cudaError_t launch_upproj(int dtype, bool in_bf16, const void* o_lat, const void* W_UV, void* out, const UpArgs& a,
                          cudaStream_t st) {
  dim3 grid(a.H, (a.d_v + 127) / 128);
  size_t smem = (size_t)kAbsorbB * a.d_c * sizeof(float);
  if (dtype == 1) {
    if (in_bf16)
      upproj_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, 128, smem, st>>>(
          (const __nv_bfloat16*)o_lat, (const __nv_bfloat16*)W_UV, (__nv_bfloat16*)out, a);
    else
      upproj_kernel<float, __nv_bfloat16><<<grid, 128, smem, st>>>((const float*)o_lat, (const __nv_bfloat16*)W_UV,
                                                                  (__nv_bfloat16*)out, a);
  } else {
    upproj_kernel<float, float><<<grid, 128, smem, st>>>((const float*)o_lat, (const float*)W_UV, (float*)out, a);
  }
  return cudaGetLastError();
}

}  // namespace mlra
