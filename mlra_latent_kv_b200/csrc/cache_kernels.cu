// Cache-writing kernels: latent_append (compress a new token and store it)
// and latent_store (store given latent rows, rotating their RoPE keys).
//
// yololab.net, "超越 GQA 的推理革命…", section "1. 鍵值聯合低秩壓縮": the
// token's K/V information is compressed into c_KV = h W_DKV, the only thing the
// cache keeps of it; section "2. 解耦旋轉位置編碼": the positional key
// k_rope = RoPE(h W_KR) is kept beside it without compression.
#include <type_traits>

#include "common.cuh"
#include "host_cache.h"
#include "append_forms.h"
#include "launch.h"
#include "ptx.cuh"

namespace mlra {

// ---------------------------------------------------------------------------
// latent_append, two-kernel form (the shapes the one-launch form below does
// not take: columns that do not split into 16-byte groups, or a hidden width
// whose chunk outgrows its shared memory), pass 1: split-K partial products
//   part[ks, b, j] = sum_{k in chunk ks} h[b, k] * Wcat[k, j],   Wcat = [W_DKV | W_KR]
// grid (KS) chunks of 64 weight rows.  A thread owns kCG adjacent columns (one
// 16-byte load per weight row) in one of kRG row groups (rows rg, rg + kRG,
// ...), issues its row loads 16 at a time (8 for fp32) before using any, so a
// bf16 chunk costs one memory round trip, and the row groups are summed
// in a fixed order through shared memory.  Batch rows are taken kAppendB at a
// time from shared memory.  Weight rows are read exactly once.  The finalize
// kernel may launch as soon as this grid starts (programmatic dependent
// launch); it waits for this grid's sums before reading them.
// ---------------------------------------------------------------------------
constexpr int kAppendRows = 64;
constexpr int kAppendB = 4;
constexpr int kMaxAppendCols = 512 + 64;  // d_c + d_r at most
// row groups: 4 with 16-byte column groups, 2 with narrower ones (<= 576 threads)
template <int kCG>
constexpr int row_groups() { return kCG >= 4 ? 4 : 2; }
template <int kCG>
constexpr int append_threads() { return kMaxAppendCols / kCG * row_groups<kCG>(); }

template <typename T, int kCG>
__global__ void __launch_bounds__(append_threads<kCG>()) append_partial_kernel(const T* __restrict__ h, const T* __restrict__ W_DKV,
                                      const T* __restrict__ W_KR, float* __restrict__ part, AppendArgs a) {
  constexpr int kRG = row_groups<kCG>();
  constexpr int kRowsPerRG = kAppendRows / kRG;
  extern __shared__ float smem_f[];
  float* hs = smem_f;                          // [kAppendB][kAppendRows]
  float* red = smem_f + kAppendB * kAppendRows;  // [kRG - 1][n_cg][kCG][kAppendB]
  const int ks = blockIdx.x;
  const int k0 = ks * kAppendRows;
  const int nk = min(kAppendRows, a.D - k0);
  const int W = a.d_c + a.d_r;
  const int n_cg = W / kCG;
  const int cg = threadIdx.x % n_cg, rg = threadIdx.x / n_cg;
  const int j = cg * kCG;
  ptx::grid_dep_launch();
  const T* wp;
  int ld;
  if (j < a.d_c) {
    wp = W_DKV + j;
    ld = a.d_c;
  } else {
    wp = W_KR + (j - a.d_c);
    ld = a.d_r;
  }
  using Vec = typename std::conditional<kCG * sizeof(T) == 16, uint4, typename std::conditional<kCG * sizeof(T) == 8, uint2, uint32_t>::type>::type;
  for (int b0 = 0; b0 < a.B; b0 += kAppendB) {
    for (int e = threadIdx.x; e < kAppendB * kAppendRows; e += blockDim.x) {
      const int bi = e / kAppendRows, k = e % kAppendRows;
      hs[e] = (k < nk && b0 + bi < a.B) ? to_f(h[(size_t)(b0 + bi) * a.D + k0 + k]) : 0.f;
    }
    __syncthreads();
    float acc[kCG][kAppendB];
#pragma unroll
    for (int c = 0; c < kCG; ++c)
#pragma unroll
      for (int i = 0; i < kAppendB; ++i) acc[c][i] = 0.f;
    constexpr int kMaxBatch = sizeof(T) == 2 ? 16 : 8;  // 16-byte loads: up to 16 rows in flight at once
    constexpr int kBatch = kRowsPerRG < kMaxBatch ? kRowsPerRG : kMaxBatch;
#pragma unroll 1
    for (int r0 = 0; r0 < kRowsPerRG; r0 += kBatch) {
      Vec wv[kBatch];
#pragma unroll
      for (int r = 0; r < kBatch; ++r) {
        const int k = rg + kRG * (r0 + r);
        if (k < nk) wv[r] = *reinterpret_cast<const Vec*>(wp + (size_t)(k0 + k) * ld);
      }
#pragma unroll
      for (int r = 0; r < kBatch; ++r) {
        const int k = rg + kRG * (r0 + r);
        if (k < nk) {
          const T* w = reinterpret_cast<const T*>(&wv[r]);
#pragma unroll
          for (int c = 0; c < kCG; ++c) {
            const float wc = to_f(w[c]);
#pragma unroll
            for (int i = 0; i < kAppendB; ++i) acc[c][i] = fmaf(hs[i * kAppendRows + k], wc, acc[c][i]);
          }
        }
      }
    }
    // row groups 1.. hand their sums to row group 0, which adds them in order
    if (rg > 0) {
      float* dst = red + ((size_t)(rg - 1) * n_cg + cg) * kCG * kAppendB;
#pragma unroll
      for (int c = 0; c < kCG; ++c)
#pragma unroll
        for (int i = 0; i < kAppendB; ++i) dst[c * kAppendB + i] = acc[c][i];
    }
    __syncthreads();
    if (rg == 0) {
      for (int g = 1; g < kRG; ++g) {
        const float* src = red + ((size_t)(g - 1) * n_cg + cg) * kCG * kAppendB;
#pragma unroll
        for (int c = 0; c < kCG; ++c)
#pragma unroll
          for (int i = 0; i < kAppendB; ++i) acc[c][i] += src[c * kAppendB + i];
      }
#pragma unroll
      for (int i = 0; i < kAppendB; ++i) {
        if (b0 + i < a.B) {
          float* dst = part + ((size_t)ks * a.B + b0 + i) * W + j;
#pragma unroll
          for (int c = 0; c < kCG; ++c) dst[c] = acc[c][i];
        }
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// latent_append, pass 2: sum the chunks, rotate the RoPE part at pos[b],
// round once and store into the page slot of position pos[b].
// One warp per (b, column pair): lane l adds chunks l, l + 32, ... in order,
// then a fixed butterfly adds the lanes (lane 0's result is used), so the sum
// has the same order on every call.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void append_finalize_kernel(const float* __restrict__ part, const int* __restrict__ pos,
                                       const int* __restrict__ page_table, T* __restrict__ lat, T* __restrict__ rop,
                                       int* __restrict__ err, AppendArgs a, RopeTable tab) {
  const int W = a.d_c + a.d_r;
  const int pairs = W / 2;
  const int lane = threadIdx.x & 31;
  const int idx = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  ptx::grid_dep_wait();  // the partial sums come from the previous kernel
  if (idx >= a.B * pairs) return;
  const int b = idx / pairs, j = 2 * (idx % pairs);
  float x0 = 0.f, x1 = 0.f;
  float2 v[4];
  for (int base = 0; base < a.KS; base += 128) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int ks = base + lane + 32 * u;
      v[u] = ks < a.KS ? *reinterpret_cast<const float2*>(part + ((size_t)ks * a.B + b) * W + j)
                       : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      x0 += v[u].x;
      x1 += v[u].y;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    x0 += __shfl_xor_sync(0xffffffffu, x0, off);
    x1 += __shfl_xor_sync(0xffffffffu, x1, off);
  }
  if (lane != 0) return;
  const int p = __ldg(pos + b);
  if (p < 0 || p >= a.maxp * kPage) {
    report_error(err, kErrDeviceCheck, b, p);
    return;
  }
  const int pg = page_for_write(page_table, a.maxp, a.num_pages, b, p, err);
  if (pg < 0) return;  // reported; nothing is written for this sequence
  const size_t slot = (size_t)pg * kPage + (p % kPage);
  if (j < a.d_c) {
    lat[slot * a.d_c + j] = from_f<T>(x0);
    lat[slot * a.d_c + j + 1] = from_f<T>(x1);
  } else {
    const int i = (j - a.d_c) / 2;
    float s, c;
    rope_sincos(tab, i, p, &s, &c);
    rop[slot * a.d_r + 2 * i] = from_f<T>(x0 * c - x1 * s);
    rop[slot * a.d_r + 2 * i + 1] = from_f<T>(x0 * s + x1 * c);
  }
}

// ---------------------------------------------------------------------------
// latent_append in one launch, for 16-byte column groups (d_r a multiple of
// 16 / sizeof(T)): one cluster of kApSplit CTAs per block of kApCols columns
// of Wcat = [W_DKV | W_KR].  Rank r of the cluster reads rows [r rc, r rc + rc)
// of its columns (rc = ceil(D / kApSplit)) exactly once, every thread with all
// of its row loads in flight at once; the CTA adds its row groups in a fixed
// order through shared memory and stores its kApCols x kAppendB sums into rank
// 0's shared memory; after the cluster barrier rank 0 adds the ranks' sums in
// rank order, rotates the RoPE pairs at pos[b], rounds once and stores the
// slot.  The partial sums never leave the chip, so this form needs no scratch,
// and the sum has the same order on every call.
// ---------------------------------------------------------------------------
constexpr int kApCols = 32;     // columns per cluster (d_c is a multiple of 32: a block is latent or rope)
constexpr int kApSplit = 8;     // CTAs per cluster: row chunks of the hidden dim
constexpr int kApThreads = 256;
constexpr int kApLoads = 10;    // row loads of a thread in flight at once (all of them at d_model = 5120)
constexpr int kApOut = kApCols * kAppendB;  // a CTA's sums: [sequence][column]
constexpr int kApRedStride = kApOut + 1;    // a row group's sums; the odd stride keeps the stores conflict-free
constexpr size_t kApMaxDynSmem = 160 * 1024;  // hs: kAppendB x rc floats

__device__ __forceinline__ void st_cluster_f32(uint32_t caddr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(caddr), "f"(v) : "memory");
}

template <typename T>
__global__ void __cluster_dims__(1, kApSplit, 1) __launch_bounds__(kApThreads, 2)
    append_cluster_kernel(const T* __restrict__ h, const T* __restrict__ W_DKV, const T* __restrict__ W_KR,
                          const int* __restrict__ pos, const int* __restrict__ page_table, T* __restrict__ lat,
                          T* __restrict__ rop, int* __restrict__ err, AppendArgs a, RopeTable tab) {
  constexpr int kCG = 16 / (int)sizeof(T);   // columns of one 16-byte load
  constexpr int kNCG = kApCols / kCG;        // column groups
  constexpr int kRG = kApThreads / kNCG;     // row groups
  __shared__ float red[kRG][kApRedStride];
  __shared__ float gath[kApSplit][kApOut];   // used in rank 0: every rank's sums
  extern __shared__ float hs[];              // [kAppendB][rc]
  const int W = a.d_c + a.d_r;
  const int rc = (a.D + kApSplit - 1) / kApSplit;
  const int rank = (int)ptx::cluster_ctarank();
  const int k0 = rank * rc;
  const int nk = max(0, min(rc, a.D - k0));
  const int cg = threadIdx.x % kNCG, rg = threadIdx.x / kNCG;
  const int j = blockIdx.x * kApCols + cg * kCG;
  const bool col_ok = j < W;
  const T* wp = !col_ok ? W_KR : j < a.d_c ? W_DKV + j : W_KR + (j - a.d_c);  // never read when !col_ok
  const int ld = j < a.d_c ? a.d_c : a.d_r;
  const uint32_t to_rank0 = ptx::map_to_cta(ptx::smem_u32(&gath[rank][0]), 0);
  // every CTA of the cluster must have started before rank 0's shared memory is written: arrive now, wait
  // just before the first remote store
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  bool first = true;
  for (int b0 = 0; b0 < a.B; b0 += kAppendB) {
    // rank 0's storing threads: thread t < kApOut / 2 stores columns (jj, jj + 1) of sequence
    // b0 + t / (kApCols / 2).  Its position is loaded now and its page id once the h rows are staged, so
    // neither lookup delays the weight loads; both have landed by the time they are used.
    const int pc = 2 * (threadIdx.x % (kApCols / 2)), si = threadIdx.x / (kApCols / 2);
    const int jj = blockIdx.x * kApCols + pc;
    const bool storer = rank == 0 && threadIdx.x < kApOut / 2 && b0 + si < a.B && jj < W;
    const int p = storer ? __ldg(pos + b0 + si) : 0;
    const bool pos_ok = p >= 0 && p < a.maxp * kPage;
    int pg = -1;
    float acc[kCG][kAppendB];
#pragma unroll
    for (int c = 0; c < kCG; ++c)
#pragma unroll
      for (int i = 0; i < kAppendB; ++i) acc[c][i] = 0.f;
#pragma unroll 1
    for (int r0 = rg; r0 < nk || r0 == rg; r0 += kRG * kApLoads) {
      uint4 wv[kApLoads];
#pragma unroll
      for (int u = 0; u < kApLoads; ++u) {
        const int k = r0 + u * kRG;
        if (col_ok && k < nk) wv[u] = __ldg(reinterpret_cast<const uint4*>(wp + (size_t)(k0 + k) * ld));
      }
      if (r0 == rg) {  // the batch's h rows are staged while the first weight rows are in flight
        // kApLoads values per thread in flight at once (all of them at d_model = 5120)
        for (int e0 = threadIdx.x; e0 < kAppendB * rc; e0 += kApThreads * kApLoads) {
          float v[kApLoads];
#pragma unroll
          for (int u = 0; u < kApLoads; ++u) {
            const int e = e0 + u * kApThreads, bi = e / rc, k = e % rc;
            v[u] = (e < kAppendB * rc && k < nk && b0 + bi < a.B) ? to_f(h[(size_t)(b0 + bi) * a.D + k0 + k]) : 0.f;
          }
#pragma unroll
          for (int u = 0; u < kApLoads; ++u)
            if (e0 + u * kApThreads < kAppendB * rc) hs[e0 + u * kApThreads] = v[u];
        }
        if (storer && pos_ok) pg = __ldg(page_table + (size_t)(b0 + si) * a.maxp + p / kPage);
        __syncthreads();
      }
#pragma unroll
      for (int u = 0; u < kApLoads; ++u) {
        const int k = r0 + u * kRG;
        if (col_ok && k < nk) {
          const T* w = reinterpret_cast<const T*>(&wv[u]);
#pragma unroll
          for (int c = 0; c < kCG; ++c) {
            const float wc = to_f(w[c]);
#pragma unroll
            for (int i = 0; i < kAppendB; ++i) acc[c][i] = fmaf(hs[i * rc + k], wc, acc[c][i]);
          }
        }
      }
    }
    float sn = 0.f, cs = 1.f;
    if (storer && pos_ok && jj >= a.d_c) rope_sincos(tab, (jj - a.d_c) / 2, p, &sn, &cs);
#pragma unroll
    for (int c = 0; c < kCG; ++c)
#pragma unroll
      for (int i = 0; i < kAppendB; ++i) red[rg][i * kApCols + cg * kCG + c] = acc[c][i];
    __syncthreads();
    float sum = 0.f;
    if (threadIdx.x < kApOut)  // row groups in order
      for (int g = 0; g < kRG; ++g) sum += red[g][threadIdx.x];
    if (first) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    first = false;
    if (threadIdx.x < kApOut) st_cluster_f32(to_rank0 + 4u * threadIdx.x, sum);  // into rank 0
    ptx::cluster_sync();  // rank 0 now holds every rank's sums
    // a position or page id out of range is reported and nothing is written for that sequence
    bool write = false;
    if (storer && !pos_ok) {
      report_error(err, kErrDeviceCheck, b0 + si, p);
    } else if (storer && (pg < 0 || pg >= a.num_pages)) {
      report_error(err, kErrDeviceCheck, b0 + si, p);
    } else {
      write = storer;
    }
    if (write) {
      const size_t slot = (size_t)pg * kPage + (p % kPage);
      float x0 = 0.f, x1 = 0.f;
      for (int q = 0; q < kApSplit; ++q) {  // ranks in order
        x0 += gath[q][si * kApCols + pc];
        x1 += gath[q][si * kApCols + pc + 1];
      }
      if (jj < a.d_c) {
        lat[slot * a.d_c + jj] = from_f<T>(x0);
        lat[slot * a.d_c + jj + 1] = from_f<T>(x1);
      } else {
        const int ir = (jj - a.d_c) / 2;
        rop[slot * a.d_r + 2 * ir] = from_f<T>(x0 * cs - x1 * sn);
        rop[slot * a.d_r + 2 * ir + 1] = from_f<T>(x0 * sn + x1 * cs);
      }
    }
    if (b0 + kAppendB < a.B) ptx::cluster_sync();  // rank 0 has read its sums before the next batch rewrites them
  }
}

template <typename T>
static size_t append_cluster_dyn_smem(const AppendArgs& a) {
  return sizeof(float) * kAppendB * (size_t)((a.D + kApSplit - 1) / kApSplit);
}

template <typename T>
static cudaError_t launch_append_cluster(const void* h, const void* W_DKV, const void* W_KR, const int* pos,
                                         const int* page_table, void* lat, void* rop, int* err, const AppendArgs& a,
                                         const RopeTable& tab, cudaStream_t st) {
  const size_t dyn = append_cluster_dyn_smem<T>(a);
  auto k = append_cluster_kernel<T>;
  const cudaError_t e = ensure_smem(reinterpret_cast<const void*>(k), (int)dyn);
  if (e != cudaSuccess) return e;
  const int n_cb = (a.d_c + a.d_r + kApCols - 1) / kApCols;
  k<<<dim3(n_cb, kApSplit), kApThreads, dyn, st>>>((const T*)h, (const T*)W_DKV, (const T*)W_KR, pos, page_table,
                                                   (T*)lat, (T*)rop, err, a, tab);
  return cudaGetLastError();
}

template <typename T, int kCG>
static cudaError_t launch_append_t(const void* h, const void* W_DKV, const void* W_KR, const int* pos,
                                   const int* page_table, void* lat, void* rop, float* part, int* err,
                                   const AppendArgs& a, const RopeTable& tab, cudaStream_t st) {
  constexpr int kRG = row_groups<kCG>();
  const int W = a.d_c + a.d_r;
  const int n_cg = W / kCG;
  const int thr = n_cg * kRG;
  const size_t smem = sizeof(float) * ((size_t)kAppendB * kAppendRows + (size_t)(kRG - 1) * n_cg * kCG * kAppendB);
  auto k1 = append_partial_kernel<T, kCG>;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  k1<<<a.KS, thr, smem, st>>>((const T*)h, (const T*)W_DKV, (const T*)W_KR, part, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the finalize kernel as a programmatic dependent of the partial sums
  const int n2 = a.B * (W / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((n2 + 7) / 8, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, append_finalize_kernel<T>, (const float*)part, pos, page_table, (T*)lat, (T*)rop,
                            err, a, tab);
}

bool append_uses_scratch(int dtype, int D, int d_c, int d_r) {
  const int cg = dtype == 1 ? 8 : 4;  // columns of a 16-byte load
  const size_t dyn = sizeof(float) * kAppendB * (size_t)((D + kApSplit - 1) / kApSplit);
  return d_c % cg != 0 || d_r % cg != 0 || dyn > kApMaxDynSmem;
}

cudaError_t launch_append(int dtype, const void* h, const void* W_DKV, const void* W_KR, const int* pos,
                          const int* page_table, void* lat, void* rop, float* part, int* err, const AppendArgs& a,
                          const RopeTable& tab, cudaStream_t st) {
  // one cluster-reduced launch where the columns split into 16-byte groups and the hidden chunk fits shared
  // memory; else the split-K pair of kernels, whose partial sums go through `part`
  if (!append_uses_scratch(dtype, a.D, a.d_c, a.d_r)) {
    if (dtype == 1)
      return launch_append_cluster<__nv_bfloat16>(h, W_DKV, W_KR, pos, page_table, lat, rop, err, a, tab, st);
    return launch_append_cluster<float>(h, W_DKV, W_KR, pos, page_table, lat, rop, err, a, tab, st);
  }
  if (dtype == 1) {
    if (a.d_c % 8 == 0 && a.d_r % 8 == 0)
      return launch_append_t<__nv_bfloat16, 8>(h, W_DKV, W_KR, pos, page_table, lat, rop, part, err, a, tab, st);
    return launch_append_t<__nv_bfloat16, 2>(h, W_DKV, W_KR, pos, page_table, lat, rop, part, err, a, tab, st);
  }
  if (a.d_c % 4 == 0 && a.d_r % 4 == 0)
    return launch_append_t<float, 4>(h, W_DKV, W_KR, pos, page_table, lat, rop, part, err, a, tab, st);
  return launch_append_t<float, 2>(h, W_DKV, W_KR, pos, page_table, lat, rop, part, err, a, tab, st);
}

// ---------------------------------------------------------------------------
// latent_store: token row i -> slot of (tok_seq[i], tok_pos[i]).
// Work item = (token, 16-byte chunk of the latent row) or (token, RoPE pair).
// The latent is copied bit for bit; the RoPE key is rotated and rounded.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void store_kernel(const T* __restrict__ c_kv, const T* __restrict__ k_rope, const int* __restrict__ tok_seq,
                             const int* __restrict__ tok_pos, const int* __restrict__ page_table, T* __restrict__ lat,
                             T* __restrict__ rop, int* __restrict__ err, StoreArgs a, RopeTable tab) {
  constexpr int kPer16 = 16 / sizeof(T);
  const int lchunks = a.d_c / kPer16;
  const int pairs = a.d_r / 2;
  const int per_tok = lchunks + pairs;
  const long long total = (long long)a.n_tokens * per_tok;
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total;
       w += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(w / per_tok);
    const int k = (int)(w % per_tok);
    const int b = __ldg(tok_seq + i);
    const int p = __ldg(tok_pos + i);
    if (b < 0 || b >= a.B || p < 0 || p >= a.maxp * kPage) {
      report_error(err, kErrDeviceCheck, i, p);
      continue;
    }
    const int pg = page_for_write(page_table, a.maxp, a.num_pages, b, p, err);
    if (pg < 0) continue;  // reported; this token is not written
    const size_t slot = (size_t)pg * kPage + (p % kPage);
    if (k < lchunks) {
      const uint4 v = *reinterpret_cast<const uint4*>(c_kv + (size_t)i * a.d_c + (size_t)k * kPer16);
      *reinterpret_cast<uint4*>(lat + slot * a.d_c + (size_t)k * kPer16) = v;
    } else {
      const int q = k - lchunks;
      const float x0 = to_f(k_rope[(size_t)i * a.d_r + 2 * q]);
      const float x1 = to_f(k_rope[(size_t)i * a.d_r + 2 * q + 1]);
      float s, c;
      rope_sincos(tab, q, p, &s, &c);
      rop[slot * a.d_r + 2 * q] = from_f<T>(x0 * c - x1 * s);
      rop[slot * a.d_r + 2 * q + 1] = from_f<T>(x0 * s + x1 * c);
    }
  }
}

cudaError_t launch_store(int dtype, const void* c_kv, const void* k_rope, const int* tok_seq, const int* tok_pos,
                         const int* page_table, void* lat, void* rop, int* err, const StoreArgs& a,
                         const RopeTable& tab, cudaStream_t st) {
  if (a.n_tokens == 0) return cudaSuccess;
  const int blocks = 148 * 8;
  if (dtype == 1)
    store_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>((const __nv_bfloat16*)c_kv, (const __nv_bfloat16*)k_rope,
                                                         tok_seq, tok_pos, page_table, (__nv_bfloat16*)lat,
                                                         (__nv_bfloat16*)rop, err, a, tab);
  else
    store_kernel<float><<<blocks, 256, 0, st>>>((const float*)c_kv, (const float*)k_rope, tok_seq, tok_pos,
                                                 page_table, (float*)lat, (float*)rop, err, a, tab);
  return cudaGetLastError();
}

}  // namespace mlra
