// Cache-writing kernels: latent_append (compress a new token and store it)
// and latent_store (store given latent rows, rotating their RoPE keys).
//
// yololab.net, "超越 GQA 的推理革命…", section "1. 鍵值聯合低秩壓縮": the
// token's K/V information is compressed into c_KV = h W_DKV, the only thing the
// cache keeps of it; section "2. 解耦旋轉位置編碼": the positional key
// k_rope = RoPE(h W_KR) is kept beside it without compression.
#include "common.cuh"
#include "launch.h"

namespace mlra {

// ---------------------------------------------------------------------------
// latent_append, pass 1: split-K partial products
//   part[ks, b, j] = sum_{k in chunk ks} h[b, k] * Wcat[k, j],   Wcat = [W_DKV | W_KR]
// grid (KS), block = one thread per column pair (2j, 2j+1); 64 rows per chunk.
// Weight rows are read once (the weights dominate the bytes); batch rows are
// processed 8 at a time from shared memory.
// ---------------------------------------------------------------------------
constexpr int kAppendRows = 64;
constexpr int kAppendB = 8;

template <typename T>
__global__ void append_partial_kernel(const T* __restrict__ h, const T* __restrict__ W_DKV,
                                      const T* __restrict__ W_KR, float* __restrict__ part, AppendArgs a) {
  __shared__ float hs[kAppendB * kAppendRows];
  const int ks = blockIdx.x;
  const int k0 = ks * kAppendRows;
  const int nk = min(kAppendRows, a.D - k0);
  const int W = a.d_c + a.d_r;
  const int j = 2 * threadIdx.x;
  const T* wp = nullptr;
  int ld = 0;
  if (j < a.d_c) {
    wp = W_DKV + j;
    ld = a.d_c;
  } else if (j < W) {
    wp = W_KR + (j - a.d_c);
    ld = a.d_r;
  }
  for (int b0 = 0; b0 < a.B; b0 += kAppendB) {
    for (int e = threadIdx.x; e < kAppendB * kAppendRows; e += blockDim.x) {
      const int bi = e / kAppendRows, k = e % kAppendRows;
      hs[e] = (k < nk && b0 + bi < a.B) ? to_f(h[(size_t)(b0 + bi) * a.D + k0 + k]) : 0.f;
    }
    __syncthreads();
    if (j < W) {
      float acc0[kAppendB], acc1[kAppendB];
#pragma unroll
      for (int i = 0; i < kAppendB; ++i) acc0[i] = acc1[i] = 0.f;
      const T* wk = wp + (size_t)k0 * ld;
      for (int k = 0; k < nk; ++k) {
        const float w0 = to_f(wk[(size_t)k * ld]);
        const float w1 = to_f(wk[(size_t)k * ld + 1]);
#pragma unroll
        for (int i = 0; i < kAppendB; ++i) {
          const float hv = hs[i * kAppendRows + k];
          acc0[i] = fmaf(hv, w0, acc0[i]);
          acc1[i] = fmaf(hv, w1, acc1[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < kAppendB; ++i) {
        if (b0 + i < a.B) {
          float2* dst = reinterpret_cast<float2*>(part + ((size_t)ks * a.B + b0 + i) * W + j);
          *dst = make_float2(acc0[i], acc1[i]);
        }
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// latent_append, pass 2: sum the chunks in order, rotate the RoPE part at
// pos[b], round once and store into the page slot of position pos[b].
// One thread per (b, column pair).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void append_finalize_kernel(const float* __restrict__ part, const int* __restrict__ pos,
                                       const int* __restrict__ page_table, T* __restrict__ lat, T* __restrict__ rop,
                                       int* __restrict__ err, AppendArgs a, RopeTable tab) {
  const int W = a.d_c + a.d_r;
  const int pairs = W / 2;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= a.B * pairs) return;
  const int b = idx / pairs, j = 2 * (idx % pairs);
  float x0 = 0.f, x1 = 0.f;
  for (int ks = 0; ks < a.KS; ++ks) {
    const float2 v = *reinterpret_cast<const float2*>(part + ((size_t)ks * a.B + b) * W + j);
    x0 += v.x;
    x1 += v.y;
  }
  const int p = __ldg(pos + b);
  if (p < 0 || p >= a.maxp * kPage) {
    report_error(err, kErrDeviceCheck, b, p);
    return;
  }
  const int pg = page_of(page_table, a.maxp, a.num_pages, b, p, err);
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

cudaError_t launch_append(int dtype, const void* h, const void* W_DKV, const void* W_KR, const int* pos,
                          const int* page_table, void* lat, void* rop, float* part, int* err, const AppendArgs& a,
                          const RopeTable& tab, cudaStream_t st) {
  const int W = a.d_c + a.d_r;
  const int thr = ((W / 2 + 31) / 32) * 32;
  const int n2 = a.B * (W / 2);
  if (dtype == 1) {
    append_partial_kernel<__nv_bfloat16><<<a.KS, thr, 0, st>>>(
        (const __nv_bfloat16*)h, (const __nv_bfloat16*)W_DKV, (const __nv_bfloat16*)W_KR, part, a);
    append_finalize_kernel<__nv_bfloat16><<<(n2 + 127) / 128, 128, 0, st>>>(
        part, pos, page_table, (__nv_bfloat16*)lat, (__nv_bfloat16*)rop, err, a, tab);
  } else {
    append_partial_kernel<float><<<a.KS, thr, 0, st>>>((const float*)h, (const float*)W_DKV,
                                                           (const float*)W_KR, part, a);
    append_finalize_kernel<float><<<(n2 + 127) / 128, 128, 0, st>>>(part, pos, page_table, (float*)lat,
                                                                     (float*)rop, err, a, tab);
  }
  return cudaGetLastError();
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
    const int pg = page_of(page_table, a.maxp, a.num_pages, b, p, err);
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
