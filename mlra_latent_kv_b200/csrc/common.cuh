// Device helpers shared by the libmlra kernels: element access, the device
// error record, the split-KV work plan and the RoPE rotation.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mlra {

constexpr int kPage = 64;          // tokens per cache page
constexpr int kMaxRopePairs = 32;  // d_r <= 64

// ---------------------------------------------------------------------------
// element access (bf16 storage, fp32 arithmetic)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------------------
// device error record: the first 16 bytes of the caller's workspace
//   [0] code (0 = none), [1] detail index, [2] second detail
// The first error wins (compare-and-swap from 0).
// ---------------------------------------------------------------------------
constexpr int kErrDeviceCheck = 5;
constexpr int kErrTimeout = 6;

__device__ __forceinline__ void report_error(int* rec, int code, int a, int b) {
  if (rec == nullptr) return;
  if (atomicCAS(rec, 0, code) == 0) {
    rec[1] = a;
    rec[2] = b;
  }
}

// Page id of token t of sequence b for a READ; an id outside [0, num_pages)
// is reported and replaced by page 0, so that no read leaves the pool (the
// call's result is void, and mlra_check_status says so).
__device__ __forceinline__ int page_of(const int* page_table, int maxp, int num_pages, int b, int t,
                                       int* err) {
  int pg = __ldg(page_table + (size_t)b * maxp + t / kPage);
  if (pg < 0 || pg >= num_pages) {
    report_error(err, kErrDeviceCheck, b, t);
    pg = 0;
  }
  return pg;
}

// Page id of token t of sequence b for a WRITE; an id outside [0, num_pages)
// is reported and -1 returned: the caller skips the store, because page 0 (or
// any other stand-in) belongs to some other live sequence.
__device__ __forceinline__ int page_for_write(const int* page_table, int maxp, int num_pages, int b, int t,
                                              int* err) {
  const int pg = __ldg(page_table + (size_t)b * maxp + t / kPage);
  if (pg < 0 || pg >= num_pages) {
    report_error(err, kErrDeviceCheck, b, t);
    return -1;
  }
  return pg;
}

// ---------------------------------------------------------------------------
// warp reductions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// ---------------------------------------------------------------------------
// split-KV work plan
//
// The pages of all sequences are laid end to end (sequence-major) into one
// range of T pages.  Worker c of G takes pages [c*T/G, (c+1)*T/G), which may
// cover the tail of one sequence and the head of the next.  Every piece
// (worker c, sequence b) writes one partial result to slot c + b; slots are
// unique because a worker's sequences are consecutive and the next worker
// starts no earlier than the last sequence of this one.  Slots < G + B - 1.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int npages_of(int L) { return L > 0 ? (L + kPage - 1) / kPage : 0; }
// Attended length of sequence b, clamped to what its page-table row can hold
// (maxL = max_pages_per_seq * page_size); every kernel reads lengths through
// this so that all of them agree on the plan.  Out-of-range lengths are
// reported by the attention kernel (see check_lengths).
__device__ __forceinline__ int seq_len_at(const int* seq_lens, int b, int maxL) {
  const int L = __ldg(seq_lens + b);
  return L < 0 ? 0 : (L > maxL ? maxL : L);
}
// Reports every length outside [0, maxL]; run by one CTA.
__device__ __forceinline__ void check_lengths(const int* seq_lens, int B, int maxL, int* err) {
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int L = __ldg(seq_lens + b);
    if (L < 0 || L > maxL) report_error(err, kErrDeviceCheck, b, L);
  }
}
__device__ __forceinline__ long long worker_start(long long c, long long T, long long G) {
  return c * T / G;
}
// worker that owns global page g (0 <= g < T)
__device__ __forceinline__ int worker_of_page(long long g, long long T, long long G) {
  return (int)(((g + 1) * G - 1) / T);
}

struct WorkerPlan {
  long long T;        // total pages
  long long start;    // first global page of this worker
  long long end;      // one past the last
  int b;              // first sequence with a page in [start, end)
  long long prefix;   // global page index of sequence b's first page
};

// Computed by one full warp (all lanes get the result).
__device__ __forceinline__ WorkerPlan plan_worker(const int* seq_lens, int B, int G, int c, int maxL) {
  const int lane = threadIdx.x & 31;
  long long T = 0;
  for (int base = 0; base < B; base += 32) {
    int np = (base + lane < B) ? npages_of(seq_len_at(seq_lens, base + lane, maxL)) : 0;
    T += warp_sum_i(np);
  }
  WorkerPlan wp;
  wp.T = T;
  wp.start = T > 0 ? worker_start(c, T, G) : 0;
  wp.end = T > 0 ? worker_start(c + 1, T, G) : 0;
  wp.b = B;
  wp.prefix = T;
  if (wp.start >= wp.end) return wp;
  long long prefix = 0;
  for (int base = 0; base < B; base += 32) {
    int np = (base + lane < B) ? npages_of(seq_len_at(seq_lens, base + lane, maxL)) : 0;
    int incl = warp_incl_scan(np);
    bool hit = np > 0 && prefix + incl > wp.start;
    unsigned m = __ballot_sync(0xffffffffu, hit);
    if (m) {
      int l = __ffs(m) - 1;
      int excl = __shfl_sync(0xffffffffu, incl - np, l);
      wp.b = base + l;
      wp.prefix = prefix + excl;
      return wp;
    }
    prefix += __shfl_sync(0xffffffffu, incl, 31);
  }
  return wp;
}

// Walks the pieces of one worker.  Usage:
//   SegWalk w(plan); while (w.next(seq_lens, B)) { w.b, w.pg0, w.pg1, w.L }
struct SegWalk {
  long long start, end, prefix;
  int b, B_, maxL;
  int pg0, pg1, L;  // current piece: pages [pg0, pg1) of sequence b (of length L)
  bool first;
  __device__ __forceinline__ SegWalk(const WorkerPlan& p, int B, int maxL_)
      : start(p.start), end(p.end), prefix(p.prefix), b(p.b), B_(B), maxL(maxL_), pg0(0), pg1(0), L(0),
        first(true) {}
  __device__ __forceinline__ bool next(const int* seq_lens) {
    if (!first) {
      prefix += npages_of(L);
      ++b;
    }
    first = false;
    while (b < B_ && prefix < end) {
      L = seq_len_at(seq_lens, b, maxL);
      int np = npages_of(L);
      if (np > 0 && prefix + np > start) {
        long long lo = start > prefix ? start : prefix;
        long long hi = end < prefix + np ? end : prefix + np;
        pg0 = (int)(lo - prefix);
        pg1 = (int)(hi - prefix);
        return true;
      }
      prefix += np;
      ++b;
    }
    return false;
  }
};

// ---------------------------------------------------------------------------
// RoPE: pair i of a vector at position pos turns by pos * theta[i], with
// theta[i] = base^(-2i/d_r) computed on the host in double precision.  The
// angle is formed and reduced to [-pi, pi] in double, then sin/cos are taken
// in single precision (accurate at any position, cheap on the device).
// ---------------------------------------------------------------------------
struct RopeTable {
  double theta[kMaxRopePairs];
};

__device__ __forceinline__ void rope_sincos(const RopeTable& tab, int i, int pos, float* s, float* c) {
  const double two_pi = 6.283185307179586476925286766559;
  double ang = (double)pos * tab.theta[i];
  double r = fma(-two_pi, rint(ang * (1.0 / two_pi)), ang);
  sincosf((float)r, s, c);
}

}  // namespace mlra
