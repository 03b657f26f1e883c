// Sequence-sharded decode across GPUs: the two steps that are not the
// single-GPU path's.
//
// When a sequence's cached tokens are spread over R GPUs, each GPU attends
// its own token range and reduces its split-KV partials to one partial per
// (sequence, head, branch): the latent output normalised over its tokens,
// and the log-sum-exp of its scores (base 2).  After the R partials are
// gathered, the merge weighs each by 2^(lse_r - lse) with
// lse = log2 sum_r 2^(lse_r), which is the softmax over all the sequence's
// tokens (flash-decoding's combine, applied across GPUs), then applies the
// branch weight and the output up-projection.  Method: yololab.net,
// "超越 GQA 的推理革命…", section "矩陣吸收" (W_UV applied after attention);
// wispaper.ai, "MLRA：突破 MLA 并行瓶颈…", section "1. 痛点" (long-context
// decode is memory-bound, so its cache bytes are what gets spread).
#include "launch.h"

namespace mlra {
namespace {

// One warp per (b, h): the split-KV partials of sequence b (pieces at slots
// c + b for workers c0..c1) reduced to o[b, h, :] normalised per branch and
// lse[b, br, h] = M + log2(L) (-inf, with o = 0, for an empty range).
// grid (B, ceil(H / 4)), block 128.
__global__ void __launch_bounds__(128) partial_kernel(const float* __restrict__ o_part,
                                                      const float* __restrict__ ml_part,
                                                      const int* __restrict__ seq_lens, float* __restrict__ o_out,
                                                      float* __restrict__ lse_out, CombineArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int h = blockIdx.y * 4 + warp;
  const int maxL = a.maxp * kPage;
  long long T = 0, P = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int bb = base + lane;
    const int np = bb < a.B ? npages_of(seq_len_at(seq_lens, bb, maxL)) : 0;
    T += warp_sum_i(np);
    P += warp_sum_i(bb < b ? np : 0);
  }
  if (h >= a.H) return;
  const int np = npages_of(seq_len_at(seq_lens, b, maxL));
  const int d_cb = a.d_c / a.n_branch;
  float* dst = o_out + ((size_t)b * a.H + h) * a.d_c;
  if (np == 0) {
    for (int d = lane; d < a.d_c; d += 32) dst[d] = 0.f;
    if (lane < a.n_branch) lse_out[((size_t)b * a.n_branch + lane) * a.H + h] = -INFINITY;
    return;
  }
  const int c0 = worker_of_page(P, T, a.G);
  const int c1 = worker_of_page(P + np - 1, T, a.G);
  auto empty = [&](int c) { return worker_start(c, T, a.G) == worker_start(c + 1, T, a.G); };
  for (int br = 0; br < a.n_branch; ++br) {
    float M = -INFINITY;
    for (int c = c0; c <= c1; ++c)
      if (!empty(c)) M = fmaxf(M, ml_part[(((size_t)(c + b) * a.n_branch + br) * 2 + 0) * a.H + h]);
    float Lsum = 0.f;
    for (int c = c0; c <= c1; ++c) {
      if (empty(c)) continue;
      const size_t base = ((size_t)(c + b) * a.n_branch + br) * 2;
      Lsum += exp2f(ml_part[(base + 0) * a.H + h] - M) * ml_part[(base + 1) * a.H + h];
    }
    const float inv = 1.f / Lsum;
    for (int d = br * d_cb + lane; d < (br + 1) * d_cb; d += 32) {
      float acc = 0.f;
      for (int c = c0; c <= c1; ++c) {
        if (empty(c)) continue;
        const size_t base = ((size_t)(c + b) * a.n_branch + br) * 2;
        acc = fmaf(exp2f(ml_part[(base + 0) * a.H + h] - M), o_part[((size_t)(c + b) * a.H + h) * a.d_c + d], acc);
      }
      dst[d] = acc * inv;
    }
    if (lane == 0) lse_out[((size_t)b * a.n_branch + br) * a.H + h] = M + log2f(Lsum);
  }
}

// One warp per (b, h): R gathered partials merged into o_lat[b, h, :]
// (branch_scale folded in), in the parts' order, so every GPU that merges
// the same gathered parts gets the same bits.  grid (B, ceil(H / 4)), block 128.
template <typename OT>
__global__ void __launch_bounds__(128) merge_kernel(const float* __restrict__ o_parts,
                                                    const float* __restrict__ lse_parts, OT* __restrict__ o_lat, int R,
                                                    int B, int H, int d_c, int n_branch, float branch_scale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int h = blockIdx.y * 4 + warp;
  if (h >= H) return;
  const int d_cb = d_c / n_branch;
  const size_t o_stride = (size_t)B * H * d_c, l_stride = (size_t)B * n_branch * H;
  OT* dst = o_lat + ((size_t)b * H + h) * d_c;
  for (int br = 0; br < n_branch; ++br) {
    const size_t li = ((size_t)b * n_branch + br) * H + h;
    float M = -INFINITY;
    for (int r = 0; r < R; ++r) M = fmaxf(M, lse_parts[r * l_stride + li]);
    if (M == -INFINITY) {  // no part holds a token of this sequence
      for (int d = br * d_cb + lane; d < (br + 1) * d_cb; d += 32) dst[d] = from_f<OT>(0.f);
      continue;
    }
    float S = 0.f;
    for (int r = 0; r < R; ++r) S += exp2f(lse_parts[r * l_stride + li] - M);
    const float scale = branch_scale / S;
    for (int d = br * d_cb + lane; d < (br + 1) * d_cb; d += 32) {
      float acc = 0.f;
      for (int r = 0; r < R; ++r)
        acc = fmaf(exp2f(lse_parts[r * l_stride + li] - M), o_parts[r * o_stride + ((size_t)b * H + h) * d_c + d], acc);
      dst[d] = from_f<OT>(acc * scale);
    }
  }
}

}  // namespace

cudaError_t launch_partial(const float* o_part, const float* ml_part, const int* seq_lens, float* o_out,
                           float* lse_out, const CombineArgs& a, cudaStream_t st) {
  partial_kernel<<<dim3(a.B, (a.H + 3) / 4), 128, 0, st>>>(o_part, ml_part, seq_lens, o_out, lse_out, a);
  return cudaGetLastError();
}

cudaError_t launch_merge(bool out_bf16, const float* o_parts, const float* lse_parts, void* o_lat, int R, int B, int H,
                         int d_c, int n_branch, float branch_scale, cudaStream_t st) {
  const dim3 grid(B, (H + 3) / 4);
  if (out_bf16)
    merge_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(o_parts, lse_parts, static_cast<__nv_bfloat16*>(o_lat), R, B,
                                                      H, d_c, n_branch, branch_scale);
  else
    merge_kernel<float><<<grid, 128, 0, st>>>(o_parts, lse_parts, static_cast<float*>(o_lat), R, B, H, d_c,
                                              n_branch, branch_scale);
  return cudaGetLastError();
}

}  // namespace mlra
