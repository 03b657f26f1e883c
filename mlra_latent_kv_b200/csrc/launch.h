// Internal launcher interface between the C-ABI host code and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace mlra {

struct AbsorbArgs {
  int B, H, Hq, d_h, d_c, d_r;
  float q_scale;  // multiplies q_lat and the rotated q_rope (1 unless the attention kernel expects pre-scaled queries)
};

struct AttnArgs {
  int B, H, d_c, d_r, n_branch, maxp, num_pages, G;
  float scale_log2;  // softmax_scale * log2(e)
};

struct CombineArgs {
  int B, H, d_c, n_branch, G, maxp;
  float branch_scale;
};

struct UpArgs {
  int B, H, d_c, d_v;
};

struct AppendArgs {
  int B, D, d_c, d_r, maxp, num_pages, KS;
};

struct StoreArgs {
  int n_tokens, B, d_c, d_r, maxp, num_pages;
};

// dtype: 0 = fp32, 1 = bf16 (storage type of inputs/caches/outputs)
cudaError_t launch_absorb(int dtype, bool q_bf16, const void* q_nope, const void* q_rope, const int* q_pos,
                          const void* W_UK, void* q_ws, const AbsorbArgs& a, const RopeTable& tab, cudaStream_t st);
cudaError_t launch_attend_simt(int dtype, const float* q_ws, const void* lat, const void* rop, const int* page_table,
                               const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                               cudaStream_t st);
cudaError_t launch_combine(bool out_bf16, const float* o_part, const float* ml_part, const int* seq_lens,
                           void* o_lat, const CombineArgs& a, cudaStream_t st);
cudaError_t launch_upproj(int dtype, bool in_bf16, const void* o_lat, const void* W_UV, void* out, const UpArgs& a,
                          cudaStream_t st);

// sequence-sharded decode (seq_parallel.cu): a rank's partial, and the merge of R gathered partials
cudaError_t launch_partial(const float* o_part, const float* ml_part, const int* seq_lens, float* o_out,
                           float* lse_out, const CombineArgs& a, cudaStream_t st);
cudaError_t launch_merge(bool out_bf16, const float* o_parts, const float* lse_parts, void* o_lat, int R, int B, int H,
                         int d_c, int n_branch, float branch_scale, cudaStream_t st);

cudaError_t launch_append(int dtype, const void* h, const void* W_DKV, const void* W_KR, const int* pos,
                          const int* page_table, void* lat, void* rop, float* part, int* err, const AppendArgs& a,
                          const RopeTable& tab, cudaStream_t st);
cudaError_t launch_store(int dtype, const void* c_kv, const void* k_rope, const int* tok_seq, const int* tok_pos,
                         const int* page_table, void* lat, void* rop, int* err, const StoreArgs& a,
                         const RopeTable& tab, cudaStream_t st);

}  // namespace mlra

#include "../../include/mlra.h"

namespace mlra {
// defined in append_noalloc.cu
void noalloc_forget_scratch();
// defined in mlra_api.cu
mlra_status internal_check_dims(const mlra_dims* d);
mlra_status internal_fail(mlra_status st, const char* msg);
RopeTable internal_rope_table(const mlra_dims* d);
}  // namespace mlra
