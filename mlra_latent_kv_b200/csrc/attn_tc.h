// tcgen05 (5th-generation tensor core) split-KV latent attention for sm_100a.
#pragma once

#include <cuda_runtime.h>

#include "launch.h"

namespace mlra {

// Query rows per sequence the tcgen05 kernels read (heads padded with zero rows).
constexpr int kTcHeads = 128;

// Whether the tcgen05 attention kernels implement this shape.
bool tc_supported(int dtype, int H, int d_c, int d_r, int n_branch, int d_h, int d_v);

// Launch the tcgen05 split-KV attention: same partial-result contract as the
// CUDA-core kernel (slot c + b per worker piece, m/l per branch in log2 units).
// pdl: launch as a programmatic dependent of the previous kernel in the stream
// (its prologue overlaps that kernel; the queries are read after it completes).
cudaError_t launch_attend_tc(const void* q_ws, const void* lat, const void* rop, const int* page_table,
                             const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                             cudaStream_t st, bool pdl);

// The MLA kernel for at most 32 heads (attn_small.cu): query rows replicated
// into every TMEM lane quarter, token-sliced softmax, exact fp32 score
// exchange, PV with the operands swapped.  launch_attend_tc dispatches to it.
bool tc_small_supported(int H, int n_branch);
cudaError_t launch_attend_tc_small(const void* q_ws, const void* lat, const void* rop, const int* page_table,
                                   const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                                   cudaStream_t st, bool pdl);

// One 128-dim branch per CTA (attn_branch.cu): the one-branch decode of a
// 128-dim latent (a branch-parallel MLRA rank's share), 33 to 128 heads.  The
// grid is n_branch x G CTAs (G page-range workers per branch).
bool tc_branch_supported(int H, int d_c, int d_r, int n_branch);
int tc_branch_workers(int sms, int n_branch);
cudaError_t launch_attend_tc_branch(const void* q_ws, const void* lat, const void* rop, const int* page_table,
                                    const int* seq_lens, float* o_part, float* ml_part, int* err, const AttnArgs& a,
                                    cudaStream_t st, bool pdl);

// Name of the attention kernel variant launch_attend_tc picks for this shape.
const char* tc_variant_name(int H, int d_c, int n_branch);

// Frees the host-side tensor-map cache.
void tc_shutdown();

}  // namespace mlra
