// tcgen05 kernels of the per-head contractions: query absorption and the
// split combine fused with the output up-projection.
#pragma once

#include <cuda_runtime.h>

#include "launch.h"

namespace mlra {

struct GemmArgs {
  int B, Bp;       // batch and batch padded to a multiple of 16 (the MMA's N)
  int H;
  int K;           // contraction length: d_h (absorption) or d_c (up-projection)
  int d_c, d_r;
  int N_out;       // d_v (up-projection)
  int G, n_branch, maxp;
  float branch_scale;
  float q_scale;   // absorption only: multiplies q_lat and the rotated q_rope before rounding
  int R;           // combine + up-projection only: sequences per CTA (the MMA's N; 16 or 32)
};

int batch_pad(int B);
// shapes the absorption kernel implements
bool absorb_tc_supported(int dtype, int B, int d_h, int d_c);
// shapes the fused combine + up-projection kernel implements
bool upproj_tc_supported(int dtype, int B, int d_c, int d_v, int G, int n_branch);

cudaError_t launch_absorb_tc(const void* q_nope, const void* q_rope, const int* q_pos, const void* W_UK, void* q_ws,
                             int* err, const GemmArgs& a, const RopeTable& tab, cudaStream_t st);
// pdl: launch as a programmatic dependent of the attention kernel (weights and
// split plan are loaded while it retires; the partials are read after it completes).
cudaError_t launch_combine_upproj_tc(const float* o_part, const float* ml_part, const int* seq_lens, const void* W_UV,
                                     void* out, int* err, const GemmArgs& a, cudaStream_t st, bool pdl);

}  // namespace mlra
