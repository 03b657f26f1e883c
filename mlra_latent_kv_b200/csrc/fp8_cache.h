// FP8 latent cache (E4M3 codes, one fp32 scale per page and tensor): the
// CUDA-core attention over it and the quantizer of a bf16 (dtype 1) or fp32
// pool (simt_kernels.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"

namespace mlra {

cudaError_t launch_attend_simt_fp8(const float* q_ws, const uint8_t* lat, const uint8_t* rop, const float* lat_scale,
                                   const float* rop_scale, const int* page_table, const int* seq_lens, float* o_part,
                                   float* ml_part, int* err, const AttnArgs& a, cudaStream_t st);
cudaError_t launch_quantize_pages(int dtype, const void* pool, int num_pages, int n_per_page, uint8_t* codes,
                                  float* scales, cudaStream_t st);

}  // namespace mlra
