// Host-side caches: TMA tensor maps and per-kernel shared-memory limits, so a
// repeated call with the same buffers does no re-encoding.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mlra {

// 2-D bf16 tensor (rows x cols, cols contiguous), box box_cols x box_rows,
// 128-byte swizzle.  Returns false if the driver rejects it.
bool tmap_2d(CUtensorMap* out, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows);
// The same with a 64-byte swizzle (box_cols * 2 <= 64).
bool tmap_2d_sw64(CUtensorMap* out, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                  uint32_t box_rows);
// [B][H][K] bf16 as a 3-D tensor, box 64 x 1 x Bp (rows past B read as zero).
bool tmap_3d_batch(CUtensorMap* out, const void* base, uint64_t K, uint64_t H, uint64_t B, uint32_t Bp);
// Raises a kernel's dynamic shared-memory limit on the current device once.
cudaError_t ensure_smem(const void* func, int bytes);
// Records `ev` on `stream`; under stream capture as an external event node,
// so that graph replays still time the stages.
void record_event(cudaEvent_t ev, cudaStream_t stream);
void host_cache_clear();

}  // namespace mlra
