// latent_append_noalloc: latent_append for callers that cannot allocate
// device memory (an engine whose cache pool owns all HBM and forbids later
// cudaMalloc, a decode loop that must not risk the synchronisation an
// allocation can cause, a plugin host that passes buffers but no allocator).
// The one-launch append keeps its partial sums on chip and needs no scratch;
// the two-kernel form (columns that do not split into 16-byte groups, or a
// hidden width too large for the one-launch form's shared memory) keeps its
// split-K partial sums here, in one fixed, file-scope device array, where
// latent_append keeps them in the caller's workspace.  There is no
// counterpart on the pages.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "append_forms.h"
#include "launch.h"

using namespace mlra;

namespace {

// The scratch: every GPU that loads the library holds one copy until exit.
static __device__ __align__(256) unsigned char g_append_scratch[MLRA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Device address of g_append_scratch per device ordinal, with the context it
// was looked up in: a context created later (after cudaDeviceReset, or after
// the primary context was released and made again) holds the array at a new
// address, so the entry is looked up again when the current context differs.
struct ScratchEntry {
  CUcontext ctx;
  void* ptr;
};
ScratchEntry g_scratch_dev[kMaxDevices] = {};
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;  // the driver's cuCtxGetCurrent, looked up through the runtime

// The calling thread's current context, or nullptr if there is none (or the
// driver function cannot be had, in which case the cache is used per device).
CUcontext current_context() {
  if (g_ctx_current == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  }
  CUcontext ctx = nullptr;
  return g_ctx_current(&ctx) == CUDA_SUCCESS ? ctx : nullptr;
}

// Device address of the scratch on the current device.  Host code cannot use
// the array's name as an address (it is a host-side stand-in), so the first
// call on each device asks the runtime for it, with that device current, and
// keeps the answer for that device's current context.
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  CUcontext ctx = current_context();
  ScratchEntry& ent = g_scratch_dev[dev];
  if (ent.ptr == nullptr || ctx == nullptr || ent.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_append_scratch);  // makes the device's primary context current if needed
    if (e != cudaSuccess) return e;
    ent.ctx = current_context();
    ent.ptr = p;
  }
  *out = ent.ptr;
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace mlra {
// Forgets every cached scratch address (mlra_shutdown calls this).
void noalloc_forget_scratch() {
  std::lock_guard<std::mutex> lock(g_mu);
  for (ScratchEntry& ent : g_scratch_dev) ent = ScratchEntry{};
}
}  // namespace mlra

extern "C" MLRA_API mlra_status latent_append_noalloc(const mlra_dims* dims, int d_model, const void* h,
                                                      const void* W_DKV, const void* W_KR, const int32_t* pos,
                                                      const int32_t* page_table, void* latent_cache,
                                                      void* rope_cache, cudaStream_t stream) {
  char msg[256];
  mlra_status st = internal_check_dims(dims);
  if (st != MLRA_OK) return st;
  if (d_model < 1) return internal_fail(MLRA_ERR_INVALID_ARG, "d_model must be >= 1");
  const void* ptrs[] = {h, W_DKV, W_KR, latent_cache, rope_cache};
  const char* names[] = {"h", "W_DKV", "W_KR", "latent_cache", "rope_cache"};
  for (int i = 0; i < 5; ++i) {
    if (ptrs[i] == nullptr || !aligned16(ptrs[i])) {
      snprintf(msg, sizeof(msg), "%s is NULL or not 16-byte aligned", names[i]);
      return internal_fail(MLRA_ERR_INVALID_ARG, msg);
    }
  }
  if (pos == nullptr || page_table == nullptr) return internal_fail(MLRA_ERR_INVALID_ARG, "pos/page_table is NULL");
  const int KS = (d_model + 63) / 64;
  const bool scratch_used = append_uses_scratch(dims->dtype, d_model, dims->d_c, dims->d_r);
  const size_t need = scratch_used ? (size_t)KS * dims->B * (dims->d_c + dims->d_r) * sizeof(float) : 0;
  if (need > MLRA_NOALLOC_SCRATCH_BYTES) {
    snprintf(msg, sizeof(msg),
             "latent_append_noalloc: B=%d, d_model=%d, d_c+d_r=%d need %zu bytes of scratch; the fixed scratch "
             "holds %u bytes (call latent_append with a workspace instead)",
             dims->B, d_model, dims->d_c + dims->d_r, need, (unsigned)MLRA_NOALLOC_SCRATCH_BYTES);
    return internal_fail(MLRA_ERR_UNSUPPORTED, msg);
  }
  void* scratch = nullptr;
  cudaError_t e = cudaSuccess;
  if (scratch_used) {
    e = scratch_address(&scratch);
    if (e != cudaSuccess) {
      snprintf(msg, sizeof(msg), "latent_append_noalloc: looking up the scratch address: %s", cudaGetErrorString(e));
      return internal_fail(MLRA_ERR_CUDA, msg);
    }
  }
  // the two-kernel form's pass 1 writes every partial sum pass 2 reads, so the scratch needs no clearing
  AppendArgs a{dims->B, d_model, dims->d_c, dims->d_r, dims->max_pages_per_seq, dims->num_pages, KS};
  e = launch_append(dims->dtype, h, W_DKV, W_KR, pos, page_table, latent_cache, rope_cache,
                    static_cast<float*>(scratch), /*err=*/nullptr, a, internal_rope_table(dims), stream);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "latent_append_noalloc launch: %s", cudaGetErrorString(e));
    return internal_fail(MLRA_ERR_CUDA, msg);
  }
  return MLRA_OK;
}
