/*
 * mlra.h -- C ABI of libmlra: latent-KV (MLA / MLRA-n) single-token decode
 * attention over a compressed, paged cache, for NVIDIA B200 (sm_100a).
 *
 * Method (pages cited by site, title, section):
 *   - yololab.net, "超越 GQA 的推理革命：DeepSeek 如何用 MLA 重新定義 LLM 的記憶體
 *     極限？": section "1. 鍵值聯合低秩壓縮" (each token caches only a latent
 *     c_KV), section "2. 解耦旋轉位置編碼" (a small RoPE'd key k_rope is kept
 *     beside it, uncompressed), section "矩陣吸收：推理加速的最後一哩路" (W_UK is
 *     folded into the query and W_UV applied after attention, so per-head K/V
 *     are never formed).
 *   - wispaper.ai, "MLRA：突破 MLA 并行瓶颈，长文本解码提速 280%", section
 *     "2.1 架构拆解": the latent is cut into branches, each with its own
 *     softmax, and the output is the weighted sum of the branch outputs.
 *
 * Conventions for every entry point
 *   - Pointers named in a comment as [a, b, ...] are DEVICE pointers to dense
 *     row-major arrays with those extents (last index fastest), 16-byte aligned.
 *     Element type: the dims' dtype (bf16 or fp32) for floating arrays, int32
 *     for index arrays.  Nothing is retained after the call returns except the
 *     host-side cache of TMA descriptors keyed by (pointer, extents).
 *   - Ownership: the caller allocates and frees every buffer, including the
 *     workspace.  The library allocates no device memory in any call.
 *   - Asynchrony: kernels are enqueued on `stream`; the call returns before
 *     they finish.  Host-side argument errors are detected before anything is
 *     enqueued and leave every buffer untouched.
 *   - Errors: every call returns an mlra_status; mlra_last_error() gives the
 *     message of the last failure on the calling thread.  Errors found on the
 *     device (a page id outside [0, num_pages), a bounded wait that gave up)
 *     are recorded in the first 16 bytes of the workspace and read with
 *     mlra_check_status().  The workspace must be zero-filled once before its
 *     first use; mlra_check_status() clears what it reports.  A bad page id
 *     met on a read (decode) is replaced by page 0, so the read stays inside
 *     the pool and that call's output is void; met on a write (latent_append,
 *     latent_store, latent_append_noalloc) the token is not written at all,
 *     so no other sequence's page is touched.
 */
#ifndef MLRA_H_
#define MLRA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MLRA_API __attribute__((visibility("default")))
#else
#define MLRA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLRA_OK = 0,
  MLRA_ERR_INVALID_ARG = 1,  /* null pointer, bad extent, misaligned pointer */
  MLRA_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels implement */
  MLRA_ERR_WORKSPACE = 3,    /* workspace smaller than the *_workspace_bytes() figure */
  MLRA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  MLRA_ERR_DEVICE_CHECK = 5, /* a device-side range check fired (see mlra_check_status) */
  MLRA_ERR_TIMEOUT = 6       /* a device-side bounded wait gave up */
} mlra_status;

typedef enum { MLRA_F32 = 0, MLRA_BF16 = 1 } mlra_dtype;

/* Which attention kernel family runs.  AUTO picks the tcgen05 kernels when the
 * shape is one they implement (bf16, d_c = 512, d_r = 64, H <= 128,
 * n_branch in {1, 2, 4}) and the CUDA-core kernels otherwise. */
typedef enum { MLRA_KERNEL_AUTO = 0, MLRA_KERNEL_SIMT = 1, MLRA_KERNEL_TC = 2 } mlra_kernel;

/* Shape and parameters of a decode batch.
 *   B            sequences in the batch
 *   H            query heads
 *   d_h          per-head query/key content width (q_nope, rows of W_UK)
 *   d_v          per-head value width (columns of W_UV)
 *   d_c          latent width c_KV (all branches together)
 *   d_r          decoupled RoPE key width (even)
 *   n_branch     MLRA branches; 1 = MLA.  Branch br owns latent columns
 *                [br*d_c/n_branch, (br+1)*d_c/n_branch)
 *   page_size    tokens per cache page (64)
 *   max_pages_per_seq  row length of page_table
 *   num_pages    pages in the cache pool
 *   softmax_scale  logit scale; 0 selects 1/sqrt(d_h + d_r)
 *   branch_scale   weight of each branch output in the sum (1 for MLA)
 *   rope_base      RoPE base; 0 selects 10000
 *   dtype        element type of caches, queries, weights and outputs
 *   num_splits   split-KV workers; 0 = chosen from the device's SM count
 *   kernel       an mlra_kernel value                                      */
typedef struct {
  int B, H, d_h, d_v, d_c, d_r;
  int n_branch;
  int page_size;
  int max_pages_per_seq;
  int num_pages;
  float softmax_scale;
  float branch_scale;
  float rope_base;
  int dtype;
  int num_splits;
  int kernel;
} mlra_dims;

/* Bytes of workspace a decode call with these dims needs (0 on invalid dims;
 * the reason is in mlra_last_error()).  With num_splits = 0 it queries the
 * current device. */
MLRA_API size_t mlra_workspace_bytes(const mlra_dims* dims);

/* mla_decode -- one decode step of MLA (n_branch must be 1; branch_scale is
 * taken as 1).  Absorbed form, yololab.net section "矩陣吸收":
 *   q_lat[b,h]  = q_nope[b,h] . W_UK[h]                         (d_c)
 *   q_rot[b,h]  = RoPE(q_rope[b,h], q_pos[b])                   (d_r)
 *   s[b,h,t]    = scale * (q_lat . c[b,t] + q_rot . k[b,t]),  t < seq_lens[b]
 *   o_lat[b,h]  = softmax_t(s) . c[b,:]                         (d_c)
 *   out[b,h]    = o_lat[b,h] . W_UV[h]                          (d_v)
 * where c[b,t] = latent_cache[page_table[b][t/64]][t%64] and k[b,t] the same
 * slot of rope_cache (stored rotated at position t).  seq_lens[b] = 0 gives a
 * zero row.
 *   q_nope [B,H,d_h]   q_rope [B,H,d_r] (un-rotated)   q_pos [B] int32
 *   W_UK [H,d_h,d_c]   W_UV [H,d_c,d_v]
 *   latent_cache [num_pages,page_size,d_c]   rope_cache [num_pages,page_size,d_r]
 *   page_table [B,max_pages_per_seq] int32   seq_lens [B] int32
 *   out [B,H,d_v]  (written)
 *   workspace: >= mlra_workspace_bytes(dims) bytes, 256-byte aligned. */
MLRA_API mlra_status mla_decode(const mlra_dims* dims, const void* q_nope, const void* q_rope,
                       const int32_t* q_pos, const void* W_UK, const void* W_UV,
                       const void* latent_cache, const void* rope_cache,
                       const int32_t* page_table, const int32_t* seq_lens, void* out,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* mlra_decode -- MLRA-n decode (wispaper.ai section "2.1 架构拆解"): the same
 * arguments as mla_decode; each branch br runs its own softmax over
 *   s_br = scale * (q_lat[br cols] . c[br cols] + q_rot . k)
 * (the rope score is shared by all branches) and
 *   out = sum_br branch_scale * softmax(s_br) . c[br cols] . W_UV[h][br rows]. */
MLRA_API mlra_status mlra_decode(const mlra_dims* dims, const void* q_nope, const void* q_rope,
                        const int32_t* q_pos, const void* W_UK, const void* W_UV,
                        const void* latent_cache, const void* rope_cache,
                        const int32_t* page_table, const int32_t* seq_lens, void* out,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* mlra_decode_profiled -- mlra_decode that also records stage_events[0..4]
 * (created by the caller) on `stream`: before query absorption, after it,
 * after split-KV attention, after the split combine, after the output
 * up-projection.  stage_events may be NULL. */
MLRA_API mlra_status mlra_decode_profiled(const mlra_dims* dims, const void* q_nope, const void* q_rope,
                                 const int32_t* q_pos, const void* W_UK, const void* W_UV,
                                 const void* latent_cache, const void* rope_cache,
                                 const int32_t* page_table, const int32_t* seq_lens, void* out,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream,
                                 cudaEvent_t* stage_events);

/* mlra_decode_host -- mlra_decode with the step's per-token inputs and its
 * output in host memory, for a caller whose queries arrive from (and whose
 * attention output goes back to) the host.  On `stream`, in order: copies
 * h_q_nope [B,H,d_h], h_q_rope [B,H,d_r], h_q_pos [B] and h_seq_lens [B] into
 * device staging space inside `workspace`, runs mlra_decode on them, and
 * copies out [B,H,d_v] to h_out.  Weights, the cache and the page table stay
 * device-resident (device pointers, as in mla_decode).  The host buffers must
 * stay valid (and h_out unread) until the stream reaches the end of the call;
 * pinned host memory makes the copies asynchronous.
 *   workspace: >= mlra_decode_host_workspace_bytes(dims) bytes, 256-byte
 *   aligned (the decode workspace followed by the staging space).
 * The pages specify no host interface; this call only moves the decode's
 * inputs and output across the host boundary. */
MLRA_API size_t mlra_decode_host_workspace_bytes(const mlra_dims* dims);
MLRA_API mlra_status mlra_decode_host(const mlra_dims* dims, const void* h_q_nope, const void* h_q_rope,
                                      const int32_t* h_q_pos, const void* W_UK, const void* W_UV,
                                      const void* latent_cache, const void* rope_cache,
                                      const int32_t* page_table, const int32_t* h_seq_lens, void* h_out,
                                      void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* FP8 latent cache (an extension: yunthe.com, "多头潜在注意力机制：内存优化与推理
 * 加速的革新方案", section "一、技术演进背景", names 8-bit quantization of the
 * KV cache as a way to shrink it, at some cost in precision; the format below
 * is this library's reading, as the page fixes none).
 *
 * Format: every element of latent_cache [P,64,d_c] and rope_cache [P,64,d_r]
 * is one FP8 E4M3 code (1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
 * no infinities, S.1111.111 = NaN, largest finite 448) in a uint8_t, and each
 * page of each tensor has one fp32 scale: value = decode(code) * scale[page].
 *
 * mlra_quantize_pages_fp8 -- quantize a bf16 (dims->dtype = MLRA_BF16) or
 * fp32 pool of dims->num_pages pages: scale = (largest finite |x| on the page)
 * / 448 in fp32 (1 for a page with no nonzero finite value); code = E4M3 of
 * fl32(x / scale), nearest with ties to even, saturating at +-448; NaN stays
 * NaN.  Outputs: latent_fp8 [P,64,d_c] and rope_fp8 [P,64,d_r] bytes,
 * latent_scale [P] and rope_scale [P] fp32 (4-byte aligned), all device
 * memory owned by the caller.  Asynchronous on `stream`; returns
 * MLRA_ERR_INVALID_ARG for a NULL pointer.
 *
 * mlra_decode_fp8 -- mlra_decode over such a cache: the same arguments, with
 * the FP8 pools and their scales in place of latent_cache and rope_cache.  It
 * runs on the CUDA-core kernels (fp32 arithmetic on the dequantized values);
 * dims->kernel = MLRA_KERNEL_TC is refused with MLRA_ERR_UNSUPPORTED.
 *   workspace: >= mlra_workspace_bytes() of the same dims with kernel =
 *   MLRA_KERNEL_SIMT, 256-byte aligned. */
MLRA_API mlra_status mlra_quantize_pages_fp8(const mlra_dims* dims, const void* latent_cache,
                                             const void* rope_cache, uint8_t* latent_fp8, uint8_t* rope_fp8,
                                             float* latent_scale, float* rope_scale, cudaStream_t stream);
MLRA_API mlra_status mlra_decode_fp8(const mlra_dims* dims, const void* q_nope, const void* q_rope,
                                     const int32_t* q_pos, const void* W_UK, const void* W_UV,
                                     const uint8_t* latent_fp8, const uint8_t* rope_fp8,
                                     const float* latent_scale, const float* rope_scale,
                                     const int32_t* page_table, const int32_t* seq_lens, void* out,
                                     void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* mlra_describe_plan -- the kernels mla_decode / mlra_decode launch for
 * `dims`, as one NUL-terminated line of ';'-separated key=value fields:
 *   family     tcgen05 | tcgen05+cuda-core | cuda-core (kernel AUTO picks
 *              tcgen05 wherever the shape allows; dims.kernel forces one)
 *   splits     split-KV workers;  kernels  launches per decode call
 *   absorb, attention, combine, upproj   the kernel of each stage
 * Touches no GPU memory.  With num_splits = 0 it reads the current device's
 * SM count (as the decode calls do).  Returns MLRA_ERR_INVALID_ARG when
 * buf_len is too short.  The pages have no counterpart: this reports which of
 * the library's own kernels serve the decode step of the method above. */
MLRA_API mlra_status mlra_describe_plan(const mlra_dims* dims, char* buf, size_t buf_len);

/* Sequence-sharded decode across GPUs (long contexts).  When the cached
 * tokens of every sequence are spread over R GPUs, each GPU attends its own
 * token range: mlra_attend_partial runs the decode's absorption and split-KV
 * attention on that GPU's cache and writes, per (sequence, head, branch), the
 * latent output normalised over its tokens and the log-sum-exp of its scores
 * in base 2 (the scores already carry softmax_scale * log2(e)):
 *   o   [B, H, d_c] fp32     o[b,h,br block] = sum_t p_t c_t,br / sum_t p_t
 *   lse [B, n_branch, H] fp32   log2 sum_t 2^(s_t)   (-inf and o = 0 when the
 *                                                     GPU holds no token of b)
 * After the R partials are gathered (the caller's all-gather, in a fixed rank
 * order), mlra_merge_upproj weighs part r by 2^(lse_r - lse) with
 * lse = log2 sum_r 2^(lse_r) -- the softmax over all of the sequence's tokens
 * -- folds in branch_scale and applies W_UV:
 *   o_parts [R, B, H, d_c] fp32, lse_parts [R, B, n_branch, H] fp32,
 *   out [B, H, d_v] (dtype), workspace >= mlra_merge_workspace_bytes(dims).
 * Positions: a GPU's cache and page table address its own tokens from 0, but
 * the stored rope keys must be rotated at their absolute positions (write the
 * cache through a page table indexed by absolute page, then attend through
 * that table's rows shifted to the GPU's first page); q_pos is absolute.
 * mlra_attend_partial takes the decode's arguments and workspace
 * (mlra_workspace_bytes) minus W_UV and out.  Method: yololab.net,
 * "超越 GQA 的推理革命…", section "矩陣吸收" (W_UV after attention); the merge
 * is the split-KV combine of the single-GPU path applied across GPUs. */
MLRA_API mlra_status mlra_attend_partial(const mlra_dims* dims, const void* q_nope, const void* q_rope,
                                         const int32_t* q_pos, const void* W_UK, const void* latent_cache,
                                         const void* rope_cache, const int32_t* page_table,
                                         const int32_t* seq_lens, float* o, float* lse, void* workspace,
                                         size_t workspace_bytes, cudaStream_t stream);
MLRA_API size_t mlra_merge_workspace_bytes(const mlra_dims* dims);
MLRA_API mlra_status mlra_merge_upproj(const mlra_dims* dims, int n_parts, const float* o_parts,
                                       const float* lse_parts, const void* W_UV, void* out, void* workspace,
                                       size_t workspace_bytes, cudaStream_t stream);

/* Bytes of workspace latent_append needs for hidden width d_model. */
MLRA_API size_t latent_append_workspace_bytes(const mlra_dims* dims, int d_model);

/* latent_append -- compress one new token per sequence into the cache
 * (yololab.net sections "1. 鍵值聯合低秩壓縮" and "2. 解耦旋轉位置編碼"):
 *   x = h[b] . [W_DKV | W_KR]           (fp32 accumulate)
 *   latent_cache[slot] = x[:d_c]          rope_cache[slot] = RoPE(x[d_c:], pos[b])
 * with slot = (page_table[b][pos[b]/page_size], pos[b] % page_size), both
 * rounded to the dtype (round to nearest even).  seq_lens is not touched; a
 * caller that then attends the new token passes seq_lens[b] = pos[b] + 1.
 *   h [B,d_model]   W_DKV [d_model,d_c]   W_KR [d_model,d_r]   pos [B] int32
 *   page_table [B,max_pages_per_seq] int32; the caches are written at one slot
 *   per sequence and nowhere else. */
MLRA_API mlra_status latent_append(const mlra_dims* dims, int d_model, const void* h, const void* W_DKV,
                          const void* W_KR, const int32_t* pos, const int32_t* page_table,
                          void* latent_cache, void* rope_cache, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream);

/* latent_store -- write already-compressed tokens into the paged cache
 * (prefill, or restoring a cache): for i < n_tokens, token row i goes to
 * sequence tok_seq[i] at position tok_pos[i]:
 *   latent_cache[slot] = c_kv[i]   (copied bit for bit)
 *   rope_cache[slot]   = RoPE(k_rope[i], tok_pos[i])   (rounded to nearest even)
 *   c_kv [n_tokens,d_c]   k_rope [n_tokens,d_r] (un-rotated)
 *   tok_seq, tok_pos [n_tokens] int32
 * workspace: at least 256 bytes (device error record). */
MLRA_API mlra_status latent_store(const mlra_dims* dims, int n_tokens, const void* c_kv, const void* k_rope,
                         const int32_t* tok_seq, const int32_t* tok_pos, const int32_t* page_table,
                         void* latent_cache, void* rope_cache, void* workspace,
                         size_t workspace_bytes, cudaStream_t stream);

/* latent_append_noalloc -- latent_append for callers that cannot allocate
 * device memory: a serving engine that reserved all HBM for its cache pool up
 * front and forbids later cudaMalloc (late allocations fragment memory or
 * fail once the pool is full), a decode loop that must not hit the device-wide
 * synchronisation cudaMalloc/cudaFree can cause, or a plugin host that hands
 * over input and output buffers but no allocator.  It computes exactly what
 * latent_append computes (same kernels, same result bits) but takes no
 * workspace: its split-K scratch is a fixed device array inside libmlra of
 * MLRA_NOALLOC_SCRATCH_BYTES (4 MiB), which every GPU that loads the library
 * holds until the process exits.  There is no counterpart on the pages; this
 * is an interface convenience only.
 *   - Scratch needed: none when the columns split into 16-byte groups (d_r
 *     a multiple of 8 for bf16, of 4 for fp32; d_c always is) and d_model <=
 *     81920: that append is one launch whose partial sums stay on chip (and
 *     latent_append_workspace_bytes is then the 256-byte error record).
 *     Otherwise the two-kernel form needs ceil(d_model/64) * B * (d_c + d_r)
 *     * 4 bytes; a call that needs more than the scratch returns
 *     MLRA_ERR_UNSUPPORTED and enqueues nothing.
 *   - The first call on each device that uses the scratch looks up the
 *     array's device address (cudaGetSymbolAddress) with that device
 *     current; make that first call before any stream capture.  The address is kept per device and
 *     context; after cudaDeviceReset (or any release of a device's primary
 *     context) call mlra_shutdown() before the next call, which forgets it.
 *   - Memory: the array lives in the same device module as every kernel of
 *     the library, so every process that uses any entry point holds its
 *     4 MiB on each device it runs on.  Under CUDA's lazy module loading (the
 *     default) that memory is taken when the library first launches a kernel
 *     or looks up a symbol on the device, not when it is loaded: an engine
 *     that reserves all free HBM for its pool should make one call of the
 *     library (e.g. a first latent_append_noalloc) on each device BEFORE it
 *     reserves the memory.
 *   - Every call shares the one array.  Each call overwrites the part it uses
 *     before reading it, so nothing has to start zeroed, but calls whose
 *     kernels overlap on the GPU (e.g. on two streams) race on it.
 *   - Device-side range checks still skip every write whose page id or
 *     position is out of range (nothing else in the cache changes), but
 *     their reports are not recorded (there is no workspace to hold them).
 * It allocates nothing and frees nothing. */
#define MLRA_NOALLOC_SCRATCH_BYTES (4u << 20)
MLRA_API mlra_status latent_append_noalloc(const mlra_dims* dims, int d_model, const void* h,
                                           const void* W_DKV, const void* W_KR, const int32_t* pos,
                                           const int32_t* page_table, void* latent_cache,
                                           void* rope_cache, cudaStream_t stream);

/* mlra_selftest_wait_timeout -- failure-detection self-test.  Launches one
 * small kernel on `stream` that waits on a device barrier nothing completes,
 * using the same bounded wait as every kernel of the library but with a limit
 * of limit_cycles SM clocks (in [1, 4e9]); the wait gives up, records
 * MLRA_ERR_TIMEOUT in the error record at the start of `workspace` (>= 256
 * bytes, zero-filled) and the kernel returns, so the context stays usable.
 * Read the result with mlra_check_status().  The pages have no counterpart:
 * this exists to test failure detection without hanging a GPU. */
MLRA_API mlra_status mlra_selftest_wait_timeout(void* workspace, long long limit_cycles, cudaStream_t stream);

/* Synchronises `stream`, reads the device error record in `workspace`, clears
 * it and returns MLRA_OK, MLRA_ERR_DEVICE_CHECK or MLRA_ERR_TIMEOUT (the
 * message, with the first offending index, goes to mlra_last_error()). */
MLRA_API mlra_status mlra_check_status(void* workspace, cudaStream_t stream);

/* Message of the last error on the calling thread ("" if none). */
MLRA_API const char* mlra_last_error(void);

/* Frees host-side caches (TMA descriptors, and the device address of
 * latent_append_noalloc's scratch).  Safe to call at any time when no call is
 * in progress on another thread. */
MLRA_API void mlra_shutdown(void);

/* ABI version: 1. */
MLRA_API int mlra_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLRA_H_ */
