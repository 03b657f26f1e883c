// libmlra C ABI: argument validation, workspace layout, split planning and
// kernel launches.  See include/mlra.h for the contract of every entry point.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "fp8_cache.h"
#include "../../include/mlra.h"
#include "attn_tc.h"
#include "gemm_tc.h"
#include "host_cache.h"
#include "append_forms.h"
#include "launch.h"

using namespace mlra;

namespace {

thread_local std::string g_err;

mlra_status fail(mlra_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
mlra_status fail(mlra_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

mlra_status cuda_fail(cudaError_t e, const char* where) {
  return fail(MLRA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr size_t kErrBytes = 256;

// ---------------------------------------------------------------------------
// dims validation shared by every entry point
// ---------------------------------------------------------------------------
mlra_status check_dims(const mlra_dims* d) {
  if (!d) return fail(MLRA_ERR_INVALID_ARG, "dims is NULL");
  if (d->B < 1 || d->H < 1 || d->d_h < 1 || d->d_v < 1 || d->d_c < 1 || d->d_r < 2)
    return fail(MLRA_ERR_INVALID_ARG, "B, H, d_h, d_v, d_c must be >= 1 and d_r >= 2");
  if (d->d_r % 2) return fail(MLRA_ERR_INVALID_ARG, "d_r=%d must be even (RoPE pairs)", d->d_r);
  if (d->n_branch < 1) return fail(MLRA_ERR_INVALID_ARG, "n_branch must be >= 1");
  if (d->d_c % d->n_branch) return fail(MLRA_ERR_INVALID_ARG, "d_c=%d not divisible by n_branch=%d", d->d_c, d->n_branch);
  if (d->dtype != MLRA_F32 && d->dtype != MLRA_BF16) return fail(MLRA_ERR_INVALID_ARG, "dtype %d unknown", d->dtype);
  if (d->max_pages_per_seq < 1 || d->num_pages < 1)
    return fail(MLRA_ERR_INVALID_ARG, "max_pages_per_seq and num_pages must be >= 1");
  if (d->num_splits < 0) return fail(MLRA_ERR_INVALID_ARG, "num_splits must be >= 0");
  if (d->kernel < MLRA_KERNEL_AUTO || d->kernel > MLRA_KERNEL_TC)
    return fail(MLRA_ERR_INVALID_ARG, "kernel %d unknown", d->kernel);
  if (!(d->softmax_scale >= 0.f) || !std::isfinite(d->softmax_scale))
    return fail(MLRA_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0 (0 = default)");
  if (!std::isfinite(d->branch_scale)) return fail(MLRA_ERR_INVALID_ARG, "branch_scale must be finite");
  if (!(d->rope_base >= 0.f) || !std::isfinite(d->rope_base))
    return fail(MLRA_ERR_INVALID_ARG, "rope_base must be finite and >= 0 (0 = 10000)");
  // implemented range
  if (d->page_size != kPage) return fail(MLRA_ERR_UNSUPPORTED, "page_size=%d: only 64 is implemented", d->page_size);
  if (d->d_c % 32 || d->d_c > 512) return fail(MLRA_ERR_UNSUPPORTED, "d_c=%d: need a multiple of 32, <= 512", d->d_c);
  if (d->d_r > 64) return fail(MLRA_ERR_UNSUPPORTED, "d_r=%d: need <= 64", d->d_r);
  if ((d->d_c / d->n_branch) % 32 || d->n_branch > 8)
    return fail(MLRA_ERR_UNSUPPORTED, "branch width d_c/n_branch=%d must be a multiple of 32, n_branch <= 8",
                d->d_c / d->n_branch);
  if (d->d_h > 512) return fail(MLRA_ERR_UNSUPPORTED, "d_h=%d: need <= 512", d->d_h);
  if (d->d_v > 65535 * 128) return fail(MLRA_ERR_UNSUPPORTED, "d_v too large");
  if ((long long)d->max_pages_per_seq * kPage > (1LL << 30))
    return fail(MLRA_ERR_UNSUPPORTED, "max_pages_per_seq too large");
  return MLRA_OK;
}

float scale_of(const mlra_dims* d) {
  return d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / std::sqrt((float)(d->d_h + d->d_r));
}

RopeTable rope_table(const mlra_dims* d) {
  RopeTable t;
  const double base = d->rope_base > 0.f ? (double)d->rope_base : 10000.0;
  for (int i = 0; i < kMaxRopePairs; ++i) t.theta[i] = (2 * i < d->d_r) ? std::pow(base, -2.0 * i / d->d_r) : 0.0;
  return t;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

// ---------------------------------------------------------------------------
// decode plan: kernel family, workers and workspace layout
// ---------------------------------------------------------------------------
struct DecodePlan {
  bool tc;
  int G;          // split-KV workers
  int Hq;         // query rows per sequence in the q workspace
  size_t q_off, opart_off, ml_off, olat_off, total;
};

mlra_status make_plan(const mlra_dims* d, DecodePlan* p) {
  mlra_status st = check_dims(d);
  if (st != MLRA_OK) return st;
  const bool tc_ok = tc_supported(d->dtype, d->H, d->d_c, d->d_r, d->n_branch, d->d_h, d->d_v);
  if (d->kernel == MLRA_KERNEL_TC && !tc_ok)
    return fail(MLRA_ERR_UNSUPPORTED, "tcgen05 kernels need bf16, d_c=512, d_r=64, H<=128, n_branch in {1,2,4}");
  p->tc = (d->kernel == MLRA_KERNEL_TC) || (d->kernel == MLRA_KERNEL_AUTO && tc_ok);
  int G = d->num_splits;
  if (G == 0) {
    const int sms = device_sms();
    if (sms <= 0) return fail(MLRA_ERR_CUDA, "num_splits=0 needs a CUDA device to size the split");
    // tcgen05: a CTA pair per page range, or (128-dim branches) one CTA per branch and page range
    G = !p->tc ? sms
               : (tc_branch_supported(d->H, d->d_c, d->d_r, d->n_branch) ? tc_branch_workers(sms, d->n_branch)
                                                                          : sms / 2);
  }
  p->G = G;
  p->Hq = d->H;
  const size_t qe = p->tc ? 2 : 4;
  const size_t slots = (size_t)G + d->B - 1;
  size_t off = kErrBytes;
  p->q_off = off;
  off = round_up(off + (size_t)d->B * p->Hq * (d->d_c + d->d_r) * qe, 256);
  p->opart_off = off;
  off = round_up(off + slots * d->H * d->d_c * 4, 256);
  p->ml_off = off;
  off = round_up(off + slots * d->n_branch * 2 * d->H * 4, 256);
  p->olat_off = off;
  off = round_up(off + (size_t)d->B * d->H * d->d_c * qe, 256);
  p->total = off;
  return MLRA_OK;
}

// The rank's partial of a sequence-sharded decode, written instead of `out`
// when decode_impl is called with one: o [B,H,d_c] fp32, lse [B,n_branch,H].
struct PartialOut {
  float* o;
  float* lse;
};

// An FP8 cache: E4M3 codes in latent_cache/rope_cache, one fp32 scale per page
// of each.  Its decode runs on the CUDA-core kernels.
struct Fp8Scales {
  const float* lat;
  const float* rop;
};

mlra_status decode_impl(const mlra_dims* d, bool mla_only, const void* q_nope, const void* q_rope,
                        const int32_t* q_pos, const void* W_UK, const void* W_UV, const void* latent_cache,
                        const void* rope_cache, const int32_t* page_table, const int32_t* seq_lens, void* out,
                        void* workspace, size_t ws_bytes, cudaStream_t stream, cudaEvent_t* ev,
                        const PartialOut* part = nullptr, const Fp8Scales* fp8 = nullptr) {
  DecodePlan p;
  mlra_dims dsimt;
  if (fp8) {  // the FP8 cache is read by the CUDA-core attention kernel
    if (!fp8->lat || !fp8->rop) return fail(MLRA_ERR_INVALID_ARG, "FP8 scales are NULL");
    if (!aligned(fp8->lat, 4) || !aligned(fp8->rop, 4)) return fail(MLRA_ERR_INVALID_ARG, "FP8 scales not 4-byte aligned");
    if (d->kernel == MLRA_KERNEL_TC) return fail(MLRA_ERR_UNSUPPORTED, "the FP8 cache runs on the CUDA-core kernels");
    dsimt = *d;
    dsimt.kernel = MLRA_KERNEL_SIMT;
    d = &dsimt;
  }
  mlra_status st = make_plan(d, &p);
  if (st != MLRA_OK) return st;
  if (mla_only && d->n_branch != 1) return fail(MLRA_ERR_INVALID_ARG, "mla_decode needs n_branch=1 (use mlra_decode)");
  const void* ptrs[] = {q_nope, q_rope, W_UK, part ? part->o : W_UV, latent_cache, rope_cache,
                        part ? part->lse : out, workspace};
  const char* names[] = {"q_nope", "q_rope", "W_UK", part ? "o" : "W_UV", "latent_cache", "rope_cache",
                         part ? "lse" : "out", "workspace"};
  for (int i = 0; i < 8; ++i) {
    if (!ptrs[i]) return fail(MLRA_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned(ptrs[i], 16)) return fail(MLRA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  if (!q_pos || !page_table || !seq_lens) return fail(MLRA_ERR_INVALID_ARG, "q_pos/page_table/seq_lens is NULL");
  if (!aligned(q_pos, 4) || !aligned(page_table, 4) || !aligned(seq_lens, 4))
    return fail(MLRA_ERR_INVALID_ARG, "index arrays must be 4-byte aligned");
  if (!aligned(workspace, 256)) return fail(MLRA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (ws_bytes < p.total)
    return fail(MLRA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, p.total);

  char* ws = static_cast<char*>(workspace);
  int* err = reinterpret_cast<int*>(ws);
  void* q_ws = ws + p.q_off;
  float* o_part = reinterpret_cast<float*>(ws + p.opart_off);
  float* ml_part = reinterpret_cast<float*>(ws + p.ml_off);
  void* o_lat = ws + p.olat_off;
  const float branch_scale = mla_only ? 1.0f : d->branch_scale;
  const RopeTable tab = rope_table(d);
  cudaError_t e;

  const bool tc_absorb = p.tc && absorb_tc_supported(d->dtype, d->B, d->d_h, d->d_c);
  const bool tc_upproj = p.tc && upproj_tc_supported(d->dtype, d->B, d->d_c, d->d_v, p.G, d->n_branch);
  // The tcgen05 attention kernel takes queries pre-multiplied by scale*log2(e)
  // (its scores are then base-2 logits directly); the CUDA-core kernel scales itself.
  const float scale_log2 = scale_of(d) * 1.4426950408889634f;
  const float q_scale = p.tc ? scale_log2 : 1.0f;
  GemmArgs ga{d->B, batch_pad(d->B), d->H, d->d_h, d->d_c, d->d_r, d->d_v, p.G, d->n_branch,
              d->max_pages_per_seq, branch_scale, q_scale};

  if (ev) record_event(ev[0], stream);
  if (tc_absorb) {
    e = launch_absorb_tc(q_nope, q_rope, q_pos, W_UK, q_ws, err, ga, tab, stream);
  } else {
    AbsorbArgs aa{d->B, d->H, p.Hq, d->d_h, d->d_c, d->d_r, q_scale};
    e = launch_absorb(d->dtype, p.tc, q_nope, q_rope, q_pos, W_UK, q_ws, aa, tab, stream);
  }
  if (e != cudaSuccess) return cuda_fail(e, "absorb launch");
  if (ev) record_event(ev[1], stream);

  AttnArgs at{d->B, d->H, d->d_c, d->d_r, d->n_branch, d->max_pages_per_seq, d->num_pages, p.G,
              p.tc ? 1.0f : scale_log2};
  if (p.tc) {
    // Programmatic dependent launches chain absorption -> attention -> combine
    // (not when stage events sit between the kernels).  The absorption kernel
    // itself is an ordinary launch, so every earlier kernel of the stream (the
    // cache append) has completed before any of the three starts.
    e = launch_attend_tc(q_ws, latent_cache, rope_cache, page_table, seq_lens, o_part, ml_part, err, at, stream,
                         tc_absorb && ev == nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "tcgen05 attention launch");
  } else if (fp8) {
    e = launch_attend_simt_fp8(static_cast<const float*>(q_ws), static_cast<const uint8_t*>(latent_cache),
                               static_cast<const uint8_t*>(rope_cache), fp8->lat, fp8->rop, page_table, seq_lens,
                               o_part, ml_part, err, at, stream);
    if (e != cudaSuccess) return cuda_fail(e, "FP8 attention launch");
  } else {
    e = launch_attend_simt(d->dtype, static_cast<const float*>(q_ws), latent_cache, rope_cache, page_table, seq_lens,
                           o_part, ml_part, err, at, stream);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  }
  if (ev) record_event(ev[2], stream);

  if (part) {  // a sequence-sharded rank: its partial instead of the combine and up-projection
    CombineArgs ca{d->B, d->H, d->d_c, d->n_branch, p.G, d->max_pages_per_seq, 1.0f};
    e = launch_partial(o_part, ml_part, seq_lens, part->o, part->lse, ca, stream);
    if (e != cudaSuccess) return cuda_fail(e, "partial launch");
    return MLRA_OK;
  }

  if (tc_upproj) {  // combine fused into the up-projection: stage 3 is empty
    if (ev) record_event(ev[3], stream);
    GemmArgs gu = ga;
    gu.K = d->d_c;
    e = launch_combine_upproj_tc(o_part, ml_part, seq_lens, W_UV, out, err, gu, stream, ev == nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "combine + up-projection launch");
  } else {
    CombineArgs ca{d->B, d->H, d->d_c, d->n_branch, p.G, d->max_pages_per_seq, branch_scale};
    e = launch_combine(p.tc, o_part, ml_part, seq_lens, o_lat, ca, stream);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    if (ev) record_event(ev[3], stream);
    UpArgs ua{d->B, d->H, d->d_c, d->d_v};
    e = launch_upproj(d->dtype, p.tc, o_lat, W_UV, out, ua, stream);
    if (e != cudaSuccess) return cuda_fail(e, "up-projection launch");
  }
  if (ev) record_event(ev[4], stream);
  return MLRA_OK;
}

}  // namespace

extern "C" {

mlra_status mlra_describe_plan(const mlra_dims* dims, char* buf, size_t buf_len) {
  if (!buf || buf_len == 0) return fail(MLRA_ERR_INVALID_ARG, "buf is NULL or empty");
  DecodePlan p;
  mlra_status st = make_plan(dims, &p);
  if (st != MLRA_OK) return st;
  const mlra_dims* d = dims;
  const bool tc_absorb = p.tc && absorb_tc_supported(d->dtype, d->B, d->d_h, d->d_c);
  const bool tc_upproj = p.tc && upproj_tc_supported(d->dtype, d->B, d->d_c, d->d_v, p.G, d->n_branch);
  const char* family = !p.tc ? "cuda-core" : (tc_absorb && tc_upproj ? "tcgen05" : "tcgen05+cuda-core");
  const int n = snprintf(buf, buf_len,
                         "family=%s;splits=%d;kernels=%d;absorb=%s;attention=%s;combine=%s;upproj=%s", family, p.G,
                         2 + (tc_upproj ? 1 : 2), tc_absorb ? "absorb_tc_kernel" : "absorb_kernel",
                         p.tc ? tc_variant_name(d->H, d->d_c, d->n_branch) : "attend_simt_kernel",
                         tc_upproj ? "fused into combine_upproj_tc_kernel" : "combine_kernel",
                         tc_upproj ? "combine_upproj_tc_kernel" : "upproj_kernel");
  if (n < 0 || (size_t)n >= buf_len) return fail(MLRA_ERR_INVALID_ARG, "buf too small (%d bytes needed)", n + 1);
  return MLRA_OK;
}

size_t mlra_workspace_bytes(const mlra_dims* dims) {
  DecodePlan p;
  if (make_plan(dims, &p) != MLRA_OK) return 0;
  return p.total;
}

mlra_status mla_decode(const mlra_dims* dims, const void* q_nope, const void* q_rope, const int32_t* q_pos,
                       const void* W_UK, const void* W_UV, const void* latent_cache, const void* rope_cache,
                       const int32_t* page_table, const int32_t* seq_lens, void* out, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
  return decode_impl(dims, true, q_nope, q_rope, q_pos, W_UK, W_UV, latent_cache, rope_cache, page_table, seq_lens,
                     out, workspace, workspace_bytes, stream, nullptr);
}

mlra_status mlra_decode(const mlra_dims* dims, const void* q_nope, const void* q_rope, const int32_t* q_pos,
                        const void* W_UK, const void* W_UV, const void* latent_cache, const void* rope_cache,
                        const int32_t* page_table, const int32_t* seq_lens, void* out, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  return decode_impl(dims, false, q_nope, q_rope, q_pos, W_UK, W_UV, latent_cache, rope_cache, page_table, seq_lens,
                     out, workspace, workspace_bytes, stream, nullptr);
}

mlra_status mlra_quantize_pages_fp8(const mlra_dims* dims, const void* latent_cache, const void* rope_cache,
                                    uint8_t* latent_fp8, uint8_t* rope_fp8, float* latent_scale, float* rope_scale,
                                    cudaStream_t stream) {
  mlra_status st = check_dims(dims);
  if (st != MLRA_OK) return st;
  const void* ptrs[] = {latent_cache, rope_cache, latent_fp8, rope_fp8, latent_scale, rope_scale};
  const char* names[] = {"latent_cache", "rope_cache", "latent_fp8", "rope_fp8", "latent_scale", "rope_scale"};
  for (int i = 0; i < 6; ++i)
    if (!ptrs[i]) return fail(MLRA_ERR_INVALID_ARG, "%s is NULL", names[i]);
  if (!aligned(latent_scale, 4) || !aligned(rope_scale, 4)) return fail(MLRA_ERR_INVALID_ARG, "scales not 4-byte aligned");
  cudaError_t e = launch_quantize_pages(dims->dtype, latent_cache, dims->num_pages, kPage * dims->d_c, latent_fp8,
                                        latent_scale, stream);
  if (e == cudaSuccess)
    e = launch_quantize_pages(dims->dtype, rope_cache, dims->num_pages, kPage * dims->d_r, rope_fp8, rope_scale,
                              stream);
  if (e != cudaSuccess) return cuda_fail(e, "FP8 quantizer launch");
  return MLRA_OK;
}

mlra_status mlra_decode_fp8(const mlra_dims* dims, const void* q_nope, const void* q_rope, const int32_t* q_pos,
                            const void* W_UK, const void* W_UV, const uint8_t* latent_fp8, const uint8_t* rope_fp8,
                            const float* latent_scale, const float* rope_scale, const int32_t* page_table,
                            const int32_t* seq_lens, void* out, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
  const Fp8Scales sc{latent_scale, rope_scale};
  return decode_impl(dims, false, q_nope, q_rope, q_pos, W_UK, W_UV, latent_fp8, rope_fp8, page_table, seq_lens, out,
                     workspace, workspace_bytes, stream, nullptr, nullptr, &sc);
}

mlra_status mlra_decode_profiled(const mlra_dims* dims, const void* q_nope, const void* q_rope, const int32_t* q_pos,
                                 const void* W_UK, const void* W_UV, const void* latent_cache, const void* rope_cache,
                                 const int32_t* page_table, const int32_t* seq_lens, void* out, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream, cudaEvent_t* stage_events) {
  return decode_impl(dims, false, q_nope, q_rope, q_pos, W_UK, W_UV, latent_cache, rope_cache, page_table, seq_lens,
                     out, workspace, workspace_bytes, stream, stage_events);
}

// Device staging space for mlra_decode_host, after the decode workspace:
// q_nope | q_rope | q_pos | seq_lens | out, each 256-byte aligned.
struct HostStaging {
  size_t q_nope, q_rope, q_pos, seq_lens, out, total;
};

static bool host_staging(const mlra_dims* d, const DecodePlan& p, HostStaging* h) {
  const size_t e = d->dtype == MLRA_BF16 ? 2 : 4;
  size_t off = round_up(p.total, 256);
  h->q_nope = off;
  off = round_up(off + (size_t)d->B * d->H * d->d_h * e, 256);
  h->q_rope = off;
  off = round_up(off + (size_t)d->B * d->H * d->d_r * e, 256);
  h->q_pos = off;
  off = round_up(off + (size_t)d->B * 4, 256);
  h->seq_lens = off;
  off = round_up(off + (size_t)d->B * 4, 256);
  h->out = off;
  off = round_up(off + (size_t)d->B * d->H * d->d_v * e, 256);
  h->total = off;
  return true;
}

size_t mlra_decode_host_workspace_bytes(const mlra_dims* dims) {
  DecodePlan p;
  if (make_plan(dims, &p) != MLRA_OK) return 0;
  HostStaging h;
  host_staging(dims, p, &h);
  return h.total;
}

mlra_status mlra_decode_host(const mlra_dims* dims, const void* h_q_nope, const void* h_q_rope,
                             const int32_t* h_q_pos, const void* W_UK, const void* W_UV, const void* latent_cache,
                             const void* rope_cache, const int32_t* page_table, const int32_t* h_seq_lens,
                             void* h_out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  DecodePlan p;
  mlra_status st = make_plan(dims, &p);
  if (st != MLRA_OK) return st;
  if (!h_q_nope || !h_q_rope || !h_q_pos || !h_seq_lens || !h_out)
    return fail(MLRA_ERR_INVALID_ARG, "a host buffer is NULL");
  if (!workspace || !aligned(workspace, 256)) return fail(MLRA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  HostStaging h;
  host_staging(dims, p, &h);
  if (workspace_bytes < h.total)
    return fail(MLRA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, h.total);
  const mlra_dims* d = dims;
  const size_t e = d->dtype == MLRA_BF16 ? 2 : 4;
  char* ws = static_cast<char*>(workspace);
  struct Copy {
    void* dst;
    const void* src;
    size_t n;
  } in[] = {{ws + h.q_nope, h_q_nope, (size_t)d->B * d->H * d->d_h * e},
            {ws + h.q_rope, h_q_rope, (size_t)d->B * d->H * d->d_r * e},
            {ws + h.q_pos, h_q_pos, (size_t)d->B * 4},
            {ws + h.seq_lens, h_seq_lens, (size_t)d->B * 4}};
  for (const Copy& c : in) {
    cudaError_t e2 = cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, stream);
    if (e2 != cudaSuccess) return cuda_fail(e2, "host-to-device copy");
  }
  st = decode_impl(d, false, ws + h.q_nope, ws + h.q_rope, reinterpret_cast<const int32_t*>(ws + h.q_pos), W_UK,
                   W_UV, latent_cache, rope_cache, page_table, reinterpret_cast<const int32_t*>(ws + h.seq_lens),
                   ws + h.out, workspace, workspace_bytes, stream, nullptr);
  if (st != MLRA_OK) return st;
  cudaError_t e3 = cudaMemcpyAsync(h_out, ws + h.out, (size_t)d->B * d->H * d->d_v * e, cudaMemcpyDeviceToHost,
                                   stream);
  if (e3 != cudaSuccess) return cuda_fail(e3, "device-to-host copy");
  return MLRA_OK;
}

mlra_status mlra_attend_partial(const mlra_dims* dims, const void* q_nope, const void* q_rope, const int32_t* q_pos,
                                const void* W_UK, const void* latent_cache, const void* rope_cache,
                                const int32_t* page_table, const int32_t* seq_lens, float* o, float* lse,
                                void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  const PartialOut part{o, lse};
  return decode_impl(dims, false, q_nope, q_rope, q_pos, W_UK, nullptr, latent_cache, rope_cache, page_table,
                     seq_lens, nullptr, workspace, workspace_bytes, stream, nullptr, &part);
}

size_t mlra_merge_workspace_bytes(const mlra_dims* dims) {
  if (check_dims(dims) != MLRA_OK) return 0;
  return round_up((size_t)dims->B * dims->H * dims->d_c * (dims->dtype == MLRA_BF16 ? 2 : 4), 256);
}

mlra_status mlra_merge_upproj(const mlra_dims* dims, int n_parts, const float* o_parts, const float* lse_parts,
                              const void* W_UV, void* out, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  mlra_status st = check_dims(dims);
  if (st != MLRA_OK) return st;
  const mlra_dims* d = dims;
  if (n_parts < 1) return fail(MLRA_ERR_INVALID_ARG, "n_parts must be >= 1");
  const void* ptrs[] = {o_parts, lse_parts, W_UV, out, workspace};
  const char* names[] = {"o_parts", "lse_parts", "W_UV", "out", "workspace"};
  for (int i = 0; i < 5; ++i) {
    if (!ptrs[i]) return fail(MLRA_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned(ptrs[i], 16)) return fail(MLRA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  const size_t need = mlra_merge_workspace_bytes(d);
  if (workspace_bytes < need) return fail(MLRA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  const bool bf16 = d->dtype == MLRA_BF16;
  cudaError_t e = launch_merge(bf16, o_parts, lse_parts, workspace, n_parts, d->B, d->H, d->d_c, d->n_branch,
                               d->branch_scale, stream);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  UpArgs ua{d->B, d->H, d->d_c, d->d_v};
  e = launch_upproj(d->dtype, bf16, workspace, W_UV, out, ua, stream);
  if (e != cudaSuccess) return cuda_fail(e, "up-projection launch");
  return MLRA_OK;
}

size_t latent_append_workspace_bytes(const mlra_dims* dims, int d_model) {
  if (check_dims(dims) != MLRA_OK) return 0;
  if (d_model < 1) {
    fail(MLRA_ERR_INVALID_ARG, "d_model must be >= 1");
    return 0;
  }
  if (!append_uses_scratch(dims->dtype, d_model, dims->d_c, dims->d_r)) return kErrBytes;  // the error record only
  const int KS = (d_model + 63) / 64;
  return kErrBytes + round_up((size_t)KS * dims->B * (dims->d_c + dims->d_r) * 4, 256);
}

mlra_status latent_append(const mlra_dims* dims, int d_model, const void* h, const void* W_DKV, const void* W_KR,
                          const int32_t* pos, const int32_t* page_table, void* latent_cache, void* rope_cache,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  mlra_status st = check_dims(dims);
  if (st != MLRA_OK) return st;
  if (d_model < 1) return fail(MLRA_ERR_INVALID_ARG, "d_model must be >= 1");
  const void* ptrs[] = {h, W_DKV, W_KR, latent_cache, rope_cache, workspace};
  const char* names[] = {"h", "W_DKV", "W_KR", "latent_cache", "rope_cache", "workspace"};
  for (int i = 0; i < 6; ++i) {
    if (!ptrs[i]) return fail(MLRA_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned(ptrs[i], 16)) return fail(MLRA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  if (!pos || !page_table) return fail(MLRA_ERR_INVALID_ARG, "pos/page_table is NULL");
  if (!aligned(workspace, 256)) return fail(MLRA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t need = latent_append_workspace_bytes(dims, d_model);
  if (workspace_bytes < need) return fail(MLRA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  char* ws = static_cast<char*>(workspace);
  AppendArgs a{dims->B, d_model, dims->d_c, dims->d_r, dims->max_pages_per_seq, dims->num_pages, (d_model + 63) / 64};
  cudaError_t e = launch_append(dims->dtype, h, W_DKV, W_KR, pos, page_table, latent_cache, rope_cache,
                                reinterpret_cast<float*>(ws + kErrBytes), reinterpret_cast<int*>(ws), a,
                                rope_table(dims), stream);
  if (e != cudaSuccess) return cuda_fail(e, "latent_append launch");
  return MLRA_OK;
}

mlra_status latent_store(const mlra_dims* dims, int n_tokens, const void* c_kv, const void* k_rope,
                         const int32_t* tok_seq, const int32_t* tok_pos, const int32_t* page_table, void* latent_cache,
                         void* rope_cache, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  mlra_status st = check_dims(dims);
  if (st != MLRA_OK) return st;
  if (n_tokens < 0) return fail(MLRA_ERR_INVALID_ARG, "n_tokens must be >= 0");
  const void* ptrs[] = {c_kv, k_rope, latent_cache, rope_cache, workspace};
  const char* names[] = {"c_kv", "k_rope", "latent_cache", "rope_cache", "workspace"};
  for (int i = 0; i < 5; ++i) {
    if (!ptrs[i]) return fail(MLRA_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned(ptrs[i], 16)) return fail(MLRA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  if (!tok_seq || !tok_pos || !page_table) return fail(MLRA_ERR_INVALID_ARG, "tok_seq/tok_pos/page_table is NULL");
  if (workspace_bytes < kErrBytes) return fail(MLRA_ERR_WORKSPACE, "workspace needs %zu bytes", kErrBytes);
  StoreArgs a{n_tokens, dims->B, dims->d_c, dims->d_r, dims->max_pages_per_seq, dims->num_pages};
  cudaError_t e = launch_store(dims->dtype, c_kv, k_rope, tok_seq, tok_pos, page_table, latent_cache, rope_cache,
                               static_cast<int*>(workspace), a, rope_table(dims), stream);
  if (e != cudaSuccess) return cuda_fail(e, "latent_store launch");
  return MLRA_OK;
}

mlra_status mlra_check_status(void* workspace, cudaStream_t stream) {
  if (!workspace) return fail(MLRA_ERR_INVALID_ARG, "workspace is NULL");
  int rec[4] = {0, 0, 0, 0};
  cudaError_t e = cudaMemcpyAsync(rec, workspace, sizeof(rec), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error record");
  if (rec[0] == 0) return MLRA_OK;
  e = cudaMemsetAsync(workspace, 0, 16, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device error record");
  if (rec[0] == kErrTimeout)
    return fail(MLRA_ERR_TIMEOUT, "a device wait gave up (site %d, detail %d)", rec[1], rec[2]);
  return fail(MLRA_ERR_DEVICE_CHECK, "device range check: item %d, position/detail %d", rec[1], rec[2]);
}

const char* mlra_last_error(void) { return g_err.c_str(); }

void mlra_shutdown(void) {
  tc_shutdown();
  noalloc_forget_scratch();
}

int mlra_version(void) { return 1; }

}  // extern "C"

// Internal helpers for entry points defined in other translation units.
namespace mlra {
mlra_status internal_check_dims(const mlra_dims* d) { return check_dims(d); }
mlra_status internal_fail(mlra_status st, const char* msg) { return fail(st, "%s", msg); }
RopeTable internal_rope_table(const mlra_dims* d) { return rope_table(d); }
}  // namespace mlra
