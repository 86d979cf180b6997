// dd_abi.cu -- the extern "C" boundary of libdd (declared in include/dd.h):
// argument validation (always before any launch), launch planning, workspace
// carving, error reporting and the block loop.  All device work happens in
// the kernels of dd_sampler.cu, dd_attn_tc.cu and dd_attn_simt.cu.
#include <cmath>
#include <utility>
#include <vector>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "dd.h"
#include "dd_internal.h"

namespace dd {

namespace {
thread_local std::string g_last_error;
thread_local uint64_t g_launches = 0;

constexpr size_t kHeaderBytes = 256;  // device error word + padding

dd_status fail(dd_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
dd_status fail(dd_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

dd_status cuda_fail(cudaError_t e, const char* what) {
  return fail(DD_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(dd_dtype t) { return t == DD_BF16 ? 2 : t == DD_E4M3 ? 1 : 4; }

// Validates the geometry and the host prefix offsets; fills total prefix.
// DD_E4M3 is accepted only where the caller can take it (allow_e4m3).
dd_status check_attn_desc(const dd_attn_desc* d, const int32_t* cu_host, int64_t* total,
                          bool allow_e4m3 = false) {
  if (!d) return fail(DD_ERR_INVALID_ARG, "desc is NULL");
  if (d->batch < 0 || d->canvas < 1 || d->heads_q < 1 || d->heads_kv < 1)
    return fail(DD_ERR_INVALID_ARG, "bad geometry B=%d C=%d Hq=%d Hkv=%d", d->batch, d->canvas,
                d->heads_q, d->heads_kv);
  if (d->heads_q % d->heads_kv != 0)
    return fail(DD_ERR_INVALID_ARG, "heads_q (%d) is not a multiple of heads_kv (%d)",
                d->heads_q, d->heads_kv);
  if (d->dtype == DD_E4M3 && !allow_e4m3)
    return fail(DD_ERR_INVALID_ARG,
                "DD_E4M3 inputs need per-tensor factors: use dd_canvas_attn_fp8");
  if (d->dtype != DD_BF16 && d->dtype != DD_F32 && d->dtype != DD_E4M3)
    return fail(DD_ERR_INVALID_ARG, "unknown dtype %d", (int)d->dtype);
  if (d->head_dim != 64 && d->head_dim != 128)
    return fail(DD_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", d->head_dim);
  if (!std::isfinite(d->scale) || d->scale <= 0.f)
    return fail(DD_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (d->batch > 0 && !cu_host) return fail(DD_ERR_INVALID_ARG, "cu_prefix_host is NULL");
  if ((int64_t)d->batch * d->canvas > INT32_MAX)
    return fail(DD_ERR_UNSUPPORTED, "batch * canvas exceeds 2^31");
  int64_t tot = 0;
  if (d->batch > 0) {
    if (cu_host[0] != 0) return fail(DD_ERR_INVALID_ARG, "cu_prefix[0] must be 0");
    for (int b = 0; b < d->batch; ++b)
      if (cu_host[b + 1] < cu_host[b])
        return fail(DD_ERR_INVALID_ARG, "cu_prefix decreases at %d", b);
    tot = cu_host[d->batch];
  }
  *total = tot;
  return DD_OK;
}

AttnArgs make_attn_args(const dd_attn_desc* d, int64_t total, const int32_t* cu_host) {
  AttnArgs a{};
  a.cu_prefix_host = cu_host;
  a.B = d->batch;
  a.C = d->canvas;
  a.Hq = d->heads_q;
  a.Hkv = d->heads_kv;
  a.D = d->head_dim;
  a.scale = d->scale;
  a.bf16 = d->dtype == DD_BF16;
  a.e4m3 = d->dtype == DD_E4M3;
  a.q_scale = a.k_scale = a.v_scale = 1.0f;
  a.total_prefix = total;
  return a;
}

size_t attn_ws_bytes(const AttnArgs& a) {
  // pointers are unknown at query time: plan for the tensor-core path when
  // the geometry allows it (its scratch is the larger of the two)
  AttnArgs t = a;
  const void* fake = reinterpret_cast<const void*>(static_cast<uintptr_t>(256));
  t.q = t.kc = t.vc = t.kp = t.vp = fake;
  if (a.B > 0 && attn_tc_supported(t)) return kHeaderBytes + attn_tc_scratch_bytes(t);
  return kHeaderBytes + attn_simt_scratch_bytes(t);
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Sampler workspace: header, then the persistent state (ticket counter and
// row keys, kept zero between calls), then the per-chunk records.
size_t sample_ws_bytes(int rows, int vocab, dd_dtype dtype) {
  (void)dtype;
  return kHeaderBytes + align256(sampler_state_bytes(rows)) + sampler_record_bytes(rows, vocab);
}

// Block-loop workspace: the attention scratch and the sampler records share
// one region (they run one after the other on the stream); the sampler's
// persistent state and a confidence buffer (used when the caller passes no
// conf_steps) follow it.
size_t block_ws_layout(const dd_attn_desc* desc, int64_t total, const int32_t* cu_prefix_host,
                       int vocab, size_t* state_off, size_t* conf_off) {
  const int rows = desc->batch * desc->canvas;
  const size_t a = attn_ws_bytes(make_attn_args(desc, total, cu_prefix_host));
  const size_t s = kHeaderBytes + sampler_record_bytes(rows, vocab);
  const size_t shared = align256(a > s ? a : s);
  const size_t cf = shared + align256(sampler_state_bytes(rows));
  if (state_off) *state_off = shared;
  if (conf_off) *conf_off = cf;
  return cf + align256((size_t)rows * sizeof(float));
}

// `f8` (NULL unless d->dtype is DD_E4M3): the per-tensor factors.
dd_status run_attn(const dd_attn_desc* d, const void* q, const void* kc, const void* vc,
                   const void* kp, const void* vp, const int32_t* cu, const int32_t* cu_host,
                   void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream,
                   const dd_fp8_scales* f8 = nullptr) {
  int64_t total = 0;
  dd_status st = check_attn_desc(d, cu_host, &total, f8 != nullptr);
  if (st != DD_OK) return st;
  if (d->batch == 0) return DD_OK;
  if (!q || !kc || !vc || !out || !cu) return fail(DD_ERR_INVALID_ARG, "NULL tensor pointer");
  if (total > 0 && (!kp || !vp)) return fail(DD_ERR_INVALID_ARG, "NULL prefix pointer");
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(out) ||
      (total > 0 && (!aligned16(kp) || !aligned16(vp))))
    return fail(DD_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(DD_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  AttnArgs a = make_attn_args(d, total, cu_host);
  if (a.e4m3) {
    a.q_scale = f8->q;
    a.k_scale = f8->k;
    a.v_scale = f8->v;
  }
  a.q = q;
  a.kc = kc;
  a.vc = vc;
  a.kp = total > 0 ? kp : kc;
  a.vp = total > 0 ? vp : vc;
  a.cu_prefix = cu;
  a.cu_prefix_host = cu_host;
  a.out = out;
  a.lse = lse;
  a.err = static_cast<uint32_t*>(ws);
  a.scratch = static_cast<uint8_t*>(ws) + kHeaderBytes;
  const bool tc = attn_tc_supported(a);
  if (a.e4m3 && !tc)
    return fail(DD_ERR_UNSUPPORTED,
                "E4M3 attention needs head_dim 128 and (heads_q / heads_kv) dividing 128");
  const size_t need = kHeaderBytes + (tc ? attn_tc_scratch_bytes(a) : attn_simt_scratch_bytes(a));
  if (ws_bytes < need)
    return fail(DD_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  a.scratch_bytes = ws_bytes - kHeaderBytes;
  cudaError_t e = tc ? launch_attn_tc(a, stream) : launch_attn_simt(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, tc ? "canvas attention (tcgen05)" : "canvas attention");
  return DD_OK;
}

// `state` is the sampler's persistent state, or nullptr for the standalone
// layout (state after the header, records after the state).
}  // namespace

// The argument checks of a sampler call that need neither a device nor a
// workspace; a call with rows == 0 passes them and then does nothing.
dd_status check_sampler_call(const void* logits, dd_dtype dtype, int rows, int vocab,
                             int64_t row_stride, const dd_sample_params* p,
                             const int32_t* tokens, const float* conf) {
  if (!p) return fail(DD_ERR_INVALID_ARG, "params is NULL");
  if (dtype != DD_BF16 && dtype != DD_F32)
    return fail(DD_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (rows < 0 || vocab < 1) return fail(DD_ERR_INVALID_ARG, "rows=%d vocab=%d", rows, vocab);
  if (row_stride < vocab)
    return fail(DD_ERR_INVALID_ARG, "row_stride (%lld) < vocab (%d)", (long long)row_stride,
                vocab);
  if (!std::isfinite(p->temperature) || p->temperature < 1e-3f)
    return fail(DD_ERR_INVALID_ARG, "temperature must be finite and >= 1e-3");
  if (!(p->renoise_rate >= 0.f && p->renoise_rate <= 1.f))
    return fail(DD_ERR_INVALID_ARG, "renoise_rate must lie in [0, 1]");
  if ((uint64_t)rows + p->row_offset > (1ull << 32))
    return fail(DD_ERR_INVALID_ARG, "row_offset + rows exceeds 2^32");
  if (rows > 0 && (!logits || !tokens || !conf))
    return fail(DD_ERR_INVALID_ARG, "NULL required pointer");
  return DD_OK;
}

namespace {

dd_status run_sampler(const void* logits, dd_dtype dtype, int rows, int vocab, int64_t row_stride,
                      const dd_sample_params* p, int32_t* tokens, int32_t* pred, float* conf,
                      float* entropy, uint8_t* renoised, void* ws, size_t ws_bytes,
                      cudaStream_t stream, void* state = nullptr) {
  dd_status st = check_sampler_call(logits, dtype, rows, vocab, row_stride, p, tokens, conf);
  if (st != DD_OK) return st;
  if (rows == 0) return DD_OK;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(DD_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const size_t need = state ? kHeaderBytes + sampler_record_bytes(rows, vocab)
                            : sample_ws_bytes(rows, vocab, dtype);
  if (ws_bytes < need)
    return fail(DD_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  if ((uint64_t)rows * (uint64_t)((vocab + 2047) / 2048) > 0xffffffffull)
    return fail(DD_ERR_UNSUPPORTED, "rows * chunks exceeds 2^32");
  uint8_t* const body = static_cast<uint8_t*>(ws) + kHeaderBytes;
  SamplerArgs a{};
  a.logits = logits;
  a.bf16 = dtype == DD_BF16;
  a.rows = rows;
  a.vocab = vocab;
  a.row_stride = row_stride;
  a.inv_tau = 1.0f / p->temperature;
  a.rate = p->renoise_rate;
  a.seed = p->seed;
  a.step = p->step;
  a.row_offset = p->row_offset;
  a.tokens = tokens;
  a.pred = pred;
  a.conf = conf;
  a.entropy = entropy;
  a.renoised = renoised;
  a.state = state ? state : body;
  a.recs = state ? body : body + align256(sampler_state_bytes(rows));
  a.err = static_cast<uint32_t*>(ws);
  cudaError_t e = launch_sampler(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "sampler");
  return DD_OK;
}

}  // namespace

void note_launch() { ++g_launches; }

constexpr uint64_t kDefaultWaitNs = 1000000000ull;
thread_local uint64_t g_stall_ns = 0;  // 0: no test stall
uint64_t pipeline_wait_ns() { return g_stall_ns ? g_stall_ns : kDefaultWaitNs; }
bool pipeline_test_stall() { return g_stall_ns != 0; }

thread_local bool g_pdl_off = false;
bool pdl_enabled() { return !g_pdl_off; }

// Entry for callers that bring their own scratch region (dd_noalloc.cu):
// the same validation and kernels as dd_sample_renoise.  After the checks,
// and before the kernels, the part of the scratch the call reads before
// writing (the error word, the work counter and this call's row maxima) is
// cleared on the stream, so a call that failed on the device earlier, and
// left that state dirty, cannot affect this one.
dd_status sample_with_scratch(const void* logits, dd_dtype dtype, int rows, int vocab,
                              int64_t row_stride, const dd_sample_params* p, int32_t* tokens,
                              int32_t* pred, float* conf, float* entropy, uint8_t* renoised,
                              void* scratch, size_t scratch_bytes, cudaStream_t stream) {
  g_last_error.clear();
  dd_status st = check_sampler_call(logits, dtype, rows, vocab, row_stride, p, tokens, conf);
  if (st != DD_OK || rows == 0) return st;
  const size_t clear = kHeaderBytes + align256(sampler_state_bytes(rows));
  if (!scratch || scratch_bytes < clear)
    return fail(DD_ERR_WORKSPACE, "scratch too small: %zu < %zu bytes", scratch_bytes, clear);
  cudaError_t e = cudaMemsetAsync(scratch, 0, clear, stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the sampler state");
  return run_sampler(logits, dtype, rows, vocab, row_stride, p, tokens, pred, conf, entropy,
                     renoised, scratch, scratch_bytes, stream);
}

dd_status set_error(dd_status st, const char* msg) {
  g_last_error = msg;
  return st;
}

}  // namespace dd

using namespace dd;

extern "C" {

size_t dd_canvas_attn_workspace(const dd_attn_desc* desc, const int32_t* cu_prefix_host) {
  int64_t total = 0;
  if (check_attn_desc(desc, cu_prefix_host, &total, true) != DD_OK) return 0;
  return attn_ws_bytes(make_attn_args(desc, total, cu_prefix_host));
}

dd_status dd_canvas_attn(const dd_attn_desc* desc, const void* q, const void* k_canvas,
                         const void* v_canvas, const void* k_prefix, const void* v_prefix,
                         const int32_t* cu_prefix, const int32_t* cu_prefix_host, void* out,
                         float* lse, void* workspace, size_t workspace_bytes, dd_stream_t stream) {
  g_last_error.clear();
  return run_attn(desc, q, k_canvas, v_canvas, k_prefix, v_prefix, cu_prefix, cu_prefix_host, out,
                  lse, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

// The per-tensor factors of one E4M3 attention call (`step` >= 0 names the
// block-loop step in the message).
static dd_status check_fp8_scales(const dd_attn_desc* desc, const dd_fp8_scales* f, int step) {
  char where[32] = "";
  if (step >= 0) snprintf(where, sizeof where, "step %d: ", step);
  if (!(std::isfinite(f->q) && f->q > 0.f && std::isfinite(f->k) && f->k > 0.f &&
        std::isfinite(f->v) && f->v > 0.f))
    return fail(DD_ERR_INVALID_ARG, "%sscale factors must be finite and > 0", where);
  const double logit_gain =
      (double)desc->scale * 1.4426950408889634 * (double)f->q * (double)f->k;
  if (!std::isfinite(logit_gain) || logit_gain > 3.0e38)
    return fail(DD_ERR_INVALID_ARG, "%sscale * q factor * k factor overflows float32", where);
  return DD_OK;
}

dd_status dd_canvas_attn_fp8(const dd_attn_desc* desc, const void* q, const void* k_canvas,
                             const void* v_canvas, const void* k_prefix, const void* v_prefix,
                             const int32_t* cu_prefix, const int32_t* cu_prefix_host,
                             const dd_fp8_scales* scales, void* out, float* lse, void* workspace,
                             size_t workspace_bytes, dd_stream_t stream) {
  g_last_error.clear();
  if (!desc) return fail(DD_ERR_INVALID_ARG, "desc is NULL");
  if (desc->dtype != DD_E4M3)
    return fail(DD_ERR_INVALID_ARG, "dd_canvas_attn_fp8 takes DD_E4M3 inputs");
  if (!scales) return fail(DD_ERR_INVALID_ARG, "scales is NULL");
  dd_status st = check_fp8_scales(desc, scales, -1);
  if (st != DD_OK) return st;
  return run_attn(desc, q, k_canvas, v_canvas, k_prefix, v_prefix, cu_prefix, cu_prefix_host, out,
                  lse, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), scales);
}

size_t dd_sample_renoise_workspace(int rows, int vocab, dd_dtype dtype) {
  if (rows < 0 || vocab < 1 || (dtype != DD_BF16 && dtype != DD_F32)) return 0;
  return sample_ws_bytes(rows, vocab, dtype);
}

dd_status dd_sample_renoise(const void* logits, dd_dtype dtype, int rows, int vocab,
                            int64_t row_stride, const dd_sample_params* params,
                            int32_t* tokens_out, int32_t* pred_out, float* conf_out,
                            float* entropy_out, uint8_t* renoised_out, void* workspace,
                            size_t workspace_bytes, dd_stream_t stream) {
  g_last_error.clear();
  return run_sampler(logits, dtype, rows, vocab, row_stride, params, tokens_out, pred_out,
                     conf_out, entropy_out, renoised_out, workspace, workspace_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

dd_status dd_init_canvas(int32_t* canvas, int rows, int vocab, uint64_t seed, uint32_t row_offset,
                         dd_stream_t stream) {
  g_last_error.clear();
  if (rows < 0 || vocab < 1) return fail(DD_ERR_INVALID_ARG, "rows=%d vocab=%d", rows, vocab);
  if ((uint64_t)rows + row_offset > (1ull << 32))
    return fail(DD_ERR_INVALID_ARG, "row_offset + rows exceeds 2^32");
  if (rows == 0) return DD_OK;
  if (!canvas) return fail(DD_ERR_INVALID_ARG, "canvas is NULL");
  cudaError_t e = launch_init_canvas(canvas, rows, vocab, seed, row_offset,
                                     reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "init canvas");
  return DD_OK;
}

size_t dd_denoise_block_workspace(const dd_attn_desc* desc, const int32_t* cu_prefix_host,
                                  int vocab) {
  int64_t total = 0;
  if (vocab < 1 || check_attn_desc(desc, cu_prefix_host, &total, true) != DD_OK) return 0;
  return block_ws_layout(desc, total, cu_prefix_host, vocab, nullptr, nullptr);
}

// The block loop behind dd_denoise_block and dd_denoise_block_fp8.  With
// E4M3 attention inputs (scales_host: one set of factors per step) the
// attention output is bf16 and the logits are bf16; otherwise both have the
// attention inputs' type.
static dd_status block_loop(const dd_attn_desc* desc, int steps, const void* q_steps,
                            const void* kc_steps, const void* vc_steps, const void* k_prefix,
                            const void* v_prefix, const int32_t* cu_prefix,
                            const int32_t* cu_prefix_host, const dd_fp8_scales* scales_host,
                            void* attn_out, const void* logits_steps, int vocab,
                            const float* rate_host, const float* temperature_host, uint64_t seed,
                            uint32_t step0, int32_t* canvas, int32_t* canvas_history,
                            float* conf_steps, void* workspace, size_t workspace_bytes,
                            dd_stream_t stream) {
  const bool f8 = scales_host != nullptr;
  if (!f8 && desc && desc->dtype == DD_E4M3)
    return fail(DD_ERR_INVALID_ARG,
                "DD_E4M3 inputs need per-step factors: use dd_denoise_block_fp8");
  int64_t total = 0;
  dd_status st = check_attn_desc(desc, cu_prefix_host, &total, f8);
  if (st != DD_OK) return st;
  if (steps < 0) return fail(DD_ERR_INVALID_ARG, "steps < 0");
  if (steps > 0 && (!rate_host || !temperature_host))
    return fail(DD_ERR_INVALID_ARG, "rate_host / temperature_host is NULL");
  if (!canvas) return fail(DD_ERR_INVALID_ARG, "canvas is NULL");
  if ((uint64_t)step0 + (uint64_t)steps > (1ull << 32))
    return fail(DD_ERR_INVALID_ARG, "step0 + steps exceeds 2^32");
  const int B = desc->batch, C = desc->canvas, Hq = desc->heads_q, Hkv = desc->heads_kv;
  const int D = desc->head_dim;
  const int rows = B * C;
  const dd_dtype out_t = f8 ? DD_BF16 : desc->dtype;  // attention output and logits
  const size_t es = elem_size(desc->dtype), os = elem_size(out_t);
  const size_t q_step = (size_t)rows * Hq * D * es;
  const size_t kv_step = (size_t)rows * Hkv * D * es;
  const size_t o_step = (size_t)rows * Hq * D * os;
  const size_t lg_step = (size_t)rows * (size_t)vocab * os;
  if (vocab < 1) return fail(DD_ERR_INVALID_ARG, "vocab=%d", vocab);
  size_t state_off = 0, conf_off = 0;
  const size_t need = block_ws_layout(desc, total, cu_prefix_host, vocab, &state_off, &conf_off);
  if (!workspace) return fail(DD_ERR_WORKSPACE, "workspace is NULL");
  if (workspace_bytes < need)
    return fail(DD_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int i = 0; i < steps; ++i) {
    st = run_attn(desc, static_cast<const uint8_t*>(q_steps) + i * q_step,
                  static_cast<const uint8_t*>(kc_steps) + i * kv_step,
                  static_cast<const uint8_t*>(vc_steps) + i * kv_step, k_prefix, v_prefix,
                  cu_prefix, cu_prefix_host, static_cast<uint8_t*>(attn_out) + i * o_step,
                  nullptr, workspace, state_off, s, f8 ? scales_host + i : nullptr);
    if (st != DD_OK) return st;
    dd_sample_params sp;
    sp.temperature = temperature_host[i];
    sp.renoise_rate = rate_host[i];
    sp.seed = seed;
    sp.step = step0 + (uint32_t)i;
    sp.row_offset = 0;
    int32_t* tok = canvas_history ? canvas_history + (size_t)i * rows : canvas;
    float* conf = conf_steps ? conf_steps + (size_t)i * rows
                             : reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + conf_off);
    st = run_sampler(static_cast<const uint8_t*>(logits_steps) + i * lg_step, out_t, rows, vocab,
                     vocab, &sp, tok, nullptr, conf, nullptr, nullptr, workspace, state_off, s,
                     static_cast<uint8_t*>(workspace) + state_off);
    if (st != DD_OK) return st;
    if (canvas_history && i == steps - 1) {
      cudaError_t e = cudaMemcpyAsync(canvas, tok, (size_t)rows * sizeof(int32_t),
                                      cudaMemcpyDeviceToDevice, s);
      if (e != cudaSuccess) return cuda_fail(e, "canvas copy");
    }
  }
  return DD_OK;
}

dd_status dd_denoise_block(const dd_attn_desc* desc, int steps, const void* q_steps,
                           const void* kc_steps, const void* vc_steps, const void* k_prefix,
                           const void* v_prefix, const int32_t* cu_prefix,
                           const int32_t* cu_prefix_host, void* attn_out,
                           const void* logits_steps, int vocab, const float* rate_host,
                           const float* temperature_host, uint64_t seed, uint32_t step0,
                           int32_t* canvas, int32_t* canvas_history, float* conf_steps,
                           void* workspace, size_t workspace_bytes, dd_stream_t stream) {
  g_last_error.clear();
  return block_loop(desc, steps, q_steps, kc_steps, vc_steps, k_prefix, v_prefix, cu_prefix,
                    cu_prefix_host, nullptr, attn_out, logits_steps, vocab, rate_host,
                    temperature_host, seed, step0, canvas, canvas_history, conf_steps, workspace,
                    workspace_bytes, stream);
}

dd_status dd_denoise_block_fp8(const dd_attn_desc* desc, int steps, const void* q_steps,
                               const void* kc_steps, const void* vc_steps, const void* k_prefix,
                               const void* v_prefix, const int32_t* cu_prefix,
                               const int32_t* cu_prefix_host, const dd_fp8_scales* scales_host,
                               void* attn_out, const void* logits_steps, int vocab,
                               const float* rate_host, const float* temperature_host,
                               uint64_t seed, uint32_t step0, int32_t* canvas,
                               int32_t* canvas_history, float* conf_steps, void* workspace,
                               size_t workspace_bytes, dd_stream_t stream) {
  g_last_error.clear();
  if (!desc) return fail(DD_ERR_INVALID_ARG, "desc is NULL");
  if (desc->dtype != DD_E4M3)
    return fail(DD_ERR_INVALID_ARG, "dd_denoise_block_fp8 takes DD_E4M3 inputs");
  if (steps > 0 && !scales_host) return fail(DD_ERR_INVALID_ARG, "scales_host is NULL");
  for (int i = 0; i < steps; ++i) {
    dd_status st = check_fp8_scales(desc, scales_host + i, i);
    if (st != DD_OK) return st;
  }
  static const dd_fp8_scales kNone = {1.f, 1.f, 1.f};
  return block_loop(desc, steps, q_steps, kc_steps, vc_steps, k_prefix, v_prefix, cu_prefix,
                    cu_prefix_host, steps > 0 ? scales_host : &kNone, attn_out, logits_steps,
                    vocab, rate_host, temperature_host, seed, step0, canvas, canvas_history,
                    conf_steps, workspace, workspace_bytes, stream);
}

dd_status dd_entropy_accept(const float* entropy, const int32_t* pred, int batch, int canvas,
                            int vocab, float budget, uint64_t seed, uint32_t step,
                            uint32_t row_offset, int32_t* tokens_out, uint8_t* accepted_out,
                            dd_stream_t stream) {
  g_last_error.clear();
  if (batch < 0 || canvas < 1 || canvas > 1024 || vocab < 1)
    return fail(DD_ERR_INVALID_ARG, "batch=%d canvas=%d (1..1024) vocab=%d", batch, canvas, vocab);
  if (std::isnan(budget)) return fail(DD_ERR_INVALID_ARG, "budget is NaN");
  if ((uint64_t)batch * (uint64_t)canvas + row_offset > (1ull << 32))
    return fail(DD_ERR_INVALID_ARG, "row_offset + rows exceeds 2^32");
  if (batch == 0) return DD_OK;
  if (!entropy || !pred || !tokens_out) return fail(DD_ERR_INVALID_ARG, "NULL required pointer");
  cudaError_t e = launch_entropy_accept(entropy, pred, batch, canvas, vocab, (double)budget, seed,
                                        step, row_offset, nullptr, nullptr, 0, tokens_out,
                                        accepted_out, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "entropy accept");
  return DD_OK;
}

dd_status dd_stop_check(const float* entropy, const int32_t* pred, const int32_t* pred_prev,
                        int batch, int canvas, float threshold, int32_t step, uint8_t* done,
                        int32_t* halt_step, dd_stream_t stream) {
  g_last_error.clear();
  if (batch < 0 || canvas < 1) return fail(DD_ERR_INVALID_ARG, "batch=%d canvas=%d", batch, canvas);
  if (batch == 0) return DD_OK;
  if (!entropy || !pred || !done || !halt_step)
    return fail(DD_ERR_INVALID_ARG, "NULL required pointer");
  cudaError_t e = launch_stop_check(entropy, pred, pred_prev, batch, canvas, (double)threshold,
                                    step, done, halt_step, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stop check");
  return DD_OK;
}

namespace {
// Adaptive-loop workspace: the block-loop layout, then two prediction
// buffers, the entropies and the per-canvas halt flags.
size_t adaptive_ws_layout(const dd_attn_desc* desc, int64_t total, const int32_t* cu_prefix_host,
                          int vocab, size_t* state_off, size_t* conf_off, size_t* extra_off) {
  const size_t base = block_ws_layout(desc, total, cu_prefix_host, vocab, state_off, conf_off);
  const size_t rows = (size_t)desc->batch * desc->canvas;
  if (extra_off) *extra_off = base;
  return base + 2 * align256(rows * 4) + align256(rows * 4) + align256((size_t)desc->batch);
}
}  // namespace

size_t dd_soft_embed_workspace(int rows, int vocab, int d) {
  if (rows < 0 || vocab < 1 || d < 64 || d % 64 != 0) return 0;
  return kHeaderBytes + soft_embed_scratch_bytes(rows, vocab, d);
}

namespace {
// The soft embedding's argument checks up to the tensor pointers (no device
// work); rows == 0 passes them.
dd_status check_soft_embed(const void* logits, dd_dtype dtype, int rows, int vocab,
                           int64_t row_stride, float temperature, const void* emb, int d,
                           const void* out) {
  if (dtype != DD_BF16 && dtype != DD_F32 && dtype != DD_E4M3)
    return fail(DD_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (dtype != DD_BF16) return fail(DD_ERR_UNSUPPORTED, "soft embedding takes bf16 logits and E");
  if (rows < 0 || vocab < 1) return fail(DD_ERR_INVALID_ARG, "rows=%d vocab=%d", rows, vocab);
  if (d < 64 || d % 64 != 0) return fail(DD_ERR_UNSUPPORTED, "d=%d (a multiple of 64)", d);
  if (row_stride < vocab || row_stride % 8 != 0)
    return fail(DD_ERR_INVALID_ARG, "row_stride (%lld) must be >= vocab and a multiple of 8",
                (long long)row_stride);
  if (!std::isfinite(temperature) || temperature < 1e-3f)
    return fail(DD_ERR_INVALID_ARG, "temperature must be finite and >= 1e-3");
  if (rows == 0) return DD_OK;
  if (rows > 65535 * 256) return fail(DD_ERR_UNSUPPORTED, "rows=%d", rows);
  if (!logits || !emb || !out) return fail(DD_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(logits) || !aligned16(emb) || !aligned16(out))
    return fail(DD_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  return DD_OK;
}

// The soft embedding's three kernels into `out`, with the workspace header
// at `ws` and its scratch right after it.
dd_status run_soft_embed(const void* logits, int rows, int vocab, int64_t row_stride,
                         float temperature, const void* emb, int d, void* out, void* ws,
                         cudaStream_t stream) {
  SoftEmbedArgs a{};
  a.logits = logits;
  a.rows = rows;
  a.vocab = vocab;
  a.row_stride = row_stride;
  a.temperature = temperature;
  a.emb = emb;
  a.d = d;
  a.out = out;
  a.err = static_cast<uint32_t*>(ws);
  a.scratch = static_cast<uint8_t*>(ws) + kHeaderBytes;
  cudaError_t e = launch_soft_embed(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "soft embedding");
  return DD_OK;
}
}  // namespace

dd_status dd_soft_embed(const void* logits, dd_dtype dtype, int rows, int vocab,
                        int64_t row_stride, float temperature, const void* emb, int d, void* out,
                        void* workspace, size_t workspace_bytes, dd_stream_t stream) {
  g_last_error.clear();
  dd_status st = check_soft_embed(logits, dtype, rows, vocab, row_stride, temperature, emb, d, out);
  if (st != DD_OK || rows == 0) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(DD_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const size_t need = kHeaderBytes + soft_embed_scratch_bytes(rows, vocab, d);
  if (workspace_bytes < need)
    return fail(DD_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  return run_soft_embed(logits, rows, vocab, row_stride, temperature, emb, d, out, workspace,
                        reinterpret_cast<cudaStream_t>(stream));
}

// ---- self-conditioning MLP
namespace {
// Shapes the dense layers take: rows >= 0, d and hidden multiples of 16.
dd_status check_ffw_shape(int rows, int d, int hidden) {
  if (rows < 0) return fail(DD_ERR_INVALID_ARG, "rows=%d", rows);
  if (d < 16 || hidden < 16) return fail(DD_ERR_INVALID_ARG, "d=%d hidden=%d", d, hidden);
  if (d % 16 != 0 || hidden % 16 != 0)
    return fail(DD_ERR_UNSUPPORTED, "d=%d hidden=%d (multiples of 16)", d, hidden);
  if ((int64_t)rows > 65535LL * 128) return fail(DD_ERR_UNSUPPORTED, "rows=%d", rows);
  return DD_OK;
}

dd_status check_ffw_ptrs(const void* w1, const void* b1, const void* w2, const void* b2,
                         const void* out) {
  if (!w1 || !b1 || !w2 || !b2 || !out) return fail(DD_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(w1) || !aligned16(b1) || !aligned16(w2) || !aligned16(b2) || !aligned16(out))
    return fail(DD_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  return DD_OK;
}

// MLP scratch: the bf16 hidden activations, then the fp32 partials of the
// K splits (one region for both layers, which run one after the other).
size_t ffw_scratch_bytes(int rows, int d, int hidden) {
  return align256((size_t)rows * hidden * 2) +
         align256(std::max(dense_partial_bytes(rows, d, hidden),
                           dense_partial_bytes(rows, hidden, d)));
}

// The two dense layers: hid = GELU(u W1 + b1), out = hid W2 + b2; `scratch`
// holds ffw_scratch_bytes.
dd_status run_ffw(const void* u, int rows, int d, int hidden, const void* w1, const void* b1,
                  const void* w2, const void* b2, void* out, void* scratch, uint32_t* err,
                  cudaStream_t stream) {
  void* hid = scratch;
  void* part = static_cast<uint8_t*>(scratch) + align256((size_t)rows * hidden * 2);
  DenseArgs l1{u, w1, b1, hid, rows, d, hidden, true, err, part};
  cudaError_t e = launch_dense(l1, stream);
  if (e != cudaSuccess) return cuda_fail(e, "self-conditioning MLP, layer 1");
  DenseArgs l2{hid, w2, b2, out, rows, hidden, d, false, err, part};
  e = launch_dense(l2, stream);
  if (e != cudaSuccess) return cuda_fail(e, "self-conditioning MLP, layer 2");
  return DD_OK;
}
}  // namespace

size_t dd_ffw_workspace(int rows, int d, int hidden) {
  if (rows < 0 || d < 16 || hidden < 16 || d % 16 || hidden % 16) return 0;
  return kHeaderBytes + ffw_scratch_bytes(rows, d, hidden);
}

dd_status dd_ffw(const void* u, int rows, int d, int hidden, const void* w1, const void* b1,
                 const void* w2, const void* b2, void* out, void* workspace,
                 size_t workspace_bytes, dd_stream_t stream) {
  g_last_error.clear();
  dd_status st = check_ffw_shape(rows, d, hidden);
  if (st != DD_OK || rows == 0) return st;
  st = check_ffw_ptrs(w1, b1, w2, b2, out);
  if (st != DD_OK) return st;
  if (!u || !aligned16(u)) return fail(DD_ERR_INVALID_ARG, "u must be non-NULL and 16-byte aligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(DD_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const size_t need = kHeaderBytes + ffw_scratch_bytes(rows, d, hidden);
  if (workspace_bytes < need)
    return fail(DD_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return run_ffw(u, rows, d, hidden, w1, b1, w2, b2, out, ws + kHeaderBytes,
                 reinterpret_cast<uint32_t*>(ws), reinterpret_cast<cudaStream_t>(stream));
}

size_t dd_self_condition_workspace(int rows, int vocab, int d, int hidden) {
  if (rows < 0 || vocab < 1 || d < 64 || d % 64 || hidden < 16 || hidden % 16) return 0;
  return kHeaderBytes + align256(soft_embed_scratch_bytes(rows, vocab, d)) +
         align256((size_t)rows * d * 2) + ffw_scratch_bytes(rows, d, hidden);
}

dd_status dd_self_condition(const void* logits, dd_dtype dtype, int rows, int vocab,
                            int64_t row_stride, float temperature, const void* emb, int d,
                            const void* w1, const void* b1, int hidden, const void* w2,
                            const void* b2, void* out, void* u_out, void* workspace,
                            size_t workspace_bytes, dd_stream_t stream) {
  g_last_error.clear();
  // every check before the first launch
  dd_status st = check_soft_embed(logits, dtype, rows, vocab, row_stride, temperature, emb, d,
                                  out);
  if (st != DD_OK) return st;
  st = check_ffw_shape(rows, d, hidden);
  if (st != DD_OK || rows == 0) return st;
  st = check_ffw_ptrs(w1, b1, w2, b2, out);
  if (st != DD_OK) return st;
  if (u_out && !aligned16(u_out)) return fail(DD_ERR_INVALID_ARG, "u_out must be 16-byte aligned");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(DD_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const size_t need = dd_self_condition_workspace(rows, vocab, d, hidden);
  if (workspace_bytes < need)
    return fail(DD_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t se = align256(soft_embed_scratch_bytes(rows, vocab, d));
  void* u = u_out ? u_out : ws + kHeaderBytes + se;
  void* hid = ws + kHeaderBytes + se + align256((size_t)rows * d * 2);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = run_soft_embed(logits, rows, vocab, row_stride, temperature, emb, d, u, workspace, s);
  if (st != DD_OK) return st;
  return run_ffw(u, rows, d, hidden, w1, b1, w2, b2, out, hid, reinterpret_cast<uint32_t*>(ws),
                 s);
}

// A captured block loop: one instantiated CUDA graph and the number of
// library kernels one replay launches.
struct dd_block_graph_st {
  cudaGraphExec_t exec;
  uint64_t launches;
};

dd_status dd_denoise_block_graph_create(
    dd_block_graph* out, const dd_attn_desc* desc, int steps, const void* q_steps,
    const void* kc_steps, const void* vc_steps, const void* k_prefix, const void* v_prefix,
    const int32_t* cu_prefix, const int32_t* cu_prefix_host, void* attn_out,
    const void* logits_steps, int vocab, const float* rate_host, const float* temperature_host,
    uint64_t seed, uint32_t step0, int32_t* canvas, int32_t* canvas_history, float* conf_steps,
    void* workspace, size_t workspace_bytes) {
  g_last_error.clear();
  if (!out) return fail(DD_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  cudaStream_t s = nullptr;
  cudaError_t e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cuda_fail(e, "capture stream");
  // relaxed mode: the first call of a kernel sets its attributes and
  // queries its occupancy, which are not stream work
  e = cudaStreamBeginCapture(s, cudaStreamCaptureModeRelaxed);
  if (e != cudaSuccess) {
    cudaStreamDestroy(s);
    return cuda_fail(e, "begin capture");
  }
  const uint64_t l0 = g_launches;
  dd_status st = dd_denoise_block(desc, steps, q_steps, kc_steps, vc_steps, k_prefix, v_prefix,
                                  cu_prefix, cu_prefix_host, attn_out, logits_steps, vocab,
                                  rate_host, temperature_host, seed, step0, canvas, canvas_history,
                                  conf_steps, workspace, workspace_bytes,
                                  reinterpret_cast<dd_stream_t>(s));
  const uint64_t launches = g_launches - l0;
  g_launches = l0;  // captured, not launched
  const std::string detail = g_last_error;
  cudaGraph_t graph = nullptr;
  e = cudaStreamEndCapture(s, &graph);
  cudaStreamDestroy(s);
  if (st != DD_OK) {
    if (graph) cudaGraphDestroy(graph);
    g_last_error = detail;
    return st;
  }
  if (e != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    return cuda_fail(e, "end capture");
  }
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (e != cudaSuccess) return cuda_fail(e, "instantiate block graph");
  *out = new dd_block_graph_st{exec, launches};
  return DD_OK;
}

dd_status dd_denoise_block_graph_launch(dd_block_graph g, dd_stream_t stream) {
  g_last_error.clear();
  if (!g) return fail(DD_ERR_INVALID_ARG, "graph is NULL");
  cudaError_t e = cudaGraphLaunch(g->exec, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "launch block graph");
  g_launches += g->launches;
  return DD_OK;
}

dd_status dd_denoise_block_graph_destroy(dd_block_graph g) {
  g_last_error.clear();
  if (!g) return DD_OK;
  cudaError_t e = cudaGraphExecDestroy(g->exec);
  delete g;
  if (e != cudaSuccess) return cuda_fail(e, "destroy block graph");
  return DD_OK;
}

size_t dd_denoise_block_adaptive_workspace(const dd_attn_desc* desc,
                                           const int32_t* cu_prefix_host, int vocab) {
  int64_t total = 0;
  if (vocab < 1 || check_attn_desc(desc, cu_prefix_host, &total) != DD_OK) return 0;
  return adaptive_ws_layout(desc, total, cu_prefix_host, vocab, nullptr, nullptr, nullptr);
}

// Validated arguments and workspace regions of one adaptive block loop.
struct AdaptiveLoop {
  const dd_attn_desc* desc;
  const uint8_t *q, *kc, *vc, *logits;
  const void *kp, *vp;
  const int32_t *cu, *cu_host;
  uint8_t* attn_out;
  int vocab, B, C, rows;
  const float* temps;
  float budget, stop_entropy;
  uint64_t seed;
  uint32_t step0;
  int32_t *canvas, *history, *halt_step;
  void* ws;
  size_t state_off, q_step, kv_step, lg_step;
  int32_t* pred[2];  // step i writes pred[i % 2] and compares with pred[(i + 1) % 2]
  float *ent, *conf;
  uint8_t* done;
};

static dd_status adaptive_prepare(AdaptiveLoop* L, const dd_attn_desc* desc, int max_steps,
                                  const void* q_steps, const void* kc_steps, const void* vc_steps,
                                  const void* k_prefix, const void* v_prefix,
                                  const int32_t* cu_prefix, const int32_t* cu_prefix_host,
                                  void* attn_out, const void* logits_steps, int vocab,
                                  const float* temperature_host, float budget, float stop_entropy,
                                  uint64_t seed, uint32_t step0, int32_t* canvas,
                                  int32_t* canvas_history, int32_t* halt_step, void* workspace,
                                  size_t workspace_bytes) {
  int64_t total = 0;
  dd_status st = check_attn_desc(desc, cu_prefix_host, &total);
  if (st != DD_OK) return st;
  if (max_steps < 0) return fail(DD_ERR_INVALID_ARG, "max_steps < 0");
  if (max_steps > 0 && !temperature_host) return fail(DD_ERR_INVALID_ARG, "temperature_host is NULL");
  if (!canvas || !halt_step) return fail(DD_ERR_INVALID_ARG, "NULL required pointer");
  if (desc->canvas > 1024) return fail(DD_ERR_UNSUPPORTED, "canvas > 1024");
  if (std::isnan(budget) || std::isnan(stop_entropy))
    return fail(DD_ERR_INVALID_ARG, "budget / stop_entropy is NaN");
  if ((uint64_t)step0 + (uint64_t)max_steps > (1ull << 32))
    return fail(DD_ERR_INVALID_ARG, "step0 + max_steps exceeds 2^32");
  if (vocab < 1) return fail(DD_ERR_INVALID_ARG, "vocab=%d", vocab);
  L->desc = desc;
  L->B = desc->batch;
  L->C = desc->canvas;
  L->rows = L->B * L->C;
  const size_t es = elem_size(desc->dtype);
  L->q_step = (size_t)L->rows * desc->heads_q * desc->head_dim * es;
  L->kv_step = (size_t)L->rows * desc->heads_kv * desc->head_dim * es;
  L->lg_step = (size_t)L->rows * (size_t)vocab * es;
  size_t conf_off = 0, extra_off = 0;
  const size_t need = adaptive_ws_layout(desc, total, cu_prefix_host, vocab, &L->state_off,
                                         &conf_off, &extra_off);
  if (!workspace) return fail(DD_ERR_WORKSPACE, "workspace is NULL");
  if (workspace_bytes < need)
    return fail(DD_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  uint8_t* const ws = static_cast<uint8_t*>(workspace);
  const size_t pred_bytes = align256((size_t)L->rows * 4);
  L->pred[0] = reinterpret_cast<int32_t*>(ws + extra_off);
  L->pred[1] = reinterpret_cast<int32_t*>(ws + extra_off + pred_bytes);
  L->ent = reinterpret_cast<float*>(ws + extra_off + 2 * pred_bytes);
  L->done = ws + extra_off + 3 * pred_bytes;
  L->conf = reinterpret_cast<float*>(ws + conf_off);
  L->q = static_cast<const uint8_t*>(q_steps);
  L->kc = static_cast<const uint8_t*>(kc_steps);
  L->vc = static_cast<const uint8_t*>(vc_steps);
  L->logits = static_cast<const uint8_t*>(logits_steps);
  L->kp = k_prefix;
  L->vp = v_prefix;
  L->cu = cu_prefix;
  L->cu_host = cu_prefix_host;
  L->attn_out = static_cast<uint8_t*>(attn_out);
  L->vocab = vocab;
  L->temps = temperature_host;
  L->budget = budget;
  L->stop_entropy = stop_entropy;
  L->seed = seed;
  L->step0 = step0;
  L->canvas = canvas;
  L->history = canvas_history;
  L->halt_step = halt_step;
  L->ws = workspace;
  return DD_OK;
}

// The work of step i on stream s: attention, the sampler (no scheduled
// re-noise: the acceptance rule decides it), the halt test against step
// i - 1's predictions, the acceptance into the canvas, the history copy.
static dd_status adaptive_step(const AdaptiveLoop& L, int i, cudaStream_t s) {
  dd_status st = run_attn(L.desc, L.q + i * L.q_step, L.kc + i * L.kv_step, L.vc + i * L.kv_step,
                          L.kp, L.vp, L.cu, L.cu_host, L.attn_out + i * L.q_step, nullptr, L.ws,
                          L.state_off, s);
  if (st != DD_OK) return st;
  dd_sample_params sp;
  sp.temperature = L.temps[i];
  sp.renoise_rate = 0.f;
  sp.seed = L.seed;
  sp.step = L.step0 + (uint32_t)i;
  sp.row_offset = 0;
  int32_t* cur = L.pred[i % 2];
  int32_t* prev = i > 0 ? L.pred[(i + 1) % 2] : nullptr;
  st = run_sampler(L.logits + i * L.lg_step, L.desc->dtype, L.rows, L.vocab, L.vocab, &sp, cur,
                   nullptr, L.conf, L.ent, nullptr, L.ws, L.state_off, s,
                   static_cast<uint8_t*>(L.ws) + L.state_off);
  if (st != DD_OK) return st;
  cudaError_t e = launch_stop_check(L.ent, cur, prev, L.B, L.C, (double)L.stop_entropy, i,
                                    L.done, L.halt_step, s);
  if (e == cudaSuccess)
    e = launch_entropy_accept(L.ent, cur, L.B, L.C, L.vocab, (double)L.budget, L.seed,
                              L.step0 + (uint32_t)i, 0, L.done, L.halt_step, i, L.canvas, nullptr,
                              s);
  if (e == cudaSuccess && L.history)
    e = cudaMemcpyAsync(L.history + (size_t)i * L.rows, L.canvas, (size_t)L.rows * sizeof(int32_t),
                        cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "adaptive step");
  return DD_OK;
}

dd_status dd_denoise_block_adaptive(const dd_attn_desc* desc, int max_steps, const void* q_steps,
                                    const void* kc_steps, const void* vc_steps,
                                    const void* k_prefix, const void* v_prefix,
                                    const int32_t* cu_prefix, const int32_t* cu_prefix_host,
                                    void* attn_out, const void* logits_steps, int vocab,
                                    const float* temperature_host, float budget,
                                    float stop_entropy, uint64_t seed, uint32_t step0,
                                    int32_t* canvas, int32_t* canvas_history,
                                    int32_t* halt_step, int* steps_run, void* workspace,
                                    size_t workspace_bytes, dd_stream_t stream) {
  g_last_error.clear();
  if (!steps_run) return fail(DD_ERR_INVALID_ARG, "NULL required pointer");
  AdaptiveLoop L;
  dd_status st = adaptive_prepare(&L, desc, max_steps, q_steps, kc_steps, vc_steps, k_prefix,
                                  v_prefix, cu_prefix, cu_prefix_host, attn_out, logits_steps,
                                  vocab, temperature_host, budget, stop_entropy, seed, step0,
                                  canvas, canvas_history, halt_step, workspace, workspace_bytes);
  if (st != DD_OK) return st;
  *steps_run = 0;
  if (L.B == 0) return DD_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(L.done, 0, (size_t)L.B, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(halt_step, 0xff, (size_t)L.B * sizeof(int32_t), s);
  if (e != cudaSuccess) return cuda_fail(e, "adaptive loop init");
  std::vector<uint8_t> done_h((size_t)L.B);
  for (int i = 0; i < max_steps; ++i) {
    st = adaptive_step(L, i, s);
    if (st != DD_OK) return st;
    e = cudaMemcpyAsync(done_h.data(), L.done, (size_t)L.B, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "adaptive step");
    *steps_run = i + 1;
    bool all = true;
    for (int b = 0; b < L.B; ++b) all = all && done_h[(size_t)b] != 0;
    if (all) break;
  }
  return DD_OK;
}

struct dd_adaptive_graph_st {
  cudaGraphExec_t exec;
  uint64_t launches;  // kernels of every step body (an upper bound per replay)
};

// Builds and instantiates the adaptive loop's graph: memset nodes that reset
// the loop state, then one IF node per step on a handle whose default is 1.
// A failed CUDA call returns DD_ERR_CUDA with the call's name.
static dd_status build_adaptive_graph(const AdaptiveLoop& L, int max_steps, int32_t* steps_run,
                                      cudaGraphExec_t* exec_out, uint64_t* launches_out) {
  dd_status st = DD_OK;
  const char* what = nullptr;  // the CUDA call that failed
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t r, const char* call) {
    if (r != cudaSuccess && e == cudaSuccess) {
      e = r;
      what = call;
    }
    return e == cudaSuccess;
  };
  cudaGraph_t graph = nullptr;
  cudaStream_t s = nullptr;
  if (!ok(cudaGraphCreate(&graph, 0), "cudaGraphCreate")) return cuda_fail(e, "cudaGraphCreate");
  // the loop's state is reset by the graph itself on every replay
  std::vector<cudaGraphNode_t> deps;
  auto add_memset = [&](void* dst, unsigned value, unsigned elem, size_t n) {
    cudaMemsetParams mp = {};
    mp.dst = dst;
    mp.pitch = n * elem;
    mp.value = value;
    mp.elementSize = elem;
    mp.width = n;
    mp.height = 1;
    cudaGraphNode_t node = nullptr;
    if (ok(cudaGraphAddMemsetNode(&node, graph, nullptr, 0, &mp), "cudaGraphAddMemsetNode"))
      deps.push_back(node);
  };
  add_memset(steps_run, 0u, 4, 1);
  if (L.B > 0) add_memset(L.done, 0u, 1, (size_t)L.B);
  if (L.B > 0) add_memset(L.halt_step, 0xffffffffu, 4, (size_t)L.B);
  // one handle per IF node (a handle serves a single conditional node): step
  // 0's defaults to 1 at every launch, the others to 0; step i's gate sets
  // step i + 1's, so once every canvas has halted no later body runs
  std::vector<cudaGraphConditionalHandle> handles(L.B > 0 ? (size_t)max_steps : 0);
  for (size_t i = 0; i < handles.size(); ++i)
    ok(cudaGraphConditionalHandleCreate(&handles[i], graph, i == 0 ? 1u : 0u,
                                        cudaGraphCondAssignDefault),
       "cudaGraphConditionalHandleCreate");
  if (L.B > 0) ok(cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking), "cudaStreamCreateWithFlags");
  const uint64_t l0 = g_launches;
  for (int i = 0; e == cudaSuccess && st == DD_OK && L.B > 0 && i < max_steps; ++i) {
    cudaGraphNodeParams np = {};
    np.type = cudaGraphNodeTypeConditional;
    np.conditional.handle = handles[(size_t)i];
    np.conditional.type = cudaGraphCondTypeIf;
    np.conditional.size = 1;
    cudaGraphNode_t node = nullptr;
    if (!ok(cudaGraphAddNode(&node, graph, deps.data(), deps.size(), &np), "cudaGraphAddNode"))
      break;
    cudaGraph_t body = np.conditional.phGraph_out[0];
    if (!ok(cudaStreamBeginCaptureToGraph(s, body, nullptr, nullptr, 0,
                                          cudaStreamCaptureModeRelaxed),
            "cudaStreamBeginCaptureToGraph"))
      break;
    st = adaptive_step(L, i, s);
    cudaError_t eg = cudaSuccess;
    if (st == DD_OK) {
      const bool has_next = i + 1 < max_steps;
      eg = launch_adaptive_gate(L.done, L.B, i, steps_run,
                                has_next ? handles[(size_t)i + 1] : handles[(size_t)i], has_next,
                                s);
    }
    cudaGraph_t captured = nullptr;
    const std::string detail = g_last_error;
    ok(cudaStreamEndCapture(s, &captured), "cudaStreamEndCapture");
    if (st != DD_OK) g_last_error = detail;
    ok(eg, "gate kernel launch");
    deps.assign(1, node);
  }
  *launches_out = g_launches - l0;
  g_launches = l0;  // captured, not launched
  if (s) cudaStreamDestroy(s);
  if (st == DD_OK && e == cudaSuccess)
    ok(cudaGraphInstantiate(exec_out, graph, 0), "cudaGraphInstantiate");
  const std::string detail = g_last_error;
  cudaGraphDestroy(graph);
  g_last_error = detail;
  if (st != DD_OK) return st;
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, what);
  }
  return DD_OK;
}

dd_status dd_denoise_block_adaptive_graph_create(
    dd_adaptive_graph* out, const dd_attn_desc* desc, int max_steps, const void* q_steps,
    const void* kc_steps, const void* vc_steps, const void* k_prefix, const void* v_prefix,
    const int32_t* cu_prefix, const int32_t* cu_prefix_host, void* attn_out,
    const void* logits_steps, int vocab, const float* temperature_host, float budget,
    float stop_entropy, uint64_t seed, uint32_t step0, int32_t* canvas, int32_t* canvas_history,
    int32_t* halt_step, int32_t* steps_run, void* workspace, size_t workspace_bytes) {
  g_last_error.clear();
  if (!out) return fail(DD_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!steps_run) return fail(DD_ERR_INVALID_ARG, "NULL required pointer");
  AdaptiveLoop L;
  dd_status st = adaptive_prepare(&L, desc, max_steps, q_steps, kc_steps, vc_steps, k_prefix,
                                  v_prefix, cu_prefix, cu_prefix_host, attn_out, logits_steps,
                                  vocab, temperature_host, budget, stop_entropy, seed, step0,
                                  canvas, canvas_history, halt_step, workspace, workspace_bytes);
  if (st != DD_OK) return st;
  cudaGraphExec_t exec = nullptr;
  uint64_t launches = 0;
  st = build_adaptive_graph(L, max_steps, steps_run, &exec, &launches);
  if (st == DD_ERR_CUDA) {
    // programmatic dependencies inside conditional bodies are not accepted
    // everywhere: build again with plain launches
    const std::string first = g_last_error;
    g_pdl_off = true;
    st = build_adaptive_graph(L, max_steps, steps_run, &exec, &launches);
    g_pdl_off = false;
    if (st != DD_OK) {
      const std::string second = g_last_error;
      return fail(st, "with programmatic launches: %s; with plain launches: %s", first.c_str(),
                  second.c_str());
    }
  }
  if (st != DD_OK) return st;
  *out = new dd_adaptive_graph_st{exec, launches};
  return DD_OK;
}

dd_status dd_denoise_block_adaptive_graph_launch(dd_adaptive_graph g, dd_stream_t stream) {
  g_last_error.clear();
  if (!g) return fail(DD_ERR_INVALID_ARG, "graph is NULL");
  cudaError_t e = cudaGraphLaunch(g->exec, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "launch adaptive graph");
  g_launches += g->launches;
  return DD_OK;
}

dd_status dd_denoise_block_adaptive_graph_destroy(dd_adaptive_graph g) {
  g_last_error.clear();
  if (!g) return DD_OK;
  cudaError_t e = cudaGraphExecDestroy(g->exec);
  delete g;
  if (e != cudaSuccess) return cuda_fail(e, "destroy adaptive graph");
  return DD_OK;
}

dd_status dd_workspace_init(void* workspace, size_t workspace_bytes, dd_stream_t stream) {
  g_last_error.clear();
  if (!workspace || workspace_bytes < kHeaderBytes)
    return fail(DD_ERR_WORKSPACE, "workspace must hold at least %zu bytes", kHeaderBytes);
  cudaError_t e =
      cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "workspace init");
  return DD_OK;
}

dd_status dd_query_device_error(void* workspace, dd_stream_t stream) {
  g_last_error.clear();
  if (!workspace) return fail(DD_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(&word, workspace, sizeof word, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(workspace, 0, sizeof word);
  if (e != cudaSuccess) return cuda_fail(e, "query device error");
  if (word & kDevErrTimeout)
    return fail(DD_ERR_DEVICE_TIMEOUT, "a kernel pipeline wait exceeded its time limit");
  if (word & kDevErrBounds)
    return fail(DD_ERR_DEVICE_BOUNDS, "device-side index check failed (inconsistent cu_prefix?)");
  return DD_OK;
}

const char* dd_status_string(dd_status s) {
  switch (s) {
    case DD_OK: return "ok";
    case DD_ERR_INVALID_ARG: return "invalid argument";
    case DD_ERR_UNSUPPORTED: return "unsupported configuration";
    case DD_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DD_ERR_CUDA: return "CUDA error";
    case DD_ERR_DEVICE_TIMEOUT: return "device pipeline wait timed out";
    case DD_ERR_DEVICE_BOUNDS: return "device index check failed";
  }
  return "unknown status";
}

const char* dd_last_error(void) { return g_last_error.c_str(); }

void dd_set_test_stall_ns(uint64_t ns) { g_stall_ns = ns; }

uint64_t dd_launch_count(void) { return g_launches; }
void dd_reset_launch_count(void) { g_launches = 0; }

}  // extern "C"
