// dd_noalloc.cu -- dd_sample_renoise_noalloc: the sampler step for callers
// that cannot allocate device memory.
//
// Some callers of this library are not allowed to call cudaMalloc: code that
// runs inside another framework's memory pool or under a fixed memory budget
// reserved at start-up, plugin or callback code that is handed only its input
// and output pointers, and latency-critical loops where cudaMalloc's implicit
// device synchronisation is not acceptable.  dd_sample_renoise needs a
// caller-provided workspace; this variant instead keeps its scratch (the
// device error word, the sampler's ticket counter and row keys, and the
// per-chunk partial records) in one file-scope static __device__ array of
// kStaticScratchBytes, which every GPU that loads the library holds until
// the process exits.  The array starts zeroed, as the counter and the row
// keys must be, and every call leaves them zero again.  The caller still
// passes the logits and every output buffer.
#include <cstdio>
#include <mutex>

#include "dd.h"
#include "dd_internal.h"

namespace dd {

dd_status sample_with_scratch(const void* logits, dd_dtype dtype, int rows, int vocab,
                              int64_t row_stride, const dd_sample_params* p, int32_t* tokens,
                              int32_t* pred, float* conf, float* entropy, uint8_t* renoised,
                              void* scratch, size_t scratch_bytes, cudaStream_t stream);
dd_status set_error(dd_status st, const char* msg);

namespace {

constexpr size_t kStaticScratchBytes = 4u << 20;  // 4 MiB per device
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code this name is only a host-side handle, not
// a device address: the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Once per device, with that device current: resolve the array's device
// address.  Returns nullptr (and sets the error text) on failure.
void* scratch_for_current_device(dd_status* st) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = set_error(DD_ERR_CUDA, "dd_sample_renoise_noalloc: no usable current CUDA device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      char msg[256];
      snprintf(msg, sizeof msg, "dd_sample_renoise_noalloc: cudaGetSymbolAddress failed: %s",
               cudaGetErrorString(e));
      *st = set_error(DD_ERR_CUDA, msg);
      return nullptr;
    }
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

}  // namespace
}  // namespace dd

using namespace dd;

extern "C" dd_status dd_sample_renoise_noalloc(const void* logits, dd_dtype dtype, int rows,
                                               int vocab, int64_t row_stride,
                                               const dd_sample_params* params,
                                               int32_t* tokens_out, int32_t* pred_out,
                                               float* conf_out, float* entropy_out,
                                               uint8_t* renoised_out, dd_stream_t stream) {
  // size check first: it needs no device
  const size_t need = dd_sample_renoise_workspace(rows, vocab, dtype);
  if (need == 0)
    return set_error(DD_ERR_INVALID_ARG, "dd_sample_renoise_noalloc: invalid rows/vocab/dtype");
  if (need > kStaticScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "dd_sample_renoise_noalloc: this call needs %zu bytes of scratch but the static "
             "scratch holds %zu; split the rows over several calls (row_offset keeps the "
             "random numbers unchanged) or use dd_sample_renoise with a workspace",
             need, kStaticScratchBytes);
    return set_error(DD_ERR_UNSUPPORTED, msg);
  }
  if (rows == 0) return DD_OK;
  dd_status st = DD_OK;
  void* scratch = scratch_for_current_device(&st);
  if (scratch == nullptr) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the error word is OR-accumulated by the kernels: it starts every call at
  // zero (the partial records need no clearing: each is written before read)
  cudaError_t e = cudaMemsetAsync(scratch, 0, 16, s);
  if (e != cudaSuccess) return set_error(DD_ERR_CUDA, "dd_sample_renoise_noalloc: memset failed");
  return sample_with_scratch(logits, dtype, rows, vocab, row_stride, params, tokens_out, pred_out,
                             conf_out, entropy_out, renoised_out, scratch, kStaticScratchBytes, s);
}
