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
// the process exits.  Every call clears the part of it that it reads before
// writing (error word, counter, its rows' maxima) on the stream before its
// kernels run, so a call that failed on the device cannot leave a later one
// wrong.  The caller still passes the logits and every output buffer.
#include <cuda.h>

#include <cstdio>
#include <mutex>

#include "dd.h"
#include "dd_internal.h"

namespace dd {

dd_status sample_with_scratch(const void* logits, dd_dtype dtype, int rows, int vocab,
                              int64_t row_stride, const dd_sample_params* p, int32_t* tokens,
                              int32_t* pred, float* conf, float* entropy, uint8_t* renoised,
                              void* scratch, size_t scratch_bytes, cudaStream_t stream);
dd_status check_sampler_call(const void* logits, dd_dtype dtype, int rows, int vocab,
                             int64_t row_stride, const dd_sample_params* p,
                             const int32_t* tokens, const float* conf);
dd_status set_error(dd_status st, const char* msg);

namespace {

constexpr size_t kStaticScratchBytes = 4u << 20;  // 4 MiB per device
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code this name is only a host-side handle, not
// a device address: the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

std::mutex g_setup_mu;

// The array's device address is looked up once per CUDA context: a device
// reset (or any teardown of the context) reloads the module, and the array
// may then sit at another address.  The context is identified by its
// driver-assigned id, which is never reused within a process.
struct ScratchAddr {
  unsigned long long ctx_id;
  void* ptr;
};
ScratchAddr g_scratch_addr[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Id of the current context, or 0 if the driver cannot tell (the address is
// then looked up again on every call).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
    cudaGetLastError();
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr &&
      get_id(ctx, &id) == CUDA_SUCCESS)
    return id;
  return 0;
}

// With the device current: the array's device address in the current
// context, looked up (cudaGetSymbolAddress) the first time a context is
// seen.  Returns nullptr (and sets the error text) on failure.
void* scratch_for_current_device(dd_status* st) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = set_error(DD_ERR_CUDA, "dd_sample_renoise_noalloc: no usable current CUDA device");
    return nullptr;
  }
  // cudaGetSymbolAddress below also makes the device's primary context
  // current if none is, so the id is read after it on a first call
  std::lock_guard<std::mutex> lock(g_setup_mu);
  ScratchAddr& slot = g_scratch_addr[dev];
  const unsigned long long id = current_context_id();
  if (slot.ptr == nullptr || id == 0 || slot.ctx_id != id) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      char msg[256];
      snprintf(msg, sizeof msg, "dd_sample_renoise_noalloc: cudaGetSymbolAddress failed: %s",
               cudaGetErrorString(e));
      *st = set_error(DD_ERR_CUDA, msg);
      return nullptr;
    }
    slot.ptr = ptr;
    slot.ctx_id = current_context_id();
  }
  return slot.ptr;
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
  // every check that needs no device comes first: a rejected call queues no
  // GPU work (and leaves nothing in a graph being captured)
  dd_status st = check_sampler_call(logits, dtype, rows, vocab, row_stride, params, tokens_out,
                                    conf_out);
  if (st != DD_OK) return st;
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
  void* scratch = scratch_for_current_device(&st);
  if (scratch == nullptr) return st;
  // clears the state this call reads, then runs the kernels
  return sample_with_scratch(logits, dtype, rows, vocab, row_stride, params, tokens_out, pred_out,
                             conf_out, entropy_out, renoised_out, scratch, kStaticScratchBytes,
                             reinterpret_cast<cudaStream_t>(stream));
}
