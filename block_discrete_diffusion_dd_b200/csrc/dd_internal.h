// dd_internal.h -- declarations shared between the C-ABI layer (dd_abi.cu)
// and the kernel files.  Not part of the public interface (include/dd.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dd {

// Per-(row, vocabulary chunk) partial record written by the sampler's first
// pass (32 bytes, one per CTA).
struct alignas(32) ChunkRecord {
  float m, s, t, best;
  int idx;
  int pad[3];
};

struct SamplerArgs {
  const void* logits;
  bool bf16;
  int rows, vocab;
  int64_t row_stride;
  float inv_tau, rate;
  uint64_t seed;
  uint32_t step, row_offset;
  int32_t* tokens;
  int32_t* pred;
  float* conf;
  float* entropy;
  uint8_t* renoised;
  ChunkRecord* recs;
  uint32_t* err;  // device error word
};

int sampler_nchunk(int vocab, bool bf16);
cudaError_t launch_sampler(const SamplerArgs& a, cudaStream_t stream);
cudaError_t launch_init_canvas(int32_t* canvas, int rows, int vocab, uint64_t seed,
                               uint32_t row_offset, cudaStream_t stream);

// Attention launch description (validated by the ABI layer).
struct AttnArgs {
  int B, C, Hq, Hkv, D;
  float scale;
  bool bf16;
  const void *q, *kc, *vc, *kp, *vp;
  const int32_t* cu_prefix;       // device [B+1]
  const int32_t* cu_prefix_host;  // host [B+1]
  int64_t total_prefix;           // cu_prefix_host[B]
  void* out;
  float* lse;
  // scratch carved from the workspace
  uint32_t* err;  // device error word
  void* scratch;
  size_t scratch_bytes;
};

// Tensor-core (tcgen05) path: bf16, D = 128, (Hq/Hkv) divides 128.
bool attn_tc_supported(const AttnArgs& a);
size_t attn_tc_scratch_bytes(const AttnArgs& a);
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t stream);

// SIMT path: any supported dtype, D in {64, 128}.
size_t attn_simt_scratch_bytes(const AttnArgs& a);
cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t stream);

// Launch accounting (per host thread).
void note_launch();

// Device error codes latched in the workspace header.
enum : uint32_t { kDevErrTimeout = 1u, kDevErrBounds = 2u };

}  // namespace dd
