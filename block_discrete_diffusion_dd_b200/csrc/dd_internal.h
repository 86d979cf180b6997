// dd_internal.h -- declarations shared between the C-ABI layer (dd_abi.cu)
// and the kernel files.  Not part of the public interface (include/dd.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

namespace dd {

// False on this host thread while work is captured where programmatic
// dependencies are not accepted (launch_pdl then launches plainly).
bool pdl_enabled();

// Launch with programmatic stream serialisation (the kernel calls pdl_wait
// before touching global memory): its launch overlaps the tail of the
// previous kernel on the stream, in eager launches and in captured graphs.
// (pdl_wait and launch_dependents are no-ops in a plain launch.)
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

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
  void* recs;     // per-chunk softmax partials, sampler_record_bytes()
  void* state;    // ticket counter and row keys, sampler_state_bytes(); zero
                  // before the first call, and left zero by every call
  uint32_t* err;  // device error word
};

// The sampler's persistent state: a ticket counter (first 256 bytes) and one
// 64-bit argmax key per row.  Zero between calls (the merge kernel clears it).
struct SamplerState {
  uint32_t* ticket;
  unsigned long long* row_key;
};
SamplerState sampler_state(void* state);
size_t sampler_state_bytes(int rows);
// Per-chunk partial records (16 bytes per chunk of 2048 entries).
size_t sampler_record_bytes(int rows, int vocab);
cudaError_t launch_sampler(const SamplerArgs& a, cudaStream_t stream);

// The pages' acceptance rule and early-halt test (dd_policy.cu); C <= 1024.
cudaError_t launch_entropy_accept(const float* entropy, const int32_t* pred, int B, int C,
                                  int vocab, double budget, uint64_t seed, uint32_t step,
                                  uint32_t row_offset, const uint8_t* done,
                                  const int32_t* halt_step, int32_t cur, int32_t* tokens,
                                  uint8_t* accepted, cudaStream_t stream);
cudaError_t launch_stop_check(const float* entropy, const int32_t* pred, const int32_t* pred_prev,
                              int B, int C, double threshold, int32_t cur, uint8_t* done,
                              int32_t* halt_step, cudaStream_t stream);
// Writes steps_run = step + 1 and (has_next) sets the next step's IF-node
// condition of the on-device adaptive loop: 1 while a canvas is running, 0
// once all have halted.
cudaError_t launch_adaptive_gate(const uint8_t* done, int B, int32_t step, int32_t* steps_run,
                                 cudaGraphConditionalHandle next, bool has_next,
                                 cudaStream_t stream);
cudaError_t launch_init_canvas(int32_t* canvas, int rows, int vocab, uint64_t seed,
                               uint32_t row_offset, cudaStream_t stream);

// Attention launch description (validated by the ABI layer).
struct AttnArgs {
  int B, C, Hq, Hkv, D;
  float scale;
  bool bf16;
  bool e4m3;                         // 8-bit E4M3 inputs, bf16 output
  float q_scale, k_scale, v_scale;   // E4M3 per-tensor factors
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

// Tensor-core (tcgen05) path: bf16 or E4M3, D = 128, (Hq/Hkv) divides 128.
bool attn_tc_supported(const AttnArgs& a);
size_t attn_tc_scratch_bytes(const AttnArgs& a);
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t stream);

// SIMT path: any supported dtype, D in {64, 128}.
size_t attn_simt_scratch_bytes(const AttnArgs& a);
cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t stream);

// Self-conditioning soft embedding (dd_soft_embed.cu): bf16 logits [rows, V]
// (row stride a multiple of 8), bf16 E [V, d] (d a multiple of 64), bf16 out
// [rows, d]; 16-byte aligned pointers, validated by the ABI layer.
struct SoftEmbedArgs {
  const void* logits;
  int rows, vocab;
  int64_t row_stride;
  float temperature;
  const void* emb;
  int d;
  void* out;
  uint32_t* err;
  void* scratch;  // soft_embed_scratch_bytes
};
struct SoftEmbedPlan {
  int ksteps, ksteps_per_split, splits, grid_x, grid_z;
};
SoftEmbedPlan soft_embed_plan(int rows, int vocab, int d);
size_t soft_embed_scratch_bytes(int rows, int vocab, int d);
cudaError_t launch_soft_embed(const SoftEmbedArgs& a, cudaStream_t stream);

// 2-D bf16 TMA map over [outer, inner] (row stride in elements), box
// (box_inner, box_outer) with box_inner * 2 bytes of swizzling (64 or 128),
// out-of-bounds elements read as zero.  False if the driver rejects it.
bool encode_2d(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t stride,
               int box_inner, int box_outer);

// One dense layer on the tensor cores (dd_ffw.cu):
//   out[r, n] = act(sum_k x[r, k] w[k, n] + bias[n]),  act = GELU or identity
// x bf16 [rows, K] (row stride K), w bf16 [K, N] (row stride N), bias bf16
// [N], out bf16 [rows, N]; K and N multiples of 16, 16-byte aligned
// pointers, validated by the ABI layer.  When K is split over CTAs, `part`
// holds their fp32 partials.
struct DenseArgs {
  const void* x;
  const void* w;
  const void* bias;
  void* out;
  int rows, K, N;
  bool gelu;
  uint32_t* err;
  void* part;  // fp32 partials, dense_partial_bytes(rows, K, N) (NULL when 0)
};
// The split of K over CTAs (device-dependent: about one wave over the SMs).
struct DensePlan {
  int ksteps_per_split, splits;
};
DensePlan dense_plan(int rows, int K, int N);
size_t dense_partial_bytes(int rows, int K, int N);
cudaError_t launch_dense(const DenseArgs& a, cudaStream_t stream);

// Time limit of the pipeline waits (mbarrier waits that can abort) of the
// tensor-core kernels launched from this host thread: 1 s unless a test
// stall is set (dd_set_test_stall_ns).  Waits that drain in-flight copies
// and MMAs before a CTA exits always keep their own 1 s limit.
uint64_t pipeline_wait_ns();
// True while a test stall is set on this host thread: each tensor-core
// kernel then makes one pipeline wait on a barrier nothing completes.
bool pipeline_test_stall();

// Launch accounting (per host thread).
void note_launch();

// Device error codes latched in the workspace header.
enum : uint32_t { kDevErrTimeout = 1u, kDevErrBounds = 2u };

}  // namespace dd
