// dd_policy.cu -- the pages' sampler policy around the sampler step
// ("DiffusionGemma Technical Report", paperfeed review, "The mechanism",
// sampler paragraph): positions accepted greedily from lowest to highest
// entropy until a cumulative entropy budget is exhausted, the rest re-noised
// to uniform random tokens; early halt when the mean canvas entropy drops
// below a threshold and the prediction is stable across two steps.
//
// Both kernels run one CTA per canvas (C <= 1024 positions).  The decisions
// are taken in float64 sums over float32 entropies, summed sequentially in
// a fixed order by one thread (256 dependent adds, about a microsecond), so
// they are the same decisions the definition gives, not just close to them.
#include "dd_device.cuh"
#include "dd_internal.h"

namespace dd {
namespace {

constexpr int kMaxCanvas = 1024;

__device__ __forceinline__ uint32_t ord_u32(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float unord_u32(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// Entropy-budget acceptance for canvas blockIdx.x.  Keys (entropy order,
// then position) are sorted by a bitonic network in shared memory; thread 0
// walks them in order with the float64 running sum.  A canvas that halted
// at an earlier step is left as it is; one that halts at this step keeps its
// whole prediction.
__global__ void __launch_bounds__(kMaxCanvas)
    entropy_accept_kernel(const float* __restrict__ entropy, const int32_t* __restrict__ pred,
                          int C, int vocab, double budget, uint64_t seed, uint32_t step,
                          uint32_t row_offset, const uint8_t* __restrict__ done,
                          const int32_t* __restrict__ halt_step, int32_t cur,
                          int32_t* __restrict__ tokens, uint8_t* __restrict__ accepted) {
  __shared__ unsigned long long key[kMaxCanvas];
  __shared__ uint8_t acc[kMaxCanvas];
  const int b = blockIdx.x, i = threadIdx.x, n = blockDim.x;  // n: power of two >= C
  bool keep_all = false;
  if (done != nullptr && done[b]) {
    if (halt_step == nullptr || halt_step[b] != cur) return;  // halted earlier
    keep_all = true;                                       // halts now
  }
  const int64_t r = (int64_t)b * C + i;
  key[i] = i < C ? ((unsigned long long)ord_u32(entropy[r]) << 32) | (unsigned)i : ~0ull;
  acc[i] = keep_all ? 1 : 0;
  __syncthreads();
  if (!keep_all) {
    for (int k = 2; k <= n; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        const int o = i ^ j;
        if (o > i) {
          const unsigned long long a = key[i], c = key[o];
          const bool up = (i & k) == 0;
          if ((a > c) == up) {
            key[i] = c;
            key[o] = a;
          }
        }
        __syncthreads();
      }
    }
    if (i == 0) {  // the sorted keys carry the entropies' bits
      double sum = 0.0;
      for (int k = 0; k < C; ++k) {
        const unsigned long long kv = key[k];
        const double next = sum + (double)unord_u32((uint32_t)(kv >> 32));
        if (!(next <= budget)) break;
        sum = next;
        acc[(uint32_t)kv] = 1;
      }
    }
    __syncthreads();
  }
  if (i < C) {
    int32_t t = pred[r];
    if (!acc[i]) {
      const uint32_t x = philox_word0(seed, row_offset + (uint32_t)r, step, 2u);
      t = (int32_t)(((uint64_t)x * (uint64_t)(uint32_t)vocab) >> 32);
    }
    tokens[r] = t;
    if (accepted) accepted[r] = acc[i];
  }
}

// Early-halt test for canvas blockIdx.x: halts (done, halt_step = cur) when
// the float64 mean of its entropies, summed in position order, is below the
// threshold and every prediction equals the previous step's.
__global__ void __launch_bounds__(256)
    stop_check_kernel(const float* __restrict__ entropy, const int32_t* __restrict__ pred,
                      const int32_t* __restrict__ pred_prev, int C, double threshold,
                      int32_t cur, uint8_t* __restrict__ done, int32_t* __restrict__ halt_step) {
  __shared__ float h[kMaxCanvas];
  const int b = blockIdx.x;
  if (done[b]) return;
  bool same = pred_prev != nullptr;
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    h[i] = entropy[(int64_t)b * C + i];
    if (pred_prev) same &= pred[(int64_t)b * C + i] == pred_prev[(int64_t)b * C + i];
  }
  same = __syncthreads_and(same) != 0;
  if (threadIdx.x == 0 && same) {
    double sum = 0.0;
    for (int i = 0; i < C; ++i) sum += (double)h[i];
    if (sum / (double)C < threshold) {
      done[b] = 1;
      halt_step[b] = cur;
    }
  }
}

// Gate between two steps of the on-device adaptive loop: one warp reads
// every canvas's halt flag, records that `step` has run, and (has_next) sets
// the condition of the next step's IF node to 1 while some canvas is still
// running and to 0 once all have halted.  A step whose body is skipped sets
// nothing, so every later condition keeps its default 0.
__global__ void __launch_bounds__(32)
    adaptive_gate_kernel(const uint8_t* __restrict__ done, int B, int32_t step,
                         int32_t* __restrict__ steps_run, cudaGraphConditionalHandle next,
                         int has_next) {
  bool all = true;
  for (int b = threadIdx.x; b < B; b += 32) all = all && done[b] != 0;
  all = __all_sync(0xffffffffu, all);
  if (threadIdx.x == 0) {
    *steps_run = step + 1;
    if (has_next) cudaGraphSetConditional(next, all ? 0u : 1u);
  }
}

int pow2_at_least(int c) {
  int n = 32;
  while (n < c) n <<= 1;
  return n;
}

}  // namespace

cudaError_t launch_entropy_accept(const float* entropy, const int32_t* pred, int B, int C,
                                  int vocab, double budget, uint64_t seed, uint32_t step,
                                  uint32_t row_offset, const uint8_t* done,
                                  const int32_t* halt_step, int32_t cur, int32_t* tokens,
                                  uint8_t* accepted, cudaStream_t stream) {
  entropy_accept_kernel<<<B, pow2_at_least(C), 0, stream>>>(entropy, pred, C, vocab, budget,
                                                            seed, step, row_offset, done,
                                                            halt_step, cur, tokens, accepted);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_stop_check(const float* entropy, const int32_t* pred, const int32_t* pred_prev,
                              int B, int C, double threshold, int32_t cur, uint8_t* done,
                              int32_t* halt_step, cudaStream_t stream) {
  stop_check_kernel<<<B, 256, 0, stream>>>(entropy, pred, pred_prev, C, threshold, cur, done,
                                           halt_step);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_adaptive_gate(const uint8_t* done, int B, int32_t step, int32_t* steps_run,
                                 cudaGraphConditionalHandle next, bool has_next,
                                 cudaStream_t stream) {
  adaptive_gate_kernel<<<1, 32, 0, stream>>>(done, B, step, steps_run, next, has_next ? 1 : 0);
  note_launch();
  return cudaGetLastError();
}

}  // namespace dd
