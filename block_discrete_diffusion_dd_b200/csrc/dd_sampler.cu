// dd_sampler.cu -- the vocabulary-wide sampler, re-noise and canvas-init
// kernels ("DiffusionGemma Technical Report", paperfeed review, "The
// mechanism": temperature-scaled logits -> per-position entropies; tokens
// that are not kept are re-noised to uniformly random vocabulary tokens).
//
// Two launches per step:
//   sample_chunk  streams the logits once (128-bit loads), and for each
//                 (row, vocabulary chunk) produces a partial record: running
//                 max, sum of exp, entropy accumulator, and the best Gumbel
//                 score with its index;
//   sample_merge  merges a row's records in a fixed order, then draws the
//                 re-noise decision and the replacement token.
// HBM traffic is one read of the logits plus a few bytes per row.
#include "dd_device.cuh"
#include "dd_internal.h"

namespace dd {

namespace {

constexpr int kSampleThreads = 256;
constexpr int kItemsPerThread = 4;  // 8 logits per item
constexpr int kChunk = kSampleThreads * kItemsPerThread * 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Partial state over a set of vocabulary entries, in log2 units:
// m = max y, s = sum 2^(y-m), t = sum 2^(y-m) (y-m), with y = logit/tau*log2 e;
// best = max Gumbel score z - ln(-ln U) (natural units), idx its index.
struct SampState {
  float m, s, t, best;
  int idx;
};

__device__ __forceinline__ void merge_state(SampState& a, const SampState& b) {
  const float M = fmaxf(a.m, b.m);
  if (M != -INFINITY) {
    float sa = 0.f, ta = 0.f, sb = 0.f, tb = 0.f;
    if (a.s > 0.f) {
      const float f = ex2_approx(a.m - M);
      sa = a.s * f;
      ta = f * fmaf(a.s, a.m - M, a.t);
    }
    if (b.s > 0.f) {
      const float f = ex2_approx(b.m - M);
      sb = b.s * f;
      tb = f * fmaf(b.s, b.m - M, b.t);
    }
    a.s = sa + sb;
    a.t = ta + tb;
  }
  a.m = M;
  if (b.best > a.best || (b.best == a.best && b.idx < a.idx)) {
    a.best = b.best;
    a.idx = b.idx;
  }
}

__device__ __forceinline__ SampState shfl_state(const SampState& s, int lane_mask) {
  SampState o;
  o.m = __shfl_xor_sync(0xffffffffu, s.m, lane_mask);
  o.s = __shfl_xor_sync(0xffffffffu, s.s, lane_mask);
  o.t = __shfl_xor_sync(0xffffffffu, s.t, lane_mask);
  o.best = __shfl_xor_sync(0xffffffffu, s.best, lane_mask);
  o.idx = __shfl_xor_sync(0xffffffffu, s.idx, lane_mask);
  return o;
}

// Butterfly over the warp; every lane ends with the same merged state and
// the merge tree is fixed, so the result does not depend on scheduling.
__device__ __forceinline__ void warp_merge(SampState& s) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    SampState o = shfl_state(s, off);
    // merge in a lane-order-independent way: always (lower lane) <- (upper)
    const int lane = threadIdx.x & 31;
    if (lane & off) {
      SampState lo = o;
      merge_state(lo, s);
      s = lo;
    } else {
      merge_state(s, o);
    }
  }
}

// Loads of 8 consecutive logits as fp32.
template <typename T, bool kVec>
struct Load8;

template <>
struct Load8<__nv_bfloat16, true> {
  uint4 raw;
  __device__ __forceinline__ void issue(const __nv_bfloat16* p, int64_t, int64_t) {
    raw = __ldcs(reinterpret_cast<const uint4*>(p));
  }
  __device__ __forceinline__ void get(float (&x)[8]) const {
    x[0] = bf16lo(raw.x); x[1] = bf16hi(raw.x);
    x[2] = bf16lo(raw.y); x[3] = bf16hi(raw.y);
    x[4] = bf16lo(raw.z); x[5] = bf16hi(raw.z);
    x[6] = bf16lo(raw.w); x[7] = bf16hi(raw.w);
  }
};

template <>
struct Load8<float, true> {
  float4 a, b;
  __device__ __forceinline__ void issue(const float* p, int64_t, int64_t) {
    a = __ldcs(reinterpret_cast<const float4*>(p));
    b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void get(float (&x)[8]) const {
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

// Scalar path for unaligned rows or a vocabulary that is not a multiple of
// 8: entries at or beyond `vocab` read as -inf and never win.
template <typename T>
struct Load8<T, false> {
  float v[8];
  __device__ __forceinline__ void issue(const T* p, int64_t v0, int64_t vocab) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (v0 + i < vocab) ? (float)p[i] : -INFINITY;
  }
  __device__ __forceinline__ void get(float (&x)[8]) const {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = v[i];
  }
};

template <typename T, bool kVec>
__global__ void __launch_bounds__(kSampleThreads)
    sample_chunk_kernel(const T* __restrict__ logits, int64_t row_stride, int vocab, int nchunk,
                        float inv_tau, uint64_t seed, uint32_t step, uint32_t row_offset,
                        ChunkRecord* __restrict__ recs) {
  const int row = blockIdx.x / nchunk;
  const int chunk = blockIdx.x - row * nchunk;
  const T* rowp = logits + (int64_t)row * row_stride;
  const int64_t c0 = (int64_t)chunk * kChunk;

  Load8<T, kVec> ld[kItemsPerThread];
  int64_t vbase[kItemsPerThread];
#pragma unroll
  for (int k = 0; k < kItemsPerThread; ++k) {
    vbase[k] = c0 + (int64_t)(k * kSampleThreads + threadIdx.x) * 8;
    if (vbase[k] < vocab) ld[k].issue(rowp + vbase[k], vbase[k], vocab);
  }

  const PhiloxKey key = philox_key(seed);
  const uint32_t grow = row_offset + (uint32_t)row;
  const float c2 = inv_tau * kLog2e;

  SampState st{-INFINITY, 0.f, 0.f, -INFINITY, 0x7fffffff};
  float Kp = 1e30f;  // (1 + 2^-8) e^(m ln 2 - best), clamped

#pragma unroll
  for (int k = 0; k < kItemsPerThread; ++k) {
    if (vbase[k] >= vocab) continue;
    float x[8];
    ld[k].get(x);
    float bm = x[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) bm = fmaxf(bm, x[i]);
    const float ym = bm * c2;
    if (ym > st.m) {
      if (st.s > 0.f) {
        const float f = ex2_approx(st.m - ym);
        st.t = f * fmaf(st.s, st.m - ym, st.t);
        st.s *= f;
      }
      st.m = ym;
      Kp = fminf(ex2_approx(st.m - st.best * kLog2e) * 1.00390625f, 1e30f);
    }
    float p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float d = fmaf(x[i], c2, -st.m);
      p[i] = ex2_approx(d);
      st.s += p[i];
      st.t = fmaf(p[i], d, st.t);
    }
    // Gumbel words for the 8 entries: two Philox blocks.
    const uint32_t q0 = (uint32_t)(vbase[k] >> 2);
    const uint4 wa = philox4x32_10(make_uint4(q0, grow, step, 0u), key);
    const uint4 wb = philox4x32_10(make_uint4(q0 + 1u, grow, step, 0u), key);
    const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    // Exponential-race prune: the score z - ln E (E = -ln U) can only beat
    // `best` if E < e^(z - best); since E >= 1 - U, entries with
    // 1 - U >= e^(z - best) are skipped without any logarithm.  The test is
    // U' > 2 - 2^-23 - p Kp with U' = 1 + (x >> 9) 2^-23 (conservative).
    bool any = false;
    float thr[8], f[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      f[i] = __uint_as_float(0x3F800000u | (w[i] >> 9));
      thr[i] = fmaf(-p[i], Kp, 1.99999988079071044921875f);
      any |= f[i] > thr[i];
    }
    if (any) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (f[i] > thr[i] && x[i] != -INFINITY) {
          const float U = uniform24(w[i]);
          const float E = -logf(U);
          const float sc = x[i] * inv_tau - logf(E);
          if (sc > st.best) {
            st.best = sc;
            st.idx = (int)(vbase[k] + i);
          }
        }
      }
      Kp = fminf(ex2_approx(st.m - st.best * kLog2e) * 1.00390625f, 1e30f);
    }
  }

  warp_merge(st);
  __shared__ SampState red[kSampleThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = st;
  __syncthreads();
  if (warp == 0) {
    SampState s = lane < kSampleThreads / 32
                      ? red[lane]
                      : SampState{-INFINITY, 0.f, 0.f, -INFINITY, 0x7fffffff};
    warp_merge(s);
    if (lane == 0) {
      ChunkRecord r;
      r.m = s.m;
      r.s = s.s;
      r.t = s.t;
      r.best = s.best;
      r.idx = s.idx;
      recs[(int64_t)row * nchunk + chunk] = r;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(128)
    sample_merge_kernel(const T* __restrict__ logits, int64_t row_stride, int rows, int vocab,
                        int nchunk, float inv_tau, float rate, uint64_t seed, uint32_t step,
                        uint32_t row_offset, const ChunkRecord* __restrict__ recs,
                        int32_t* __restrict__ tokens, int32_t* __restrict__ pred,
                        float* __restrict__ conf, float* __restrict__ entropy,
                        uint8_t* __restrict__ renoised) {
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  SampState st{-INFINITY, 0.f, 0.f, -INFINITY, 0x7fffffff};
  for (int c = lane; c < nchunk; c += 32) {
    const ChunkRecord r = recs[(int64_t)row * nchunk + c];
    SampState o{r.m, r.s, r.t, r.best, r.idx};
    merge_state(st, o);
  }
  warp_merge(st);
  if (lane != 0) return;
  const int p = st.idx;
  const float x = (float)logits[(int64_t)row * row_stride + p];
  const float c2 = inv_tau * kLog2e;
  const float cf = ex2_approx(fmaf(x, c2, -st.m)) / st.s;
  const float ent = logf(st.s) - kLn2 * (st.t / st.s);
  const uint32_t grow = row_offset + (uint32_t)row;
  const float u1 = uniform24(philox_word0(seed, grow, step, 1u));
  const bool rn = u1 < rate;
  const uint32_t x2 = philox_word0(seed, grow, step, 2u);
  const int32_t repl = (int32_t)(((uint64_t)x2 * (uint64_t)(uint32_t)vocab) >> 32);
  tokens[row] = rn ? repl : p;
  if (pred) pred[row] = p;
  conf[row] = cf;
  if (entropy) entropy[row] = ent;
  if (renoised) renoised[row] = rn ? 1 : 0;
}

__global__ void init_canvas_kernel(int32_t* __restrict__ canvas, int rows, int vocab,
                                   uint64_t seed, uint32_t row_offset) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const uint32_t x = philox_word0(seed, row_offset + (uint32_t)r, 0u, 3u);
  canvas[r] = (int32_t)(((uint64_t)x * (uint64_t)(uint32_t)vocab) >> 32);
}

template <typename T>
cudaError_t launch_sampler_t(const SamplerArgs& a, cudaStream_t stream) {
  const int nchunk = sampler_nchunk(a.vocab);
  const T* lg = static_cast<const T*>(a.logits);
  const size_t esz = sizeof(T);
  const bool vec = ((reinterpret_cast<uintptr_t>(lg) & 15u) == 0) &&
                   (((size_t)a.row_stride * esz) % 16 == 0) && (a.vocab % 8 == 0);
  const int64_t grid = (int64_t)a.rows * nchunk;
  if (vec)
    sample_chunk_kernel<T, true><<<(unsigned)grid, kSampleThreads, 0, stream>>>(
        lg, a.row_stride, a.vocab, nchunk, a.inv_tau, a.seed, a.step, a.row_offset, a.recs);
  else
    sample_chunk_kernel<T, false><<<(unsigned)grid, kSampleThreads, 0, stream>>>(
        lg, a.row_stride, a.vocab, nchunk, a.inv_tau, a.seed, a.step, a.row_offset, a.recs);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sample_merge_kernel<T><<<(a.rows + 3) / 4, 128, 0, stream>>>(
      lg, a.row_stride, a.rows, a.vocab, nchunk, a.inv_tau, a.rate, a.seed, a.step,
      a.row_offset, a.recs, a.tokens, a.pred, a.conf, a.entropy, a.renoised);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

int sampler_nchunk(int vocab) { return (vocab + kChunk - 1) / kChunk; }

cudaError_t launch_sampler(const SamplerArgs& a, cudaStream_t stream) {
  if (a.bf16) return launch_sampler_t<__nv_bfloat16>(a, stream);
  return launch_sampler_t<float>(a, stream);
}

cudaError_t launch_init_canvas(int32_t* canvas, int rows, int vocab, uint64_t seed,
                               uint32_t row_offset, cudaStream_t stream) {
  init_canvas_kernel<<<(rows + 255) / 256, 256, 0, stream>>>(canvas, rows, vocab, seed,
                                                              row_offset);
  note_launch();
  return cudaGetLastError();
}

}  // namespace dd
