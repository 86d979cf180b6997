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

// Exact Gumbel score z - ln(-ln U) in fp32.  -ln U is taken as
// -log1p(-(1 - U)) for U >= 1/2, where 1 - U is exact, so it stays accurate
// as U approaches 1.
__device__ __forceinline__ float gumbel_score(float z, uint32_t w) {
  const float U = uniform24(w);
  const float lnU = U < 0.5f ? logf(U) : log1pf(-(1.0f - U));
  return z - logf(-lnU);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// Logits below -2^15 are treated as -2^15: exp underflows to 0 either way
// (unless the whole row lies below it), and -inf entries and padding stay
// out of 0 * inf products.  A power of two keeps x * c2 exact, so a thread
// that has seen only padding gets d = 0 exactly.
constexpr float kFloorLogit = -32768.0f;

// Per-thread running state.  Softmax sums in log2 units relative to a lazy
// reference m (raised only when an entry exceeds it by more than 2^8, so the
// terms stay below 256), kept as packed pairs so two entries update with one
// f32x2 instruction; best = best Gumbel score (natural units), idx its index.
struct Run {
  float m;
  float2 s2, t2;
  float best;
  int idx;
};

constexpr float kLazy = 8.0f;  // log2 headroom of the lazy reference

// Raise the lazy reference of `st` to ym, rescaling its sums.
__device__ __forceinline__ void raise_ref(Run& st, float ym) {
  const float s = st.s2.x + st.s2.y, t = st.t2.x + st.t2.y;
  if (s > 0.f) {
    const float f = ex2_approx(st.m - ym);
    st.t2 = make_float2(f * fmaf(s, st.m - ym, t), 0.f);
    st.s2 = make_float2(s * f, 0.f);
  }
  st.m = ym;
}

// Prune threshold factor Kp = (1 + 2^-8) e^(m ln 2 - best_w), clamped; 0 in
// a warp that holds padding alone (best_w = -inf).
__device__ __forceinline__ float prune_factor(float m, float best_w) {
  return best_w == -INFINITY ? 0.f
                             : fminf(ex2_approx(m - best_w * kLog2e) * 1.00390625f, 1e30f);
}

// bf16 pairs in a 32-bit word, floored at kFloorLogit (max.bf16x2 is exact).
__device__ __forceinline__ uint32_t floor_bf16x2(uint32_t w) {
  uint32_t r;
  // 0xC700 is the bf16 value -32768 = kFloorLogit
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(0xC700C700u));
  return r;
}
__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ void unpack8(uint4 raw, float (&x)[8], float& bm) {
  raw.x = floor_bf16x2(raw.x);
  raw.y = floor_bf16x2(raw.y);
  raw.z = floor_bf16x2(raw.z);
  raw.w = floor_bf16x2(raw.w);
  const uint32_t mx = max_bf16x2(max_bf16x2(raw.x, raw.y), max_bf16x2(raw.z, raw.w));
  bm = fmaxf(bf16lo(mx), bf16hi(mx));
  x[0] = bf16lo(raw.x); x[1] = bf16hi(raw.x);
  x[2] = bf16lo(raw.y); x[3] = bf16hi(raw.y);
  x[4] = bf16lo(raw.z); x[5] = bf16hi(raw.z);
  x[6] = bf16lo(raw.w); x[7] = bf16hi(raw.w);
}

__device__ __forceinline__ void unpack8(float4 a, float4 b, float (&x)[8], float& bm) {
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = fmaxf(x[i], kFloorLogit);
  bm = fmaxf(fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3])), fmaxf(fmaxf(x[4], x[5]), fmaxf(x[6], x[7])));
}

// Reduce the CTA's states and write its chunk record.  Within a warp: the
// common reference M first, then every lane rescales its sums to M and the
// sums and the argmax (lowest index on equal scores) reduce by butterflies,
// a fixed tree, so the result does not depend on scheduling.
__device__ __forceinline__ SampState warp_reduce(const Run& r) {
  float M = r.m;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float s = r.s2.x + r.s2.y, t = r.t2.x + r.t2.y;
  if (s > 0.f) {
    const float f = ex2_approx(r.m - M);
    t = f * fmaf(s, r.m - M, t);
    s *= f;
  } else {
    s = 0.f;
    t = 0.f;
  }
  float best = r.best;
  int idx = r.idx;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, off);
    t += __shfl_xor_sync(0xffffffffu, t, off);
    const float ob = __shfl_xor_sync(0xffffffffu, best, off);
    const int oi = __shfl_xor_sync(0xffffffffu, idx, off);
    if (ob > best || (ob == best && oi < idx)) {
      best = ob;
      idx = oi;
    }
  }
  return SampState{M, s, t, best, idx};
}

__device__ __forceinline__ void write_record(const Run& r, ChunkRecord* rec) {
  const SampState st = warp_reduce(r);
  __shared__ SampState red[kSampleThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = st;
  __syncthreads();
  if (threadIdx.x == 0) {
    SampState a = red[0];
#pragma unroll
    for (int w = 1; w < kSampleThreads / 32; ++w) merge_state(a, red[w]);
    ChunkRecord out;
    out.m = a.m;
    out.s = a.s;
    out.t = a.t;
    out.best = a.best;
    out.idx = a.idx;
    *rec = out;
  }
}

constexpr uint32_t kStageBytes = 32768;  // logits per CTA (one bulk copy)

template <typename T>
__host__ __device__ constexpr int chunk_elems() { return (int)(kStageBytes / sizeof(T)); }

// Gumbel scores order like floats; as ints for atomicMax on shared memory.
__device__ __forceinline__ int ord_float(float f) {
  const int b = __float_as_int(f);
  return b ^ ((b >> 31) & 0x7fffffff);
}
__device__ __forceinline__ float unord_float(int o) {
  return __int_as_float(o ^ ((o >> 31) & 0x7fffffff));
}

// One item = 8 consecutive entries x[0..7] (floored, finite) starting at v0,
// with bm = their max.  `src` points at the item's first entry (in shared
// memory, or in global memory on the scalar path) and is re-read only on the
// rare exact path.  best_w is the warp's view of the best Gumbel score so far;
// cta_best holds the best over the whole CTA (ordered int), which every warp
// adopts when it is higher than its own.
template <typename T>
__device__ __forceinline__ void process_item(Run& st, float& best_w, float& Kp, const float (&x)[8],
                                             float bm, uint32_t v0, bool seed, const T* src,
                                             const PhiloxKey& key, const PhiloxRow& prow,
                                             float c2, float inv_tau, int* cta_best) {
  const float ym = bm * c2;
  if (ym > st.m + kLazy) {  // rare after the first item
    raise_ref(st, ym);
    Kp = prune_factor(st.m, best_w);
  }
  {
    const float cb = unord_float(*reinterpret_cast<volatile int*>(cta_best));
    if (cb > best_w) {
      best_w = cb;
      Kp = prune_factor(st.m, best_w);
    }
  }
  const float2 c22 = make_float2(c2, c2);
  const float2 nm = make_float2(-st.m, -st.m);
  float2 p[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 d = __ffma2_rn(make_float2(x[2 * j], x[2 * j + 1]), c22, nm);
    p[j] = make_float2(ex2_approx(d.x), ex2_approx(d.y));
    st.s2 = __fadd2_rn(st.s2, p[j]);
    st.t2 = __ffma2_rn(p[j], d, st.t2);
  }
  // Gumbel words for the 8 entries: two Philox blocks.
  const uint4 wa = philox4x32_10_row(v0 >> 2, 0u, prow, key);
  const uint4 wb = philox4x32_10_row((v0 >> 2) + 1u, 0u, prow, key);
  bool changed = false;
  if (seed) {
    // seed the threshold with the exact score of this lane's largest entry
    if (bm > kFloorLogit) {
      int j = 7;
#pragma unroll
      for (int i = 6; i >= 0; --i) j = (x[i] == bm) ? i : j;
      const uint4 wq = j < 4 ? wa : wb;
      const uint32_t i4 = (uint32_t)j & 3u;
      const uint32_t wj = i4 == 0 ? wq.x : i4 == 1 ? wq.y : i4 == 2 ? wq.z : wq.w;
      st.best = gumbel_score(bm * inv_tau, wj);
      st.idx = (int)(v0 + (uint32_t)j);
    }
    // the seeded threshold applies to this item's own test below
    best_w = fmaxf(best_w, warp_max(st.best));
    if ((threadIdx.x & 31) == 0) atomicMax(cta_best, ord_float(best_w));
    Kp = prune_factor(st.m, best_w);
  }
  // Exponential-race prune: the score z - ln E (E = -ln U) can beat best_w
  // only if E < e^(z - best_w); since E >= 1 - U, an entry with
  // 1 - U >= e^(z - best_w) (1 + 2^-8) is skipped without a logarithm.  With
  // U' = 1 + (x >> 9) 2^-23 = U + 1 - 2^-24 the test reads
  // U' > 2 - 2^-23 - p Kp.
  const float2 kk = make_float2(-Kp, -Kp);
  const float2 cc = make_float2(1.99999988079071044921875f, 1.99999988079071044921875f);
  const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
  float thr[8];
  bool any = false;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 t = __ffma2_rn(p[j], kk, cc);
    thr[2 * j] = t.x;
    thr[2 * j + 1] = t.y;
    any |= __uint_as_float(0x3F800000u | (w[2 * j] >> 9)) > t.x;
    any |= __uint_as_float(0x3F800000u | (w[2 * j + 1] >> 9)) > t.y;
  }
  if (any) {
    // rare exact path: one entry at a time (the logit re-read, its word
    // selected from the two blocks above), so the code below exists once
    uint32_t cmask = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      cmask |= (__uint_as_float(0x3F800000u | (w[i] >> 9)) > thr[i]) ? (1u << i) : 0u;
    while (cmask) {
      const int i = __ffs(cmask) - 1;
      cmask &= cmask - 1;
      const float xi = fmaxf((float)src[i], kFloorLogit);
      const uint32_t v = v0 + (uint32_t)i;
      const uint4 wq = i < 4 ? wa : wb;
      const int i4 = i & 3;
      const uint32_t wi = i4 == 0 ? wq.x : i4 == 1 ? wq.y : i4 == 2 ? wq.z : wq.w;
      const float sc = gumbel_score(xi * inv_tau, wi);
      if (sc > st.best || (sc == st.best && (int)v < st.idx)) {
        st.best = sc;
        st.idx = (int)v;
        changed = true;
      }
    }
  }
  if (__any_sync(0xffffffffu, changed)) {
    best_w = fmaxf(best_w, warp_max(st.best));
    if ((threadIdx.x & 31) == 0) atomicMax(cta_best, ord_float(best_w));
    Kp = prune_factor(st.m, best_w);
  }
}

// Vector path: rows 16-byte aligned and V % 8 == 0.  Thread 0 fetches the
// CTA's 32 KB slice of the row with one bulk asynchronous copy into shared
// memory; all 256 threads then stream it 8 entries at a time.
template <typename T>
__global__ void __launch_bounds__(kSampleThreads, 4)
    sample_chunk_bulk_kernel(const T* __restrict__ logits, int64_t row_stride, int vocab,
                             int nchunk, float inv_tau, uint64_t seed, uint32_t step,
                             uint32_t row_offset, ChunkRecord* __restrict__ recs,
                             uint32_t* __restrict__ err) {
  constexpr int kElems = chunk_elems<T>();
  constexpr int kItems = kElems / (kSampleThreads * 8);
  __shared__ __align__(128) uint8_t buf[kStageBytes];
  __shared__ uint64_t bar;
  __shared__ int cta_best;
  const int row = blockIdx.x / nchunk;
  const int chunk = blockIdx.x - row * nchunk;
  const int c0 = chunk * kElems;
  const int n = min(kElems, vocab - c0);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    cta_best = ord_float(-INFINITY);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar, (uint32_t)(n * sizeof(T)));
    bulk_load(buf, logits + (int64_t)row * row_stride + c0, (uint32_t)(n * sizeof(T)), &bar);
  }
  const PhiloxKey key = philox_key(seed);
  const uint32_t grow = row_offset + (uint32_t)row;
  const PhiloxRow prow = philox_row(grow, step, 0u, key);
  const float c2 = inv_tau * kLog2e;
  Run st{-INFINITY, make_float2(0.f, 0.f), make_float2(0.f, 0.f), -INFINITY, 0x7fffffff};
  float best_w = -INFINITY, Kp = 0.f;
  if (!mbar_wait_bounded(&bar, 0, nullptr, 1000000000ull)) {
    // never observed: the copy is plain memory traffic; report and drain
    if (threadIdx.x == 0) atomicOr(err, kDevErrTimeout);
    mbar_wait_bounded(&bar, 0, nullptr, 4000000000ull);
    return;
  }
  const T* tb = reinterpret_cast<const T*>(buf);
#pragma unroll 1
  for (int k = 0; k < kItems; ++k) {
    const int e = (k * kSampleThreads + (int)threadIdx.x) * 8;
    float x[8], bm;
    if (e < n) {
      if constexpr (sizeof(T) == 2) {
        unpack8(*reinterpret_cast<const uint4*>(buf + e * 2), x, bm);
      } else {
        const float4* q = reinterpret_cast<const float4*>(buf + e * 4);
        unpack8(q[0], q[1], x, bm);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = kFloorLogit;
      bm = kFloorLogit;
    }
    process_item<T>(st, best_w, Kp, x, bm, (uint32_t)(c0 + e), k == 0, tb + e, key, prow, c2,
                    inv_tau, &cta_best);
  }
  write_record(st, recs + (int64_t)row * nchunk + chunk);
}

// Scalar path for unaligned rows or V % 8 != 0: direct loads with bounds
// checks; entries at or beyond V read as kFloorLogit and never win (their p
// is 0, so the prune never selects them and they are never re-read).
template <typename T>
__global__ void __launch_bounds__(kSampleThreads)
    sample_chunk_scalar_kernel(const T* __restrict__ logits, int64_t row_stride, int vocab,
                               int nchunk, float inv_tau, uint64_t seed, uint32_t step,
                               uint32_t row_offset, ChunkRecord* __restrict__ recs) {
  constexpr int kElems = chunk_elems<T>();
  constexpr int kItems = kElems / (kSampleThreads * 8);
  const int row = blockIdx.x / nchunk;
  const int chunk = blockIdx.x - row * nchunk;
  const int c0 = chunk * kElems;
  const T* rowp = logits + (int64_t)row * row_stride;
  const PhiloxKey key = philox_key(seed);
  const uint32_t grow = row_offset + (uint32_t)row;
  const PhiloxRow prow = philox_row(grow, step, 0u, key);
  const float c2 = inv_tau * kLog2e;
  Run st{-INFINITY, make_float2(0.f, 0.f), make_float2(0.f, 0.f), -INFINITY, 0x7fffffff};
  float best_w = -INFINITY, Kp = 0.f;
  __shared__ int cta_best;
  if (threadIdx.x == 0) cta_best = ord_float(-INFINITY);
  __syncthreads();
#pragma unroll 1
  for (int k = 0; k < kItems; ++k) {
    const int v0 = c0 + (k * kSampleThreads + (int)threadIdx.x) * 8;
    float x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      x[i] = (v0 + i < vocab) ? fmaxf((float)rowp[v0 + i], kFloorLogit) : kFloorLogit;
    float bm = x[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) bm = fmaxf(bm, x[i]);
    process_item<T>(st, best_w, Kp, x, bm, (uint32_t)v0, k == 0, rowp + v0, key, prow, c2,
                    inv_tau, &cta_best);
  }
  write_record(st, recs + (int64_t)row * nchunk + chunk);
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
  const int nchunk = (a.vocab + chunk_elems<T>() - 1) / chunk_elems<T>();
  const T* lg = static_cast<const T*>(a.logits);
  const size_t esz = sizeof(T);
  const bool vec = ((reinterpret_cast<uintptr_t>(lg) & 15u) == 0) &&
                   (((size_t)a.row_stride * esz) % 16 == 0) && (a.vocab % 8 == 0);
  const int64_t grid = (int64_t)a.rows * nchunk;
  if (vec)
    sample_chunk_bulk_kernel<T><<<(unsigned)grid, kSampleThreads, 0, stream>>>(
        lg, a.row_stride, a.vocab, nchunk, a.inv_tau, a.seed, a.step, a.row_offset, a.recs,
        a.err);
  else
    sample_chunk_scalar_kernel<T><<<(unsigned)grid, kSampleThreads, 0, stream>>>(
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

int sampler_nchunk(int vocab, bool bf16) {
  const int ce = bf16 ? chunk_elems<__nv_bfloat16>() : chunk_elems<float>();
  return (vocab + ce - 1) / ce;
}

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
