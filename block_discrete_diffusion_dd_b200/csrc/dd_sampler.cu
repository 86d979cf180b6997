// dd_sampler.cu -- the vocabulary-wide sampler, re-noise and canvas-init
// kernels ("DiffusionGemma Technical Report", paperfeed review, "The
// mechanism": temperature-scaled logits -> per-position entropies; tokens
// that are not kept are re-noised to uniformly random vocabulary tokens).
//
// Two launches per step:
//   sample_scan   one persistent pass over the logits.  Rows are cut into
//                 chunks of kChunk items (an item = 256 consecutive entries,
//                 8 per lane of a warp); warps take chunks from a ticket
//                 counter, so every warp stays busy until the pass ends
//                 whatever the scheduler's order.  Per chunk the warp writes
//                 the softmax partials (running max, sum of exp, entropy
//                 accumulator); the row's best Gumbel score and its index go
//                 to one 64-bit atomic maximum per row, which all warps also
//                 read back as the threshold of the exponential-race prune.
//   sample_merge  merges a row's chunk partials in chunk order (so the sums
//                 do not depend on which warp took which chunk), reads the
//                 argmax, draws the re-noise decision and the replacement
//                 token, and clears the counter and the row maxima for the
//                 next call.
// HBM traffic is one read of the logits plus a few bytes per chunk and row.
#include <algorithm>
#include <atomic>

#include "dd_device.cuh"
#include "dd_internal.h"

namespace dd {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Softmax partials over a set of vocabulary entries, in log2 units:
// m = max y, s = sum 2^(y-m), t = sum 2^(y-m) (y-m), with y = logit/tau*log2 e.
struct SumState {
  float m, s, t;
};

__device__ __forceinline__ void merge_sums(SumState& a, const SumState& b) {
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
}

// Butterfly over the warp; every lane ends with the same merged state and
// the merge tree is fixed, so the result does not depend on scheduling.
__device__ __forceinline__ void warp_merge_sums(SumState& s) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    SumState o;
    o.m = __shfl_xor_sync(0xffffffffu, s.m, off);
    o.s = __shfl_xor_sync(0xffffffffu, s.s, off);
    o.t = __shfl_xor_sync(0xffffffffu, s.t, off);
    // always (lower lane) <- (upper lane), whichever lane computes it
    if (lane & off) {
      SumState lo = o;
      merge_sums(lo, s);
      s = lo;
    } else {
      merge_sums(s, o);
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
// out of 0 * inf products.  A power of two keeps x * c2 exact.
constexpr float kFloorLogit = -32768.0f;

// Per-lane running state.  Softmax sums in log2 units relative to a lazy
// reference m (raised only when an entry exceeds it by more than kLazy, so
// the terms stay below 2^kLazy), kept as packed pairs so two entries update
// with one f32x2 instruction; best = the lane's best exact Gumbel score
// (natural units), idx its index.
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

// Prune threshold factor Kp = (1 + 2^-8) e^(m ln 2 - best_w).  Before any
// score is known (best_w = -inf) it is 2^126, which makes every entry whose
// relative weight p is nonzero a candidate.
__device__ __forceinline__ float prune_factor(float m, float best_w) {
  return best_w == -INFINITY ? 8.507059173023462e37f
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

// ------------------------------------------------------ row argmax keys
// The row's best (score, index) as one 64-bit key whose unsigned maximum is
// the highest score and, among equal scores, the lowest index: the score's
// bits mapped to an order-preserving unsigned word, then the complemented
// index.  Key 0 means "no score yet" (it lies below every real score).
__device__ __forceinline__ uint32_t ord_u32(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ unsigned long long pack_key(float best, int idx) {
  return ((unsigned long long)ord_u32(best) << 32) | (unsigned long long)(~(uint32_t)idx);
}
__device__ __forceinline__ float key_score(unsigned long long k) {
  if (k == 0ull) return -INFINITY;
  const uint32_t u = (uint32_t)(k >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
__device__ __forceinline__ int key_index(unsigned long long k) { return (int)~(uint32_t)k; }

// Row keys sit 128 bytes apart: every warp reads its row's key often, and
// keys of different rows then never share a cache line.
constexpr int kKeyStride = 16;

// ---------------------------------------------------------------- scan pass
constexpr int kScanThreads = 256;
constexpr int kScanWarpsPerCta = kScanThreads / 32;
constexpr int kItem = 256;  // entries per warp-item
constexpr int kChunk = 8;   // items per chunk (one ticket)

struct ScanParams {
  PhiloxKey key;      // round keys of the seed (read from the constant bank)
  int64_t row_stride;
  uint32_t nchunks;   // rows * nck
  int rows;
  int nck;            // chunks per row, ceil(ipr / kChunk)
  int ipr;            // items per row, ceil(V / 256)
  int vocab;
  int jtail;          // index of a row's partial last item, or -1
  float c2, inv_c2, inv_tau;
  uint32_t step, row_offset;
};

// One lane's 8 entries of an item, as loaded.
template <typename T, bool kVec>
struct ItemBuf {
  float v[8];  // scalar path: converted on load, padding as kFloorLogit
};
template <>
struct ItemBuf<__nv_bfloat16, true> {
  uint4 a;
};
template <>
struct ItemBuf<float, true> {
  float4 a, b;
};

// Load entries v0 .. v0+7 of a row (v0 = 256 j + 8 lane).  On the vector
// path (rows 16-byte aligned, V % 8 == 0) lanes past V re-read the row's
// last 8 entries instead, which the caller then discards as padding.
template <typename T, bool kVec>
__device__ __forceinline__ void load_item(ItemBuf<T, kVec>& b, const T* __restrict__ rowp, int v0,
                                          int vocab) {
  if constexpr (kVec) {
    const int off = min(v0, vocab - 8);
    if constexpr (sizeof(T) == 2) {
      b.a = __ldg(reinterpret_cast<const uint4*>(rowp + off));
    } else {
      b.a = __ldg(reinterpret_cast<const float4*>(rowp + off));
      b.b = __ldg(reinterpret_cast<const float4*>(rowp + off) + 1);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) b.v[i] = (v0 + i < vocab) ? (float)rowp[v0 + i] : kFloorLogit;
  }
}

// Lazy-reference test: does the item hold an entry above the threshold X
// (X <= (m + kLazy) / c2, the logit at which d = y - m would exceed kLazy)?
// The bf16 path compares in bf16 with X rounded down to a bf16 value.
template <typename T, bool kVec>
struct LazyTest {
  float x;
  __device__ __forceinline__ void set(float m, float inv_c2) { x = (m + kLazy) * inv_c2; }
};
template <>
struct LazyTest<__nv_bfloat16, true> {
  uint32_t x2;  // the threshold as a bf16 pair
  __device__ __forceinline__ void set(float m, float inv_c2) {
    const uint32_t f = __float_as_uint((m + kLazy) * inv_c2);
    uint32_t b = f >> 16;                         // truncation: toward zero
    if ((f & 0x80000000u) && (f & 0xffffu)) ++b;  // negative: one step further down
    x2 = b | (b << 16);
  }
};

// Unpack one item to floored floats x[8] and test it against the lazy
// reference threshold.
template <typename T, bool kVec>
__device__ __forceinline__ bool unpack_item(const ItemBuf<T, kVec>& b, const LazyTest<T, kVec>& lz,
                                            float (&x)[8]) {
  if constexpr (kVec && sizeof(T) == 2) {
    const uint32_t r0 = floor_bf16x2(b.a.x), r1 = floor_bf16x2(b.a.y);
    const uint32_t r2 = floor_bf16x2(b.a.z), r3 = floor_bf16x2(b.a.w);
    const uint32_t mx = max_bf16x2(max_bf16x2(r0, r1), max_bf16x2(r2, r3));
    x[0] = bf16lo(r0); x[1] = bf16hi(r0);
    x[2] = bf16lo(r1); x[3] = bf16hi(r1);
    x[4] = bf16lo(r2); x[5] = bf16hi(r2);
    x[6] = bf16lo(r3); x[7] = bf16hi(r3);
    return max_bf16x2(mx, lz.x2) != lz.x2;
  } else {
    if constexpr (kVec) {
      x[0] = b.a.x; x[1] = b.a.y; x[2] = b.a.z; x[3] = b.a.w;
      x[4] = b.b.x; x[5] = b.b.y; x[6] = b.b.z; x[7] = b.b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = b.v[i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = fmaxf(x[i], kFloorLogit);
    const float mx = fmaxf(fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3])),
                           fmaxf(fmaxf(x[4], x[5]), fmaxf(x[6], x[7])));
    return mx > lz.x;
  }
}

// Exponential-race prune: the score z - ln E (E = -ln U) can beat best_w
// only if E < e^(z - best_w); since E >= 1 - U, an entry with
// 1 - U >= e^(z - best_w) (1 + 2^-8) = p Kp is skipped without a logarithm.
// With U' = 1 + (x >> 9) 2^-23 = U + 1 - 2^-24 an entry stays a candidate
// when U' > 2 - 2^-23 - p Kp (the constant rounded down to an fp32 value,
// which only adds candidates).
constexpr float kPadD = -1000.0f;  // d of padding entries: 2^d flushes to 0

__device__ __forceinline__ float u_prime(uint32_t w) {
  return __uint_as_float(0x3F800000u | (w >> 9));
}
constexpr float kTwoMinus = 1.99999988079071044921875f;  // 2 - 2^-23

__device__ __forceinline__ uint32_t word_of(const uint4& wa, const uint4& wb, int i) {
  const uint4 wq = i < 4 ? wa : wb;
  const int i4 = i & 3;
  return i4 == 0 ? wq.x : i4 == 1 ? wq.y : i4 == 2 ? wq.z : wq.w;
}

// Per-warp scan state of one chunk.
struct PartState {
  Run st;
  float best_w;  // best Gumbel score of the row known to this warp
  float Kp;      // prune factor for this lane's reference m
};

// Exact scores of the item's candidates (rare).  The test is redone entry
// by entry from re-read logits (L1 hits) exactly as in scan_item, so the
// same entries qualify; only those get logarithms.  Arguments and results
// travel by value, so the caller's state stays in registers.
struct ExactOut {
  float best;
  int idx;
  bool changed;
};

template <typename T, bool kVec, bool kTail>
__device__ __noinline__ ExactOut exact_scores(const T* __restrict__ rowp, int v0, uint4 wa,
                                              uint4 wb, float m, float Kp, float best, int idx,
                                              float c2, float inv_tau, int vocab) {
  ItemBuf<T, kVec> rb;
  load_item<T, kVec>(rb, rowp, v0, vocab);
  LazyTest<T, kVec> none;
  none.set(-INFINITY, 1.f);
  float x[8];
  (void)unpack_item<T, kVec>(rb, none, x);
  uint32_t cmask = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float d = fmaf(x[i], c2, -m);
    if (kTail && v0 + i >= vocab) d = kPadD;
    const float pw = ex2_approx(d);
    if (u_prime(word_of(wa, wb, i)) > fmaf(pw, -Kp, kTwoMinus)) cmask |= 1u << i;
  }
  ExactOut o{best, idx, false};
  while (cmask) {
    const int i = __ffs(cmask) - 1;
    cmask &= cmask - 1;
    const uint32_t v = (uint32_t)(v0 + i);
    const float xi = fmaxf((float)rowp[v], kFloorLogit);
    const float sc = gumbel_score(xi * inv_tau, word_of(wa, wb, i));
    if (sc > o.best || (sc == o.best && (int)v < o.idx)) {
      o.best = sc;
      o.idx = (int)v;
      o.changed = true;
    }
  }
  return o;
}

// One item, in an order that keeps few values live: the Philox words, the
// lazy-reference raise (rare, one warp vote), then weights, softmax sums and
// the candidate test in one sweep, and the exact scores of candidates (rare,
// one warp vote), whose improvements go to the row key.  `next` (or nullptr)
// is the lane's address of the item two ahead, loaded into `buf` once this
// item is unpacked.  kTail: the item reaches past V.
template <typename T, bool kVec, bool kTail>
__device__ __forceinline__ void scan_item(PartState& ps, LazyTest<T, kVec>& lz,
                                          ItemBuf<T, kVec>& buf, const T* next,
                                          const T* __restrict__ rowp, int v0,
                                          const ScanParams& p, const PhiloxRow& prow,
                                          unsigned long long* rkey) {
  const uint32_t cword = (uint32_t)v0 >> 2;
  const uint4 wa = philox4x32_10_row(cword, 0u, prow, p.key);
  const uint4 wb = philox4x32_10_row(cword + 1u, 0u, prow, p.key);
  float x[8];
  const bool pend = unpack_item<T, kVec>(buf, lz, x);
  if (next != nullptr) load_item<T, kVec>(buf, next, 0, 1 << 30);
  if (__any_sync(0xffffffffu, pend)) {
    if (pend) {
      float bm = x[0];
#pragma unroll
      for (int i = 1; i < 8; ++i) bm = fmaxf(bm, x[i]);
      raise_ref(ps.st, fmaxf(bm * p.c2, ps.st.m));
      ps.Kp = prune_factor(ps.st.m, ps.best_w);
      lz.set(ps.st.m, p.inv_c2);
    }
  }
  const float2 c22 = make_float2(p.c2, p.c2);
  const float2 nm = make_float2(-ps.st.m, -ps.st.m);
  float pmax = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float2 d = __ffma2_rn(make_float2(x[2 * j], x[2 * j + 1]), c22, nm);
    if constexpr (kTail) {
      if (v0 + 2 * j >= p.vocab) d.x = kPadD;
      if (v0 + 2 * j + 1 >= p.vocab) d.y = kPadD;
    }
    const float2 pw = make_float2(ex2_approx(d.x), ex2_approx(d.y));
    ps.st.s2 = __fadd2_rn(ps.st.s2, pw);
    ps.st.t2 = __ffma2_rn(pw, d, ps.st.t2);
    pmax = fmaxf(pmax, fmaxf(pw.x, pw.y));
  }
  // One test for the lane's 8 entries: an entry i is a candidate only if
  // U'_i > 2 - 2^-23 - p_i Kp, which implies max U' > 2 - 2^-23 - max p Kp
  // (fma is monotone in p), so the rare path below runs for every item that
  // holds a candidate and finds the candidates themselves entry by entry.
  const uint32_t wmax = __vimax3_u32(__vimax3_u32(wa.x, wa.y, wa.z),
                                     __vimax3_u32(wa.w, wb.x, wb.y), max(wb.z, wb.w));
  const bool cand = u_prime(wmax) > fmaf(pmax, -ps.Kp, kTwoMinus);
  if (__any_sync(0xffffffffu, cand)) {
    bool changed = false;
    if (cand) {
      const ExactOut o = exact_scores<T, kVec, kTail>(rowp, v0, wa, wb, ps.st.m, ps.Kp,
                                                      ps.st.best, ps.st.idx, p.c2, p.inv_tau,
                                                      p.vocab);
      ps.st.best = o.best;
      ps.st.idx = o.idx;
      changed = o.changed;
      if (changed) atomicMax(rkey, pack_key(o.best, o.idx));
    }
    if (__any_sync(0xffffffffu, changed)) {
      ps.best_w = fmaxf(ps.best_w, warp_max(ps.st.best));
      ps.Kp = prune_factor(ps.st.m, ps.best_w);
    }
  }
}

// Seed of a chunk that finds no score for its row yet: the exact score of
// each lane's largest entry in the chunk's first item (lowest index among
// equal values), published to the row key by the warp's best lane.  The
// reference m is still unset here; the first item always raises it, which
// recomputes Kp.
template <typename T, bool kVec>
__device__ __forceinline__ void seed_chunk(PartState& ps, const ItemBuf<T, kVec>& b, int v0,
                                           const ScanParams& p, const PhiloxRow& prow,
                                           unsigned long long* rkey) {
  LazyTest<T, kVec> none;
  none.set(-INFINITY, 1.f);
  float x[8];
  (void)unpack_item<T, kVec>(b, none, x);
  float bm = -INFINITY;
  int jm = -1;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (v0 + i < p.vocab && x[i] > bm) {
      bm = x[i];
      jm = i;
    }
  if (jm >= 0) {
    const uint32_t v = (uint32_t)(v0 + jm);
    const uint4 w = philox4x32_10_row(v >> 2, 0u, prow, p.key);
    const uint32_t i4 = v & 3u;
    const uint32_t wj = i4 == 0 ? w.x : i4 == 1 ? w.y : i4 == 2 ? w.z : w.w;
    ps.st.best = gumbel_score(bm * p.inv_tau, wj);
    ps.st.idx = (int)v;
  }
  ps.best_w = warp_max(ps.st.best);
  // the lowest lane holding the warp's best has the lowest index among them
  const unsigned hit = __ballot_sync(0xffffffffu, jm >= 0 && ps.st.best == ps.best_w);
  if (hit && (int)(threadIdx.x & 31) == __ffs(hit) - 1)
    atomicMax(rkey, pack_key(ps.st.best, ps.st.idx));
}

// Adopt the row's best score known grid-wide when it is higher (any score in
// the row bounds the row's maximum from below, whichever warp found it).
__device__ __forceinline__ void adopt_key(PartState& ps, unsigned long long k) {
  const float cb = key_score(k);
  if (cb > ps.best_w) {
    ps.best_w = cb;
    ps.Kp = prune_factor(ps.st.m, cb);
  }
}

// Where chunk g lies: row r, items ja .. jb-1, of which ja .. jm-1 are full
// (jm = jb - 1 when the chunk ends with the row's partial last item).
template <typename T>
struct ChunkPos {
  const T* rowp;
  uint32_t r;
  int ja, jm, jb;
};

// Tickets run over the chunks column by column (chunk 0 of every row, then
// chunk 1, ...), so the chunks of one row are spread over the whole pass and
// most of them start with a good threshold from the row key.
template <typename T>
__device__ __forceinline__ ChunkPos<T> chunk_pos(const T* __restrict__ logits,
                                                 const ScanParams& p, uint32_t g) {
  ChunkPos<T> c;
  const uint32_t cc = g / (uint32_t)p.rows;
  c.r = g - cc * (uint32_t)p.rows;
  c.ja = (int)cc * kChunk;
  c.jb = min(c.ja + kChunk, p.ipr);
  c.jm = (c.jb - 1 == p.jtail) ? c.jb - 1 : c.jb;
  c.rowp = logits + (int64_t)c.r * p.row_stride;
  return c;
}

// One chunk: its items with loads issued two items ahead; the partial last
// item of a row is peeled off and processed with the padding checks.  A and
// B arrive holding the chunk's first two items when `pre` says so, and
// `key` its row key.  When `cross`, the last two items' prefetches fetch the
// first two items of the next chunk `cn` instead, with its row key, which
// then come back in A, B and `key`; the next chunk starts at item nja of
// row nr.  Writes the chunk's softmax partials to recs[r * nck + chunk].
template <typename T, bool kVec>
__device__ __forceinline__ void scan_chunk(const T* __restrict__ logits, const ScanParams& p,
                                           uint32_t g, const ChunkPos<T>& c, int lane,
                                           ItemBuf<T, kVec>& A, ItemBuf<T, kVec>& B, bool pre,
                                           unsigned long long& key, bool cross, uint32_t nr,
                                           int nja, float4* __restrict__ recs,
                                           unsigned long long* __restrict__ row_key) {
  const int lo8 = lane * 8;
  const T* rowp = c.rowp;
  unsigned long long* rkey = row_key + (size_t)c.r * kKeyStride;
  if (!pre) {
    if (c.jm > c.ja) load_item<T, kVec>(A, rowp, c.ja * kItem + lo8, p.vocab);
    if (c.jm > c.ja + 1) load_item<T, kVec>(B, rowp, (c.ja + 1) * kItem + lo8, p.vocab);
    key = __ldcg(rkey);
  }
  const PhiloxRow prow = philox_row(p.row_offset + c.r, p.step, 0u, p.key);
  PartState ps;
  ps.st = Run{-INFINITY, make_float2(0.f, 0.f), make_float2(0.f, 0.f), -INFINITY, 0x7fffffff};
  ps.best_w = key_score(key);
  ps.Kp = 0.f;
  LazyTest<T, kVec> lz;
  lz.set(-INFINITY, p.inv_c2);
  if constexpr (kVec) {
    const int ja = c.ja, jm = c.jm;
    if (jm > ja) {
      if (ps.best_w == -INFINITY) seed_chunk<T, kVec>(ps, A, ja * kItem + lo8, p, prow, rkey);
      const T* base = rowp + ja * kItem + lo8;  // this lane's entries of item j
#pragma unroll 1
      for (int j = ja; j < jm; j += 2, base += 2 * kItem) {
        const T* na = base + 2 * kItem;
        if (j + 2 >= jm) {  // past this chunk: the next chunk's first items
          na = nullptr;
          if (cross) {
            na = logits + (int64_t)nr * p.row_stride + nja * kItem + lo8;
            key = __ldcg(row_key + (size_t)nr * kKeyStride);
          }
        }
        scan_item<T, kVec, false>(ps, lz, A, na, rowp, j * kItem + lo8, p, prow, rkey);
        if (j + 1 < jm)
          scan_item<T, kVec, false>(ps, lz, B, na == nullptr ? nullptr : na + kItem, rowp,
                                    (j + 1) * kItem + lo8, p, prow, rkey);
      }
    }
    if (jm < c.jb) {
      ItemBuf<T, kVec> X;
      load_item<T, kVec>(X, rowp, jm * kItem + lo8, p.vocab);
      if (ps.best_w == -INFINITY) seed_chunk<T, kVec>(ps, X, jm * kItem + lo8, p, prow, rkey);
      adopt_key(ps, __ldcg(rkey));
      scan_item<T, kVec, true>(ps, lz, X, nullptr, rowp, jm * kItem + lo8, p, prow, rkey);
    }
  } else {
#pragma unroll 1
    for (int j = c.ja; j < c.jb; ++j) {
      ItemBuf<T, kVec> X;
      load_item<T, kVec>(X, rowp, j * kItem + lo8, p.vocab);
      if (ps.best_w == -INFINITY) seed_chunk<T, kVec>(ps, X, j * kItem + lo8, p, prow, rkey);
      adopt_key(ps, __ldcg(rkey));
      scan_item<T, kVec, true>(ps, lz, X, nullptr, rowp, j * kItem + lo8, p, prow, rkey);
    }
  }
  // the chunk's softmax partials: common reference first, then the sums by
  // a fixed butterfly
  float M = ps.st.m;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float s = ps.st.s2.x + ps.st.s2.y, t = ps.st.t2.x + ps.st.t2.y;
  if (s > 0.f) {
    const float f = ex2_approx(ps.st.m - M);
    t = f * fmaf(s, ps.st.m - M, t);
    s *= f;
  } else {
    s = 0.f;
    t = 0.f;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, off);
    t += __shfl_xor_sync(0xffffffffu, t, off);
  }
  if (lane == 0) recs[(size_t)c.r * p.nck + (uint32_t)(c.ja / kChunk)] = make_float4(M, s, t, 0.f);
}

// Persistent: each warp takes chunk tickets until they run out.  Tickets are
// drawn one chunk ahead, and on the vector path the next chunk's first two
// items and its row key are in flight while the current chunk ends, so a
// chunk boundary costs no memory latency.  The hand-over needs an even
// number of full items in the current chunk (the items alternate between two
// buffers) and two full items at the start of the next; other chunks (rows
// whose item count is not a multiple of the chunk, partial last items) load
// their first items when they start.
template <typename T, bool kVec>
__global__ void __launch_bounds__(kScanThreads, 3)
    sample_scan_kernel(const T* __restrict__ logits, const __grid_constant__ ScanParams p,
                       float4* __restrict__ recs, unsigned long long* __restrict__ row_key,
                       uint32_t* __restrict__ ticket) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  uint32_t g = 0, gn_req = 0;
  if (lane == 0) {
    g = atomicAdd(ticket, 1u);
    gn_req = atomicAdd(ticket, 1u);
  }
  g = __shfl_sync(0xffffffffu, g, 0);
  ItemBuf<T, kVec> A, B;
  unsigned long long key = 0ull;
  bool pre = false;
  while (g < p.nchunks) {
    const uint32_t gn = __shfl_sync(0xffffffffu, gn_req, 0);  // drawn one chunk ago
    if (lane == 0) gn_req = atomicAdd(ticket, 1u);
    const ChunkPos<T> c = chunk_pos<T>(logits, p, g);
    const bool has_next = gn < p.nchunks;
    bool cross = false;
    uint32_t nr = 0;
    int nja = 0;
    if (kVec && has_next && ((c.jm - c.ja) % 2 == 0) && c.jm == c.jb) {
      const ChunkPos<T> cn = chunk_pos<T>(logits, p, gn);
      cross = cn.jm - cn.ja >= 2;
      nr = cn.r;
      nja = cn.ja;
    }
    scan_chunk<T, kVec>(logits, p, g, c, lane, A, B, pre, key, cross, nr, nja, recs, row_key);
    pre = cross;
    g = gn;
  }
}

// Merge of a row's chunk partials (in chunk order), the argmax from the row
// key, then the re-noise draw.  One warp per row.  Clears the ticket counter,
// the row key and the row's chunk records for the next call: a completed
// call leaves every byte of state and records it used at zero, so calls of
// other shapes that share the workspace (and lay these out differently)
// start from a clear state.  An argmax index outside the row (a state the
// caller did not clear) is replaced by 0 and latched as a bounds error.
template <typename T>
__global__ void __launch_bounds__(128)
    sample_merge_kernel(const T* __restrict__ logits, int64_t row_stride, int rows, int vocab,
                        int nck, float inv_tau, float rate, uint64_t seed, uint32_t step,
                        uint32_t row_offset, float4* __restrict__ recs,
                        unsigned long long* __restrict__ row_key, uint32_t* __restrict__ ticket,
                        int32_t* __restrict__ tokens, int32_t* __restrict__ pred,
                        float* __restrict__ conf, float* __restrict__ entropy,
                        uint8_t* __restrict__ renoised, uint32_t* __restrict__ err) {
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0u;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  SumState st{-INFINITY, 0.f, 0.f};
  for (int c = lane; c < nck; c += 32) {
    float4* rc = recs + (int64_t)row * nck + c;
    const float4 r = *rc;
    *rc = make_float4(0.f, 0.f, 0.f, 0.f);
    merge_sums(st, SumState{r.x, r.y, r.z});
  }
  warp_merge_sums(st);
  if (lane != 0) return;
  const unsigned long long key = row_key[(size_t)row * kKeyStride];
  row_key[(size_t)row * kKeyStride] = 0ull;
  int p = key ? key_index(key) : 0;
  if ((unsigned)p >= (unsigned)vocab) {
    p = 0;
    atomicOr(err, kDevErrBounds);
  }
  const float x = fmaxf((float)logits[(int64_t)row * row_stride + p], kFloorLogit);
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

// CTAs of the persistent scan grid on the current device (resident CTAs per
// SM x SMs), cached per device and variant.
template <typename T, bool kVec>
int scan_ctas() {
  constexpr int kMaxDev = 64;
  static std::atomic<int> cache[kMaxDev];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 1;
  if (dev < kMaxDev) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int sms = 0, occ = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, sample_scan_kernel<T, kVec>,
                                                    kScanThreads, 0) != cudaSuccess) {
    cudaGetLastError();
    sms = 1;
    occ = 1;
  }
  const int n = std::max(1, sms * std::max(occ, 1));
  if (dev < kMaxDev) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

int chunks_per_row(int vocab) {
  const int ipr = (vocab + kItem - 1) / kItem;
  return (ipr + kChunk - 1) / kChunk;
}

template <typename T, bool kVec>
cudaError_t launch_sampler_v(const SamplerArgs& a, cudaStream_t stream) {
  const T* lg = static_cast<const T*>(a.logits);
  ScanParams p;
  p.key = philox_key(a.seed);
  p.row_stride = a.row_stride;
  p.vocab = a.vocab;
  p.ipr = (a.vocab + kItem - 1) / kItem;
  p.nck = chunks_per_row(a.vocab);
  p.nchunks = (uint32_t)((uint64_t)a.rows * (uint64_t)p.nck);
  p.rows = a.rows;
  p.jtail = (a.vocab % kItem) ? p.ipr - 1 : -1;
  p.c2 = a.inv_tau * kLog2e;
  p.inv_c2 = 1.0f / p.c2;
  p.inv_tau = a.inv_tau;
  p.step = a.step;
  p.row_offset = a.row_offset;
  const SamplerState s = sampler_state(a.state);
  float4* recs = static_cast<float4*>(a.recs);
  const int64_t want = ((int64_t)p.nchunks + kScanWarpsPerCta - 1) / kScanWarpsPerCta;
  const int ctas = (int)std::min<int64_t>(scan_ctas<T, kVec>(), want);
  cudaError_t e = launch_pdl(sample_scan_kernel<T, kVec>, dim3(ctas), dim3(kScanThreads), 0,
                             stream, lg, p, recs, s.row_key, s.ticket);
  note_launch();
  if (e != cudaSuccess) return e;
  e = launch_pdl(sample_merge_kernel<T>, dim3((a.rows + 3) / 4), dim3(128), 0, stream, lg,
                 a.row_stride, a.rows, a.vocab, p.nck, a.inv_tau, a.rate, a.seed, a.step,
                 a.row_offset, recs, s.row_key, s.ticket, a.tokens, a.pred, a.conf, a.entropy,
                 a.renoised, a.err);
  note_launch();
  return e;
}

template <typename T>
cudaError_t launch_sampler_t(const SamplerArgs& a, cudaStream_t stream) {
  const size_t esz = sizeof(T);
  const bool vec = ((reinterpret_cast<uintptr_t>(a.logits) & 15u) == 0) &&
                   (((size_t)a.row_stride * esz) % 16 == 0) && (a.vocab % 8 == 0);
  return vec ? launch_sampler_v<T, true>(a, stream) : launch_sampler_v<T, false>(a, stream);
}

}  // namespace

size_t sampler_state_bytes(int rows) {
  return 256 + (size_t)rows * kKeyStride * sizeof(unsigned long long);
}

size_t sampler_record_bytes(int rows, int vocab) {
  return (size_t)rows * (size_t)chunks_per_row(vocab) * sizeof(float4);
}

SamplerState sampler_state(void* state) {
  SamplerState s;
  s.ticket = static_cast<uint32_t*>(state);
  s.row_key = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(state) + 256);
  return s;
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
