// dd_soft_embed.cu -- the self-conditioning soft embedding
//   out[r, :] = sum_v softmax(logits[r, :] / tau)_v * E[v, :]
// ("DiffusionGemma Technical Report", paperfeed review, "The mechanism",
// self-conditioning paragraph: the step's predicted token distribution,
// pushed through the embedding matrix, is the input of a small MLP that
// conditions the next step).
//
// A [rows x V] . [V x d] contraction with V = 262,144: at d = 2048 and 256
// rows, 275 GFLOP against 1.07 GB of E, right at the B200 ridge point.
// Three kernels:
//   row_lse_kernel      the log2-domain log-sum-exp of each row of
//                       logits * log2(e) / tau (one CTA per row, one pass);
//   soft_embed_kernel   split-K tcgen05 GEMM.  A CTA owns 256 rows (two
//                       128-row MMA tiles), 256 embedding columns and a range
//                       of the vocabulary.  Per 32-entry vocabulary step, TMA
//                       brings the logits tile and the E tile (a 4-deep
//                       ring); sixteen warps (two threads per row) turn the
//                       logits into probabilities 2^(z log2(e)/tau - lse)
//                       and write them as bf16 straight into the swizzled
//                       A-operand layout; one elected lane of the MMA warp
//                       multiplies them with E (B operand, MN-major) into
//                       fp32 accumulators in tensor memory (2 x 256
//                       columns).  Eight of those warps write the CTA's fp32
//                       partial at the end;
//   soft_embed_reduce   sums the partials of the vocabulary splits in a
//                       fixed order and rounds to bf16.
// Every mbarrier wait is bounded; on expiry the CTA latches an error word,
// drains its own asynchronous work and frees its tensor memory.
#include <algorithm>
#include <mutex>

#include "dd_device.cuh"
#include "dd_internal.h"

namespace dd {
namespace {

constexpr int SE_BM = 128;        // rows per MMA tile
constexpr int SE_MT = 2;          // MMA tiles per CTA
constexpr int SE_ROWS = SE_BM * SE_MT;
constexpr int SE_BK = 32;         // vocabulary entries per stage (64 bytes of bf16)
constexpr int SE_BN = 256;        // embedding columns per CTA
constexpr int SE_STAGES = 4;
#ifndef DD_SE_PWARPS
#define DD_SE_PWARPS 16
#endif
// probability warps: 8 (one thread per row) or 16 (two threads per row,
// 16 vocabulary entries each); the first 8 also run the epilogue
constexpr int SE_PWARPS = DD_SE_PWARPS;
static_assert(SE_PWARPS == 8 || SE_PWARPS == 16, "one or two threads per row");
constexpr int SE_WARP_TMA = 0, SE_WARP_MMA = 1, SE_WARP_P0 = 2;
constexpr int SE_THREADS = (SE_WARP_P0 + SE_PWARPS) * 32;
constexpr uint32_t SE_LTILE = SE_ROWS * SE_BK * 2;  // logits tile, 16 KB (64-byte rows)
constexpr uint32_t SE_PHALF = SE_BM * SE_BK * 2;    // one 128-row P tile, 8 KB
constexpr uint32_t SE_PTILE = SE_MT * SE_PHALF;     // 16 KB
constexpr uint32_t SE_EBOX = SE_BK * 64 * 2;        // 32 vocabulary rows x 64 columns, 4 KB
constexpr uint32_t SE_ETILE = (SE_BN / 64) * SE_EBOX;  // 16 KB
constexpr uint32_t SE_STAGE = SE_LTILE + SE_PTILE + SE_ETILE;
constexpr uint32_t SE_OFF_BAR = SE_STAGES * SE_STAGE;
constexpr uint64_t SE_WAIT_NS = 1000000000ull;

struct SeBars {
  uint64_t full[SE_STAGES], pfull[SE_STAGES], empty[SE_STAGES];
  uint64_t acc_full, mma_final;
  uint64_t never;  // completed by nothing: the target of the test stall
  uint32_t tmem_base;
  int abort;
};
constexpr uint32_t SE_SMEM = SE_OFF_BAR + sizeof(SeBars) + 1024;
static_assert(SE_SMEM <= 232448, "shared memory budget");

struct SeParams {
  int rows, vocab, d;
  int ksteps, ksteps_per_split, splits;
  float c_log2;          // log2(e) / tau
  const float* lse2;     // [rows] log2-domain log-sum-exp of logits * c_log2
  float* part;           // [splits][rows][d] fp32
  uint32_t* err;
  uint64_t wait_ns;      // limit of each pipeline wait (waits that drain use SE_WAIT_NS)
  int stall;             // test stall: one wait on `never` once the first MMAs are issued
};

// ---------------------------------------------------------------- row LSE
// Running (max, sum) pair: s = sum 2^(t - m) over the values seen so far.
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;  // both empty
  s = s * ex2_approx(m - mn) + s2 * ex2_approx(m2 - mn);
  m = mn;
}

// lse2[r] = log2 sum_v 2^(z_v c), c = log2(e) / tau: one pass over the row.
// Each thread loads four 16-byte vectors at a time (32 entries, all four
// requests in flight before the arithmetic), keeps a running maximum m and
// the sum of 2^(t - m), rescaled once per 32 entries when m grows; the
// pairs are merged across the CTA.
constexpr int LSE_THREADS = 512;
__device__ __forceinline__ void lse_vec8(uint4 w, float c, float (&t)[8]) {
  const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t[2 * k] = bf16lo(ww[k]) * c;
    t[2 * k + 1] = bf16hi(ww[k]) * c;
  }
}

template <int U>
__device__ __forceinline__ void lse_block(const uint4 (&w)[U], float c, float& m, float& s) {
  float t[U][8];
  float mx = -INFINITY;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    lse_vec8(w[u], c, t[u]);
#pragma unroll
    for (int k = 0; k < 8; ++k) mx = fmaxf(mx, t[u][k]);
  }
  const float mn = fmaxf(m, mx);
  if (mn == -INFINITY) return;
  float acc = (m == mn) ? s : s * ex2_approx(m - mn);
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc += ex2_approx(t[u][k] - mn);
  s = acc;
  m = mn;
}

__global__ void __launch_bounds__(LSE_THREADS)
    row_lse_kernel(const __nv_bfloat16* __restrict__ logits, int64_t row_stride, int vocab,
                   float c, float* __restrict__ lse2) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red_m[LSE_THREADS / 32], red_s[LSE_THREADS / 32];
  const int r = blockIdx.x;
  const __nv_bfloat16* row = logits + (int64_t)r * row_stride;
  const uint4* rv = reinterpret_cast<const uint4*>(row);
  const int nvec = vocab / 8;
  constexpr int U = 4;
  float m = -INFINITY, s = 0.f;
  int i = threadIdx.x;
  for (; i + (U - 1) * LSE_THREADS < nvec; i += U * LSE_THREADS) {
    uint4 w[U];
#pragma unroll
    for (int u = 0; u < U; ++u) w[u] = __ldcs(rv + i + u * LSE_THREADS);
    lse_block<U>(w, c, m, s);
  }
  for (; i < nvec; i += LSE_THREADS) {
    const uint4 w[1] = {__ldcs(rv + i)};
    lse_block<1>(w, c, m, s);
  }
  for (int v = nvec * 8 + threadIdx.x; v < vocab; v += LSE_THREADS)
    lse_merge(m, s, __bfloat162float(row[v]) * c, 1.f);
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse_merge(m, s, m2, s2);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    red_m[warp] = m;
    red_s[warp] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float mm = red_m[0], ss = red_s[0];
    for (int k = 1; k < LSE_THREADS / 32; ++k) lse_merge(mm, ss, red_m[k], red_s[k]);
    lse2[r] = mm + __log2f(ss);
  }
}

// The 16-byte chunk c of row r of a tile with 64-byte rows and 64-byte
// swizzling (the layout TMA writes and the MMA reads): c ^ ((r >> 1) & 3).
__device__ __forceinline__ uint32_t sw64_off(int r, int c) {
  return (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

// One probability row chunk: 8 logits (16 bytes) -> 8 bf16 probabilities
// 2^(z c - lse).  Entries at or past `vocab` (the last step of the
// vocabulary; TMA fills them with zeros) are masked only when `tail`.
template <bool kTail>
__device__ __forceinline__ uint4 probs8(uint4 raw, float2 c2, float2 nl2, int v0, int vocab) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __ffma2_rn(make_float2(bf16lo(w[i]), bf16hi(w[i])), c2, nl2);
    float a = ex2_approx(t.x), b = ex2_approx(t.y);
    if constexpr (kTail) {
      const int v = v0 + 2 * i;
      if (v >= vocab) a = 0.f;
      if (v + 1 >= vocab) b = 0.f;
    }
    o[i] = pack_bf16x2(a, b);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__global__ void __launch_bounds__(SE_THREADS, 1)
    soft_embed_kernel(const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmE,
                      const SeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  SeBars* bars = reinterpret_cast<SeBars*>(smem + SE_OFF_BAR);
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort;
  const int n0 = blockIdx.x * SE_BN;
  const int split = blockIdx.y;
  const int row0 = blockIdx.z * SE_ROWS;
  const int ks0 = split * p.ksteps_per_split;
  const int nk = max(0, min(p.ksteps, ks0 + p.ksteps_per_split) - ks0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SE_STAGES; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->pfull[s], SE_PWARPS);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->mma_final, 1);
    mbar_init(&bars->never, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == SE_WARP_MMA) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == SE_WARP_TMA) {
    if (lane == 0 && nk > 0) {
      prefetch_tensormap(&tmL);
      prefetch_tensormap(&tmE);
      // E boxes wholly right of column d are not loaded (their columns
      // are never written out)
      const int nbox = min(SE_BN / 64, (p.d - n0) / 64);
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int s = i % SE_STAGES, rd = i / SE_STAGES;
        if (rd > 0 && !mbar_wait_bounded(&bars->empty[s], (rd - 1) & 1, abort_flag, p.wait_ns))
          break;
        uint8_t* st = smem + s * SE_STAGE;
        const int v0 = (ks0 + i) * SE_BK;
        mbar_arrive_expect_tx(&bars->full[s], SE_LTILE + nbox * SE_EBOX);
        tma_load_2d(st, &tmL, &bars->full[s], v0, row0);
        for (int b = 0; b < nbox; ++b)
          tma_load_2d(st + SE_LTILE + SE_PTILE + b * SE_EBOX, &tmE, &bars->full[s], n0 + 64 * b,
                      v0);
        issued = i + 1;
      }
      // drain: loads in flight must land before the CTA exits
      for (int i = max(0, issued - SE_STAGES); i < issued; ++i)
        mbar_wait_bounded(&bars->full[i % SE_STAGES], (i / SE_STAGES) & 1, nullptr, SE_WAIT_NS);
    }
    __syncwarp();
  } else if (warp == SE_WARP_MMA) {
    if (nk > 0) {
      // converged warp: uniform operands, one elected lane issues
      const bool leader = elect_one_sync();
      // P: K-major, 64-byte rows with 64-byte swizzling (8-row groups 512
      // bytes apart); E: MN-major, 128-byte swizzling, 64-column boxes 4 KB
      // apart along N, 8-row groups 1 KB apart along K
      const uint64_t dP = smem_desc_sw64(smem_u32(smem + SE_LTILE), 16, 512);
      const uint64_t dE = smem_desc_sw128(smem_u32(smem + SE_LTILE + SE_PTILE), SE_EBOX, 1024);
      constexpr uint32_t idesc = idesc_bf16_f32(SE_BM, SE_BN, 0, 1);
      bool ok = true;
      for (int i = 0; ok && i < nk; ++i) {
        const int s = i % SE_STAGES;
        const uint32_t ph = (i / SE_STAGES) & 1;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->full[s], ph, abort_flag, p.wait_ns) &&
                                         mbar_wait_bounded(&bars->pfull[s], ph, abort_flag, p.wait_ns));
        if (!ok) break;
        tc_fence_after();
        const uint32_t so = s * SE_STAGE;
        if (leader) {
#pragma unroll
          for (int mt = 0; mt < SE_MT; ++mt)
#pragma unroll
            for (int kk = 0; kk < SE_BK / 16; ++kk)
              tc_mma_ss(tmem + (uint32_t)(mt * SE_BN), dP + ((so + mt * SE_PHALF + kk * 32) >> 4),
                        dE + ((so + kk * 16 * 128) >> 4), idesc, (i > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&bars->empty[s]);
        }
        __syncwarp();
        // test stall: a wait nothing completes, with the first MMAs in flight
        if (i == 0 && p.stall)
          ok = __all_sync(0xffffffffu,
                          mbar_wait_bounded(&bars->never, 0, abort_flag, p.wait_ns));
      }
      if (leader) {
        if (ok) tc_commit(&bars->acc_full);
        // every MMA issued above has completed before tensor memory is freed
        tc_commit(&bars->mma_final);
      }
      __syncwarp();
      mbar_wait_bounded(&bars->mma_final, 0, nullptr, SE_WAIT_NS);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- probabilities, epilogue
    const int tid = threadIdx.x - SE_WARP_P0 * 32;
    const int t = tid % SE_ROWS;                   // row within the CTA
    constexpr int kChunks = SE_BK / 8 / (SE_PWARPS / 8);  // 16-byte chunks per thread
    const int j0 = (tid / SE_ROWS) * kChunks;
    const int r = row0 + t;
    // rows past the end: TMA reads them as zeros, and lse = +inf makes
    // their probabilities 0
    const float lse = r < p.rows ? p.lse2[r] : INFINITY;
    const float2 c2 = make_float2(p.c_log2, p.c_log2), nl2 = make_float2(-lse, -lse);
    const int mt = t / SE_BM, rr = t % SE_BM;
    bool ok = true;
    for (int i = 0; i < nk; ++i) {
      const int s = i % SE_STAGES;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars->full[s], (i / SE_STAGES) & 1,
                                                     abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      const uint8_t* lt = smem + s * SE_STAGE;  // logits rows, 64-byte swizzle
      uint8_t* pt = smem + s * SE_STAGE + SE_LTILE + mt * SE_PHALF;
      const int v0 = (ks0 + i) * SE_BK;
      if (v0 + SE_BK <= p.vocab) {
#pragma unroll
        for (int j = j0; j < j0 + kChunks; ++j) {
          const uint4 raw = *reinterpret_cast<const uint4*>(lt + sw64_off(t, j));
          *reinterpret_cast<uint4*>(pt + sw64_off(rr, j)) =
              probs8<false>(raw, c2, nl2, v0 + 8 * j, p.vocab);
        }
      } else {
        for (int j = j0; j < j0 + kChunks; ++j) {
          const uint4 raw = *reinterpret_cast<const uint4*>(lt + sw64_off(t, j));
          *reinterpret_cast<uint4*>(pt + sw64_off(rr, j)) =
              probs8<true>(raw, c2, nl2, v0 + 8 * j, p.vocab);
        }
      }
      fence_proxy_async_smem();  // generic-proxy stores -> the MMA's reads
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->pfull[s]);
    }
    const bool epilogue = warp < SE_WARP_P0 + 8;
    if (ok && nk > 0 && epilogue)
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->acc_full, 0, abort_flag, p.wait_ns));
    if (ok && nk > 0 && epilogue) {
      tc_fence_after();
      // TMEM lanes of this warp: 32 * (warp % 4); warps 2-5 hold tile 0,
      // 6-9 tile 1, so (mt, rr) above is this thread's lane
      const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
      const int rrow = mt * SE_BM + 32 * (warp & 3) + lane;
      const int gr = row0 + rrow;
      float* dst = p.part + ((size_t)split * p.rows + gr) * p.d + n0;
      const int ncols = min(SE_BN, p.d - n0);
#pragma unroll 1
      for (int c0 = 0; c0 < SE_BN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(mt * SE_BN + c0), v);
        if (gr < p.rows && c0 < ncols) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(dst + c0 + c) =
                make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                            __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
        }
      }
    }
  }

  if (*abort_flag && threadIdx.x == 0) atomicOr(p.err, kDevErrTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == SE_WARP_MMA) tmem_dealloc(tmem, 512);
}

// out[r, c] = bf16(sum over splits, in split order, of part[s][r][c]).
__global__ void __launch_bounds__(256)
    soft_embed_reduce(const float* __restrict__ part, int splits, int rows, int d,
                      __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int64_t n4 = (int64_t)rows * d / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 a = reinterpret_cast<const float4*>(part)[i];
    for (int s = 1; s < splits; ++s) {
      const float4 b = reinterpret_cast<const float4*>(part + (size_t)s * rows * d)[i];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    uint2 o;
    o.x = pack_bf16x2(a.x, a.y);
    o.y = pack_bf16x2(a.z, a.w);
    reinterpret_cast<uint2*>(out)[i] = o;
  }
}

// ----------------------------------------------------------------- host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

int sm_count_se() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

// 2-D bf16 map over [outer, inner] with a row stride in elements, box
// (box_inner, box_outer), box_inner * 2 bytes of swizzling (64 or 128),
// zero fill out of bounds.
bool encode_2d(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t stride,
               int box_inner, int box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  const cuuint64_t strides[1] = {(cuuint64_t)stride * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw =
      box_inner * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Vocabulary splits: about one wave of CTAs over the SMs, at least 16 steps
// of 32 entries per split.
SoftEmbedPlan soft_embed_plan(int rows, int vocab, int d) {
  SoftEmbedPlan pl{};
  pl.ksteps = (vocab + SE_BK - 1) / SE_BK;
  const int ntiles = (d + SE_BN - 1) / SE_BN;
  const int rblocks = (rows + SE_ROWS - 1) / SE_ROWS;
  const int base = ntiles * rblocks;
  int splits = std::max(1, sm_count_se() / std::max(1, base));
  splits = std::min(splits, std::max(1, pl.ksteps / 16));
  pl.ksteps_per_split = (pl.ksteps + splits - 1) / splits;
  pl.splits = (pl.ksteps + pl.ksteps_per_split - 1) / pl.ksteps_per_split;
  pl.grid_x = ntiles;
  pl.grid_z = rblocks;
  return pl;
}

size_t soft_embed_scratch_bytes(int rows, int vocab, int d) {
  const SoftEmbedPlan pl = soft_embed_plan(rows, vocab, d);
  const size_t lse = ((size_t)rows * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return lse + (size_t)pl.splits * rows * d * sizeof(float);
}

cudaError_t launch_soft_embed(const SoftEmbedArgs& a, cudaStream_t stream) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(soft_embed_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)SE_SMEM);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const SoftEmbedPlan pl = soft_embed_plan(a.rows, a.vocab, a.d);
  uint8_t* scratch = static_cast<uint8_t*>(a.scratch);
  float* lse2 = reinterpret_cast<float*>(scratch);
  float* part = reinterpret_cast<float*>(
      scratch + (((size_t)a.rows * sizeof(float) + 255) & ~static_cast<size_t>(255)));
  const float c = (float)(1.4426950408889634 / (double)a.temperature);

  cudaError_t e = launch_pdl(row_lse_kernel, dim3(a.rows), dim3(LSE_THREADS), 0, stream,
                             static_cast<const __nv_bfloat16*>(a.logits), a.row_stride, a.vocab,
                             c, lse2);
  note_launch();
  if (e != cudaSuccess) return e;

  CUtensorMap mL, mE;
  if (!encode_2d(&mL, a.logits, a.vocab, a.rows, a.row_stride, SE_BK, SE_ROWS) ||
      !encode_2d(&mE, a.emb, a.d, a.vocab, a.d, 64, SE_BK))
    return cudaErrorInvalidValue;
  SeParams p;
  p.rows = a.rows;
  p.vocab = a.vocab;
  p.d = a.d;
  p.ksteps = pl.ksteps;
  p.ksteps_per_split = pl.ksteps_per_split;
  p.splits = pl.splits;
  p.c_log2 = c;
  p.lse2 = lse2;
  p.part = part;
  p.err = a.err;
  p.wait_ns = pipeline_wait_ns();
  p.stall = pipeline_test_stall() ? 1 : 0;
  e = launch_pdl(soft_embed_kernel, dim3(pl.grid_x, pl.splits, pl.grid_z), dim3(SE_THREADS),
                 SE_SMEM, stream, mL, mE, p);
  note_launch();
  if (e != cudaSuccess) return e;
  const int64_t n4 = (int64_t)a.rows * a.d / 4;
  const int blocks = (int)std::min<int64_t>((n4 + 255) / 256, 4 * sm_count_se());
  e = launch_pdl(soft_embed_reduce, dim3(blocks), dim3(256), 0, stream, (const float*)part,
                 pl.splits, a.rows, a.d, static_cast<__nv_bfloat16*>(a.out));
  note_launch();
  return e;
}

}  // namespace dd
