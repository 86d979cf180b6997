// dd_ffw.cu -- the self-conditioning MLP ("DiffusionGemma Technical Report",
// paperfeed review, "The mechanism", self-conditioning paragraph: the
// previous step's predicted distribution, pushed through the embedding
// matrix, goes through a small MLP of 7.8M parameters, z_t = FFW(p0 E)).
//
// The MLP is two dense layers:
//   hid = GELU(u W1 + b1)    [rows, h]
//   z   = hid W2 + b2        [rows, d]
// Each layer is dense_kernel: a CTA computes a 128-row x 128-column tile
// over a range of K.  One warp issues TMA loads of the x tile (K-major,
// 128-byte swizzle) and the weight tile (N-major, two 64-column boxes) into
// a 6-deep ring, one elected lane of a second warp issues the tcgen05 MMAs
// (M = 128, N = 128, K = 16 each) into 128 fp32 columns of tensor memory,
// and four warps read them back (one TMEM lane quarter each).  K and N
// tails come in as TMA zero fill.
// At 256 rows a layer has only 30-32 output tiles, so K is split over up to
// four CTAs per tile to fill the SMs: the splits write fp32 partials and
// dense_finish adds them in split order (the result does not depend on
// scheduling), adds the bias, applies the activation and rounds to bf16.
// With enough tiles (2048 rows) there is one split and the GEMM's own
// epilogue does that.
// Every mbarrier wait is bounded; on expiry the CTA latches an error word,
// drains its asynchronous work and frees its tensor memory.
#include <algorithm>
#include <mutex>

#include "dd_device.cuh"
#include "dd_internal.h"

namespace dd {
namespace {

constexpr int FF_BM = 128;  // rows per tile (one MMA)
constexpr int FF_BN = 128;  // output columns per tile (two 64-column weight boxes)
constexpr int FF_BK = 64;   // K per stage: one 128-byte swizzle row of bf16
constexpr int FF_STAGES = 6;
constexpr int FF_WARP_TMA = 0, FF_WARP_MMA = 1, FF_WARP_EPI = 2;
constexpr int FF_THREADS = (FF_WARP_EPI + 4) * 32;
constexpr uint32_t FF_ATILE = FF_BM * FF_BK * 2;  // 16 KB
constexpr uint32_t FF_BBOX = FF_BK * 64 * 2;      // 64 K rows x 64 columns, 8 KB
constexpr uint32_t FF_BTILE = 2 * FF_BBOX;          // 16 KB
constexpr uint32_t FF_STAGE = FF_ATILE + FF_BTILE;
constexpr uint32_t FF_OFF_BAR = FF_STAGES * FF_STAGE;
constexpr uint32_t FF_TMEM_COLS = FF_BN;
constexpr uint64_t FF_WAIT_NS = 1000000000ull;

struct FfBars {
  uint64_t full[FF_STAGES], empty[FF_STAGES];
  uint64_t acc_full, mma_final;
  uint64_t never;  // completed by nothing: the target of the test stall
  uint32_t tmem_base;
  int abort;
};
constexpr uint32_t FF_SMEM = FF_OFF_BAR + sizeof(FfBars) + 1024;
static_assert(FF_SMEM <= 232448, "shared memory budget");

struct FfParams {
  int rows, K, N;
  int ksteps_per_split, splits;
  const __nv_bfloat16* bias;
  __nv_bfloat16* out;  // splits == 1: the finished bf16 output
  float* part;         // splits > 1: fp32 partials [splits][rows][N]
  uint32_t* err;
  uint64_t wait_ns;    // limit of each pipeline wait (waits that drain use FF_WAIT_NS)
  int stall;           // test stall: one wait on `never` once the first MMAs are issued
};

// GELU(x) = x * Phi(x), Phi the standard normal distribution function.
__device__ __forceinline__ float gelu(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}

template <bool kGelu>
__global__ void __launch_bounds__(FF_THREADS)
    dense_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const FfParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  FfBars* bars = reinterpret_cast<FfBars*>(smem + FF_OFF_BAR);
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort;
  const int n0 = blockIdx.x * FF_BN, m0 = blockIdx.y * FF_BM, split = blockIdx.z;
  const int ksteps = (p.K + FF_BK - 1) / FF_BK;
  const int k0 = split * p.ksteps_per_split;
  const int nk = max(0, min(ksteps, k0 + p.ksteps_per_split) - k0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < FF_STAGES; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->mma_final, 1);
    mbar_init(&bars->never, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == FF_WARP_MMA) {
    tmem_alloc(&bars->tmem_base, FF_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == FF_WARP_TMA) {
    if (lane == 0) {
      prefetch_tensormap(&tmX);
      prefetch_tensormap(&tmW);
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int s = i % FF_STAGES, rd = i / FF_STAGES;
        if (rd > 0 && !mbar_wait_bounded(&bars->empty[s], (rd - 1) & 1, abort_flag, p.wait_ns))
          break;
        uint8_t* st = smem + s * FF_STAGE;
        mbar_arrive_expect_tx(&bars->full[s], FF_STAGE);
        const int kc = (k0 + i) * FF_BK;
        tma_load_2d(st, &tmX, &bars->full[s], kc, m0);
        tma_load_2d(st + FF_ATILE, &tmW, &bars->full[s], n0, kc);
        tma_load_2d(st + FF_ATILE + FF_BBOX, &tmW, &bars->full[s], n0 + 64, kc);
        issued = i + 1;
      }
      // drain: loads in flight must land before the CTA exits
      for (int i = max(0, issued - FF_STAGES); i < issued; ++i)
        mbar_wait_bounded(&bars->full[i % FF_STAGES], (i / FF_STAGES) & 1, nullptr, FF_WAIT_NS);
    }
    __syncwarp();
  } else if (warp == FF_WARP_MMA) {
    const bool leader = elect_one_sync();
    // x: K-major, 128-byte rows, 8-row groups 1 KB apart, K = 16 steps of
    // 32 bytes along the swizzled row; W: N-major, two 64-column boxes 8 KB
    // apart along N, K rows of 128 bytes, 8-row groups 1 KB apart, K = 16
    // steps of 2 KB
    const uint64_t dX = smem_desc_sw128(smem_u32(smem), 16, 1024);
    const uint64_t dW = smem_desc_sw128(smem_u32(smem + FF_ATILE), FF_BBOX, 1024);
    constexpr uint32_t idesc = idesc_bf16_f32(FF_BM, FF_BN, 0, 1);
    bool ok = true;
    for (int i = 0; i < nk; ++i) {
      const int s = i % FF_STAGES;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->full[s], (i / FF_STAGES) & 1,
                                                     abort_flag, p.wait_ns));
      if (!ok) break;
      tc_fence_after();
      const uint32_t so = s * FF_STAGE;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < FF_BK / 16; ++kk)
          tc_mma_ss(tmem, dX + ((so + kk * 32) >> 4), dW + ((so + kk * 16 * 128) >> 4), idesc,
                    (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&bars->empty[s]);
      }
      __syncwarp();
      // test stall: a wait nothing completes, with the first MMAs in flight
      if (i == 0 && p.stall) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars->never, 0, abort_flag, p.wait_ns));
        if (!ok) break;
      }
    }
    if (leader) {
      if (ok) tc_commit(&bars->acc_full);
      // every MMA issued above has completed before tensor memory is freed
      tc_commit(&bars->mma_final);
    }
    __syncwarp();
    mbar_wait_bounded(&bars->mma_final, 0, nullptr, FF_WAIT_NS);
  } else {
    // epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31, i.e. tile rows
    const bool ok = nk > 0 && __all_sync(0xffffffffu, mbar_wait_bounded(&bars->acc_full, 0,
                                                                         abort_flag, p.wait_ns));
    if (ok) {
      tc_fence_after();
      const int q = warp & 3;
      const int row = m0 + 32 * q + lane;
#pragma unroll 1
      for (int h = 0; h < FF_BN / 64; ++h) {
        uint32_t v[64];
        tmem_ld64(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(h * 64), v);
        const int nb = n0 + h * 64;
        if (row < p.rows) {
          if (p.splits == 1) {
            __nv_bfloat16* dst = p.out + (size_t)row * p.N + nb;
#pragma unroll
            for (int c = 0; c < 64; c += 8) {
              if (nb + c < p.N) {
                const uint4 braw = *reinterpret_cast<const uint4*>(p.bias + nb + c);
                const uint32_t bw[4] = {braw.x, braw.y, braw.z, braw.w};
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  float a = __uint_as_float(v[c + 2 * j]) + bf16lo(bw[j]);
                  float b = __uint_as_float(v[c + 2 * j + 1]) + bf16hi(bw[j]);
                  if constexpr (kGelu) {
                    a = gelu(a);
                    b = gelu(b);
                  }
                  o[j] = pack_bf16x2(a, b);
                }
                *reinterpret_cast<uint4*>(dst + c) = make_uint4(o[0], o[1], o[2], o[3]);
              }
            }
          } else {
            float* dst = p.part + ((size_t)split * p.rows + row) * p.N + nb;
#pragma unroll
            for (int c = 0; c < 64; c += 4)
              if (nb + c < p.N)
                *reinterpret_cast<float4*>(dst + c) =
                    make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                                __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
          }
        }
      }
    }
  }

  if (*abort_flag && threadIdx.x == 0) atomicOr(p.err, kDevErrTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == FF_WARP_MMA) tmem_dealloc(tmem, FF_TMEM_COLS);
}

constexpr int FF_MAX_SPLITS = 8;

// out[r, n] = act(bias[n] + sum over splits, in split order, of
// part[s][r][n]), rounded to bf16; 8 columns per thread.  Every split's
// values are requested before the first is added (one memory round trip).
template <bool kGelu>
__global__ void __launch_bounds__(256)
    dense_finish(const float* __restrict__ part, int splits, int rows, int N,
                 const __nv_bfloat16* __restrict__ bias, __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int n8 = N / 8;
  const int64_t total = (int64_t)rows * n8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / n8;
    const int c = (int)(i - r * n8) * 8;
    const float* src = part + r * N + c;
    float4 x[FF_MAX_SPLITS], y[FF_MAX_SPLITS];
#pragma unroll
    for (int s = 0; s < FF_MAX_SPLITS; ++s) {
      if (s < splits) {
        const float* q = src + (size_t)s * rows * N;
        x[s] = *reinterpret_cast<const float4*>(q);
        y[s] = *reinterpret_cast<const float4*>(q + 4);
      }
    }
    const uint4 braw = *reinterpret_cast<const uint4*>(bias + c);
    float4 a = x[0], b = y[0];
#pragma unroll
    for (int s = 1; s < FF_MAX_SPLITS; ++s) {
      if (s < splits) {
        a.x += x[s].x; a.y += x[s].y; a.z += x[s].z; a.w += x[s].w;
        b.x += y[s].x; b.y += y[s].y; b.z += y[s].z; b.w += y[s].w;
      }
    }
    float v[8] = {a.x + bf16lo(braw.x), a.y + bf16hi(braw.x), a.z + bf16lo(braw.y),
                  a.w + bf16hi(braw.y), b.x + bf16lo(braw.z), b.y + bf16hi(braw.z),
                  b.z + bf16lo(braw.w), b.w + bf16hi(braw.w)};
    if constexpr (kGelu) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = gelu(v[j]);
    }
    *reinterpret_cast<uint4*>(out + r * N + c) =
        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                   pack_bf16x2(v[6], v[7]));
  }
}

template <bool kGelu>
cudaError_t set_smem_attr() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(dense_kernel<kGelu>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)FF_SMEM);
  });
  return err;
}

int sm_count_ff() {
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

// K splits of one layer: enough CTAs for about one wave over the SMs, at
// least four K steps of 64 per split.
DensePlan dense_plan(int rows, int K, int N) {
  DensePlan pl{};
  const int tiles = ((N + FF_BN - 1) / FF_BN) * ((rows + FF_BM - 1) / FF_BM);
  const int ksteps = (K + FF_BK - 1) / FF_BK;
  int splits = std::max(1, sm_count_ff() / std::max(1, tiles));
  splits = std::min(std::min(splits, FF_MAX_SPLITS), std::max(1, ksteps / 4));
  pl.ksteps_per_split = (ksteps + splits - 1) / splits;
  pl.splits = (ksteps + pl.ksteps_per_split - 1) / pl.ksteps_per_split;
  return pl;
}

size_t dense_partial_bytes(int rows, int K, int N) {
  const DensePlan pl = dense_plan(rows, K, N);
  return pl.splits > 1 ? (size_t)pl.splits * rows * N * sizeof(float) : 0;
}

cudaError_t launch_dense(const DenseArgs& a, cudaStream_t stream) {
  cudaError_t e = a.gelu ? set_smem_attr<true>() : set_smem_attr<false>();
  if (e != cudaSuccess) return e;
  if (a.rows == 0) return cudaSuccess;
  CUtensorMap mX, mW;
  if (!encode_2d(&mX, a.x, a.K, a.rows, a.K, FF_BK, FF_BM) ||
      !encode_2d(&mW, a.w, a.N, a.K, a.N, 64, FF_BK))
    return cudaErrorInvalidValue;
  const DensePlan pl = dense_plan(a.rows, a.K, a.N);
  FfParams p;
  p.rows = a.rows;
  p.K = a.K;
  p.N = a.N;
  p.ksteps_per_split = pl.ksteps_per_split;
  p.splits = pl.splits;
  p.bias = static_cast<const __nv_bfloat16*>(a.bias);
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.part = static_cast<float*>(a.part);
  p.err = a.err;
  p.wait_ns = pipeline_wait_ns();
  p.stall = pipeline_test_stall() ? 1 : 0;
  const dim3 grid((a.N + FF_BN - 1) / FF_BN, (a.rows + FF_BM - 1) / FF_BM, pl.splits);
  e = a.gelu ? launch_pdl(dense_kernel<true>, grid, dim3(FF_THREADS), FF_SMEM, stream, mX, mW, p)
             : launch_pdl(dense_kernel<false>, grid, dim3(FF_THREADS), FF_SMEM, stream, mX, mW, p);
  note_launch();
  if (e != cudaSuccess || pl.splits == 1) return e;
  const int64_t work = (int64_t)a.rows * (a.N / 8);
  const int blocks = (int)std::min<int64_t>((work + 255) / 256, 4 * sm_count_ff());
  e = a.gelu ? launch_pdl(dense_finish<true>, dim3(blocks), dim3(256), 0, stream,
                          (const float*)p.part, pl.splits, a.rows, a.N, p.bias, p.out)
             : launch_pdl(dense_finish<false>, dim3(blocks), dim3(256), 0, stream,
                          (const float*)p.part, pl.splits, a.rows, a.N, p.bias, p.out);
  note_launch();
  return e;
}

}  // namespace dd
