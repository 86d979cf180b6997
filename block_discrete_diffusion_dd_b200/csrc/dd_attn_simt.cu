// dd_attn_simt.cu -- canvas attention on the CUDA cores (fp32 FMA).
//
// Serves fp32 inputs (whose accuracy target, 1e-5, is below what the tensor
// cores' TF32/bf16 inputs can reach) and any geometry the tcgen05 kernel does
// not cover (head_dim 64, odd head groupings).  Same definition as the
// tensor-core path ("DiffusionGemma Technical Report", paperfeed review,
// "The mechanism"): for canvas row i of batch b and query head h, one
// unmasked softmax over [prefix_b || canvas_b] keys of kv head h/(Hq/Hkv).
//
// A CTA owns 4 * RPW packed query rows (position i, head-in-group hh) of one
// (batch, kv head); 32-key tiles of K and V are staged in shared memory as
// fp32; lane j of a warp scores key j for the warp's RPW rows, then the warp
// runs an online softmax (base 2, on scores pre-scaled by log2 e) and each
// lane accumulates D/32 output columns.  RPW = 4 amortises the K/V tiles
// over more rows; small problems take RPW = 1 to spread over more SMs.
#include "dd_device.cuh"
#include "dd_internal.h"

namespace dd {
namespace {

constexpr int kWarps = 4;
constexpr int kKeyTile = 32;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T>
__device__ __forceinline__ float ld_f(const T* p) { return (float)(*p); }

template <typename T, int D, int kRowsPerWarp>
__global__ void __launch_bounds__(kWarps * 32)
    attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
                     const T* __restrict__ kp, const T* __restrict__ vp,
                     const int32_t* __restrict__ cu_prefix, int C, int Hq, int Hkv, float scale,
                     int row_blocks, T* __restrict__ out, float* __restrict__ lse) {
  constexpr int DPL = D / 32;  // output columns per lane
  constexpr int kRowsPerCta = kRowsPerWarp * kWarps;
  const float scale2 = scale * kLog2e;  // scores in log2 units
  __shared__ float sK[kKeyTile][D + 1];
  __shared__ float sV[kKeyTile][D];
  __shared__ float sQ[kRowsPerCta][D];

  const int group = Hq / Hkv;
  const int rb = blockIdx.x % row_blocks;
  const int g = (blockIdx.x / row_blocks) % Hkv;
  const int b = blockIdx.x / (row_blocks * Hkv);
  const int M = C * group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int p0 = cu_prefix[b];
  const int L = cu_prefix[b + 1] - p0;

  // stage the CTA's query rows
  for (int e = threadIdx.x; e < kRowsPerCta * D; e += blockDim.x) {
    const int lr = e / D, d = e - lr * D;
    const int r = rb * kRowsPerCta + lr;
    float v = 0.f;
    if (r < M) {
      const int i = r / group, h = g * group + (r - i * group);
      v = ld_f(q + (((int64_t)b * C + i) * Hq + h) * D + d);
    }
    sQ[lr][d] = v;
  }

  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][DPL];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int k = 0; k < DPL; ++k) o[r][k] = 0.f;
  }

  // K/V tiles move as 16-byte vectors; each thread holds its share of the
  // next tile in registers while the current one is scored
  constexpr int kVec = 16 / (int)sizeof(T);          // elements per vector
  constexpr int kVecPerRow = D / kVec;
  constexpr int kVecPerThread = kKeyTile * kVecPerRow / (kWarps * 32);
  static_assert(kKeyTile * kVecPerRow % (kWarps * 32) == 0, "tile splits evenly");
  const int nk = L + C;
  uint4 pk[kVecPerThread], pv[kVecPerThread];
  auto fetch = [&](int j0) {
#pragma unroll
    for (int t = 0; t < kVecPerThread; ++t) {
      const int e = threadIdx.x + t * kWarps * 32;
      const int jj = e / kVecPerRow, c = e - jj * kVecPerRow;
      const int j = j0 + jj;
      pk[t] = make_uint4(0u, 0u, 0u, 0u);
      pv[t] = make_uint4(0u, 0u, 0u, 0u);
      if (j < nk) {
        const int64_t row = j < L ? (int64_t)(p0 + j) * Hkv + g : ((int64_t)b * C + (j - L)) * Hkv + g;
        pk[t] = *reinterpret_cast<const uint4*>((j < L ? kp : kc) + row * D + c * kVec);
        pv[t] = *reinterpret_cast<const uint4*>((j < L ? vp : vc) + row * D + c * kVec);
      }
    }
  };
  auto stash = [&]() {
#pragma unroll
    for (int t = 0; t < kVecPerThread; ++t) {
      const int e = threadIdx.x + t * kWarps * 32;
      const int jj = e / kVecPerRow, c = e - jj * kVecPerRow;
      const T* ke = reinterpret_cast<const T*>(&pk[t]);
      const T* ve = reinterpret_cast<const T*>(&pv[t]);
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        sK[jj][c * kVec + u] = ld_f(ke + u);
        sV[jj][c * kVec + u] = ld_f(ve + u);
      }
    }
  };
  fetch(0);
  for (int j0 = 0; j0 < nk; j0 += kKeyTile) {
    __syncthreads();
    stash();
    __syncthreads();
    if (j0 + kKeyTile < nk) fetch(j0 + kKeyTile);
    const bool valid = j0 + lane < nk;
    float s[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) s[r] = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) {
      const float kd = sK[lane][d];
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) s[r] = fmaf(sQ[warp * kRowsPerWarp + r][d], kd, s[r]);
    }
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const float sr = valid ? s[r] * scale2 : -INFINITY;
      float mx = sr;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mn = fmaxf(m[r], mx);
      const float alpha = ex2_approx(m[r] - mn);  // m[r] = -inf on the first tile -> 0
      const float p = valid ? ex2_approx(sr - mn) : 0.f;
      float ps = p;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[r] = l[r] * alpha + ps;
      m[r] = mn;
#pragma unroll
      for (int k = 0; k < DPL; ++k) o[r][k] *= alpha;
#pragma unroll 8
      for (int jj = 0; jj < kKeyTile; ++jj) {
        const float pj = __shfl_sync(0xffffffffu, p, jj);
#pragma unroll
        for (int k = 0; k < DPL; ++k) o[r][k] = fmaf(pj, sV[jj][lane + 32 * k], o[r][k]);
      }
    }
  }

#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int pr = rb * kRowsPerCta + warp * kRowsPerWarp + r;
    if (pr >= M) continue;
    const int i = pr / group, h = g * group + (pr - i * group);
    const float inv = 1.f / l[r];
    T* orow = out + (((int64_t)b * C + i) * Hq + h) * D;
#pragma unroll
    for (int k = 0; k < DPL; ++k) orow[lane + 32 * k] = (T)(o[r][k] * inv);
    if (lse && lane == 0) lse[((int64_t)b * Hq + h) * C + i] = (m[r] + log2f(l[r])) / kLog2e;
  }
}

template <typename T, int D, int RPW>
cudaError_t launch_rpw(const AttnArgs& a, cudaStream_t stream) {
  constexpr int kRowsPerCta = RPW * kWarps;
  const int M = a.C * (a.Hq / a.Hkv);
  const int row_blocks = (M + kRowsPerCta - 1) / kRowsPerCta;
  const int64_t grid = (int64_t)a.B * a.Hkv * row_blocks;
  attn_simt_kernel<T, D, RPW><<<(unsigned)grid, kWarps * 32, 0, stream>>>(
      static_cast<const T*>(a.q), static_cast<const T*>(a.kc), static_cast<const T*>(a.vc),
      static_cast<const T*>(a.kp), static_cast<const T*>(a.vp), a.cu_prefix, a.C, a.Hq, a.Hkv,
      a.scale, row_blocks, static_cast<T*>(a.out), a.lse);
  note_launch();
  return cudaGetLastError();
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  return n;
}

// Four rows per warp unless that leaves fewer CTAs than about two per SM.
template <typename T, int D>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t stream) {
  const int M = a.C * (a.Hq / a.Hkv);
  const int64_t ctas4 = (int64_t)a.B * a.Hkv * ((M + 4 * kWarps - 1) / (4 * kWarps));
  if (ctas4 >= 2 * (int64_t)sm_count()) return launch_rpw<T, D, 4>(a, stream);
  return launch_rpw<T, D, 1>(a, stream);
}

}  // namespace

size_t attn_simt_scratch_bytes(const AttnArgs&) { return 0; }

cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t stream) {
  if (a.bf16) {
    if (a.D == 64) return launch_t<__nv_bfloat16, 64>(a, stream);
    return launch_t<__nv_bfloat16, 128>(a, stream);
  }
  if (a.D == 64) return launch_t<float, 64>(a, stream);
  return launch_t<float, 128>(a, stream);
}

}  // namespace dd
