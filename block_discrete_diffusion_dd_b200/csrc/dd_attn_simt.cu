// dd_attn_simt.cu -- canvas attention on the CUDA cores (fp32 FMA).
//
// Serves fp32 inputs (whose accuracy target, 1e-5, is below what the tensor
// cores' TF32/bf16 inputs can reach) and any geometry the tcgen05 kernel does
// not cover (head_dim 64, odd head groupings).  Same definition as the
// tensor-core path ("DiffusionGemma Technical Report", paperfeed review,
// "The mechanism"): for canvas row i of batch b and query head h, one
// unmasked softmax over [prefix_b || canvas_b] keys of kv head h/(Hq/Hkv).
//
// A CTA owns 16 packed query rows (position i, head-in-group hh) of one
// (batch, kv head); 32-key tiles of K and V are staged in shared memory as
// fp32; lane j of a warp scores key j for the warp's 4 rows, then the warp
// runs an online softmax and each lane accumulates D/32 output columns.
#include "dd_device.cuh"
#include "dd_internal.h"

namespace dd {
namespace {

constexpr int kRowsPerWarp = 4;
constexpr int kWarps = 4;
constexpr int kRowsPerCta = kRowsPerWarp * kWarps;
constexpr int kKeyTile = 32;

template <typename T>
__device__ __forceinline__ float ld_f(const T* p) { return (float)(*p); }

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
    attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
                     const T* __restrict__ kp, const T* __restrict__ vp,
                     const int32_t* __restrict__ cu_prefix, int C, int Hq, int Hkv, float scale,
                     int row_blocks, T* __restrict__ out, float* __restrict__ lse) {
  constexpr int DPL = D / 32;  // output columns per lane
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

  const int nk = L + C;
  for (int j0 = 0; j0 < nk; j0 += kKeyTile) {
    __syncthreads();
    for (int e = threadIdx.x; e < kKeyTile * D; e += blockDim.x) {
      const int jj = e / D, d = e - jj * D;
      const int j = j0 + jj;
      float kv = 0.f, vv = 0.f;
      if (j < nk) {
        const int64_t off = j < L ? ((int64_t)(p0 + j) * Hkv + g) * D + d
                                  : (((int64_t)b * C + (j - L)) * Hkv + g) * D + d;
        kv = ld_f((j < L ? kp : kc) + off);
        vv = ld_f((j < L ? vp : vc) + off);
      }
      sK[jj][d] = kv;
      sV[jj][d] = vv;
    }
    __syncthreads();
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
      const float sr = valid ? s[r] * scale : -INFINITY;
      float mx = sr;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mn = fmaxf(m[r], mx);
      const float alpha = expf(m[r] - mn);  // m[r] = -inf on the first tile -> 0
      const float p = valid ? expf(sr - mn) : 0.f;
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
    if (lse && lane == 0) lse[((int64_t)b * Hq + h) * C + i] = m[r] + logf(l[r]);
  }
}

template <typename T, int D>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t stream) {
  const int M = a.C * (a.Hq / a.Hkv);
  const int row_blocks = (M + kRowsPerCta - 1) / kRowsPerCta;
  const int64_t grid = (int64_t)a.B * a.Hkv * row_blocks;
  attn_simt_kernel<T, D><<<(unsigned)grid, kWarps * 32, 0, stream>>>(
      static_cast<const T*>(a.q), static_cast<const T*>(a.kc), static_cast<const T*>(a.vc),
      static_cast<const T*>(a.kp), static_cast<const T*>(a.vp), a.cu_prefix, a.C, a.Hq, a.Hkv,
      a.scale, row_blocks, static_cast<T*>(a.out), a.lse);
  note_launch();
  return cudaGetLastError();
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
