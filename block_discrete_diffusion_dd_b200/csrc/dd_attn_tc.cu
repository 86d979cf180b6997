// dd_attn_tc.cu -- canvas attention on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory, operands staged by TMA).
//
// Definition ("DiffusionGemma Technical Report", paperfeed review, "The
// mechanism"): canvas queries attend bidirectionally to the canvas and to
// the causally encoded cache.  For batch row b and kv head g, the
// Hq/Hkv query heads that share g are packed with the canvas positions into
// M = C * (Hq/Hkv) query rows (row r = position * group + head-in-group);
// they all see the same key range [prefix_b || canvas_b] under one unmasked
// softmax.
//
// Work unit (one CTA): (b, g, pair of 128-row query tiles, split s of the
// key tiles).  The key range of b is cut into 128-key tiles -- prefix tiles
// first, then canvas tiles, each read through its own tensor map so a tile
// never straddles the prefix/canvas boundary; the last tile of each part is
// masked by key index.  The host picks each batch row's number of splits
// (its tiles shared out evenly) and launches the units longest first, so
// the SMs finish together; a second kernel merges the splits by their
// log-sum-exp.  When the units take more than one round of the SMs, each
// split CTA counts itself done on its (b, g, tile pair) counter with a
// release add once its partials are written, and the merge CTAs of that
// group poll the counter (acquire): a group is merged as soon as its own
// splits are done -- during the tail of the attention grid, on SMs it has
// left -- instead of after the whole grid.  The merge grid is launched as a
// programmatic dependent, which is scheduled only once every attention CTA
// has started, so a polling CTA never waits for a CTA that is not resident.
// With a single round every split ends at about the same time, and the
// merge waits for the whole grid instead (no counters).
//
// Inside a CTA (18 warps) the two query tiles share every key tile:
//   warps 0-7 / 8-15  softmax of query tile 0 / 1.  Each warp owns 16
//              query rows (TMEM lanes): through the 16-lane tcgen05.ld
//              shape a row's 128 key columns sit in four threads of the
//              warp, which reduce the row max and sum with two shuffles.
//              They run the online softmax in fp32 (log2 domain; O is
//              rescaled only when the running max grows past a margin) and
//              write P back (bf16 pairs in columns 0-63, E4M3 quads in
//              0-31) into the same TMEM region, where the P.V MMA reads it;
//   warp 16    TMA producer: Q, then K and V tiles (rings of 128 keys, 2
//              stages for bf16, 4 for E4M3) in the order the MMAs consume
//              them;
//   warp 17    allocates all 512 TMEM columns (per query tile: S/P 128, O
//              128) and issues every MMA from one elected lane of the
//              converged warp, in the order PV_0(j), S_0(j+1), PV_1(j),
//              S_1(j+1): each softmax warpgroup works while the tensor core
//              runs the other tile's MMAs.
// The tensor core executes one thread's MMAs in issue order, so:
//   - S_q(j+1) overwrites P_q(j) only after PV_q(j) has read it;
//   - when S_q(j) is complete, PV_q(j-1) is complete too, so the softmax
//     may rescale O_q at that point without a further wait.
// Every mbarrier wait is bounded in time; on expiry the CTA latches an
// error word, drains its own asynchronous work and frees its TMEM.
#include <algorithm>
#include <functional>
#include <mutex>
#include <queue>
#include <vector>

#include "dd_device.cuh"
#include "dd_internal.h"

namespace dd {
namespace {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int HD = 128;  // head dim
constexpr int kQT = 2;   // query tiles per CTA
constexpr int kMaxStages = 4;
constexpr int kSoftmaxWarps = 8 * kQT;  // two warps per 32 query rows
constexpr int kWarpTMA = kSoftmaxWarps, kWarpMMA = kSoftmaxWarps + 1;
constexpr int kThreads = (kSoftmaxWarps + 2) * 32;
constexpr uint32_t kHalf = 128 * 64 * 2;  // bf16: 128 rows x 64 elements (128 bytes)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = kQT * BN;     // O columns start after the S/P regions
constexpr int kStageWords = HD / 2 + 4;    // padded row (fp16 pairs) of the O staging area
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait

struct Barriers {
  uint64_t q_full;
  uint64_t k_full[kMaxStages], k_empty[kMaxStages], v_full[kMaxStages], v_empty[kMaxStages];
  uint64_t s_full[kQT], p_full[kQT], o_done[kQT];
  uint64_t staged[kQT];  // per query tile: all 8 warps have staged their O rows
  uint64_t mma_final;
  uint64_t never;  // completed by nothing: the target of the test stall
  uint32_t tmem_base;
  int abort;
  int unit_b, unit_g, unit_tp, unit_s, unit_valid, unit_nsplit, unit_slot0;
};

// Operand layout per input type.  A query or key row of HD elements is one
// 128-byte swizzle atom wide for E4M3 and two (the halves d < 64, d >= 64,
// kHalf apart) for bf16.  The E4M3 tiles are half the size, so they get a
// deeper K/V ring, which also leaves room for the O staging area.
//
// P = 2^(x - m_ref) with x the log2-domain score.  O is rescaled only when
// the row max exceeds m_ref + kLazy + kBias, and m_ref is set kBias below
// the row max, so every P lies in (0, 2^8].  For E4M3 P (largest finite
// value 448) the bias keeps P in the normal range down to 2^-12 of the row
// maximum (E4M3 subnormals start at 2^-6).
template <bool kF8>
struct Lay {
  static constexpr uint32_t kRow = kF8 ? HD : 2 * HD;  // bytes per row
  static constexpr uint32_t kTile = BM * kRow;
  static constexpr int kStages = kF8 ? 4 : 2;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQT * kTile;
  static constexpr uint32_t kOffV = kOffK + kStages * kTile;
  static constexpr uint32_t kOffBar = kOffV + kStages * kTile;
  static constexpr uint32_t kSmemBytes = kOffBar + sizeof(Barriers) + 1024;
  static constexpr float kBias = kF8 ? 6.0f : 0.0f;  // log2 units
  static constexpr float kLazy = kF8 ? 2.0f : 8.0f;  // log2 units
  static_assert(kStages <= kMaxStages, "barrier arrays");
  static_assert(kQT * BM * kStageWords * 4 <= kOffBar, "O staging fits the operand buffers");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// The host's split plan, passed by value (kernel parameter space).  Batch
// rows are launched in `order`: the i-th row in that order owns the units
// [ubase[i], ubase[i + 1]).  Row b has ns[b] key splits, its partials start
// at slot sbase[b], and its prefix rows are [p0[b], p0[b] + len[b]) of the
// packed prefix (the host's copy of cu_prefix, which also sized the prefix
// tensor maps), so no CTA reads cu_prefix before its first copies.  With
// more than kMaxPlanRows batch rows, n = 0 and the kernels derive a uniform
// plan from TcParams::chunk and the device cu_prefix instead.
constexpr int kMaxPlanRows = 128;
struct RowPlan {
  int n;
  int ubase[kMaxPlanRows + 1];
  int order[kMaxPlanRows];
  int sbase[kMaxPlanRows];
  int ns[kMaxPlanRows];
  int p0[kMaxPlanRows];
  int len[kMaxPlanRows];
};

struct TcParams {
  int B, C, Hq, Hkv, group, T, chunk;  // chunk: key tiles per split (uniform plan only)
  float scale_log2;  // softmax scale * log2(e), times the Q and K factors
  float out_scale;   // the V factor (1 for bf16)
  const int32_t* cu_prefix;
  // split partials, slot = (b, g, t, split): O / l of each row as fp16
  // pairs scaled by 2^-e_row, and (log2-domain LSE, 2^e_row) per row
  uint32_t* part_o;   // [slots][BM][HD / 2]
  float2* part_lse;   // [slots][BM]
  // per (b, g, tile pair): splits done, and merge CTAs that have seen them
  // all (the last one clears both for the next call); zero between calls
  uint32_t* done;
  uint32_t* seen;
  int poll;  // 1: the merge polls `done` per group; 0: it waits for the grid
  uint32_t* err;
  uint64_t wait_ns;  // limit of each pipeline wait (waits that drain use kWaitLimitNs)
  int stall;         // test stall: one wait on `never` once the first MMAs are issued
};

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// 2^e as a float for e in [-126, 127] (built from the exponent field).
__device__ __forceinline__ float pow2(int e) { return __int_as_float((127 + e) << 23); }

// The scale exponent of a partial row whose largest magnitude is m: e with
// m 2^-e in [2^14, 2^15) (below fp16's largest finite value, 65504), kept
// within [-126, 113] so that 2^e and 2^-e are normal floats; 0 for a row of
// zeros or a non-finite maximum.
__device__ __forceinline__ int row_exponent(float m) {
  if (!(m > 0.f) || !(m <= 3.4e38f)) return 0;
  return min(113, max(-126, ilogbf(m) - 14));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float2 unpack_f16x2(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

// blockIdx.x -> (b, g, query-tile pair tp, split s): a binary search of the
// plan's unit ranges, or (uniform plan) a walk over the batch rows.
// slot0 = partial slot of (b, g, 2 tp, s).
__device__ void resolve_unit(const TcParams& p, const RowPlan& rp, Barriers* bars) {
  const int TP = cdiv(p.T, kQT);
  int u = blockIdx.x;
  int valid = 0, b = 0, g = 0, tp = 0, s = 0, nsplit = 1, slot0 = 0;
  if (rp.n > 0) {
    if (u < rp.ubase[rp.n]) {
      int lo = 0, hi = rp.n;  // rp.ubase[lo] <= u < rp.ubase[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (rp.ubase[mid] <= u) lo = mid;
        else hi = mid;
      }
      b = rp.order[lo];
      nsplit = rp.ns[b];
      const int lu = u - rp.ubase[lo];
      s = lu % nsplit;
      tp = (lu / nsplit) % TP;
      g = lu / (nsplit * TP);
      slot0 = rp.sbase[b] + (g * p.T + tp * kQT) * nsplit + s;
      valid = 1;
    }
  } else {
    const int nc = cdiv(p.C, BN);
    int slots = 0;
    for (int bb = 0; bb < p.B; ++bb) {
      const int L = p.cu_prefix[bb + 1] - p.cu_prefix[bb];
      const int ns = cdiv(cdiv(L, BN) + nc, p.chunk);
      const int units = p.Hkv * TP * ns;
      if (u < units) {
        s = u % ns;
        tp = (u / ns) % TP;
        g = u / (ns * TP);
        b = bb;
        nsplit = ns;
        slot0 = slots + (g * p.T + tp * kQT) * ns + s;
        valid = 1;
        break;
      }
      u -= units;
      slots += p.Hkv * p.T * ns;
    }
  }
  bars->unit_b = b;
  bars->unit_g = g;
  bars->unit_tp = tp;
  bars->unit_s = s;
  bars->unit_valid = valid;
  bars->unit_nsplit = nsplit;
  bars->unit_slot0 = slot0;
}

// Shared-memory descriptors are built once per CTA; an operand at byte
// offset `off` from a 1024-aligned base has the base descriptor plus off/16
// in its start-address field (bits 0-13; every address here is below 2^18,
// so the field never carries).
__device__ __forceinline__ uint64_t desc_at(uint64_t base, uint32_t off) {
  return base + (uint64_t)(off >> 4);
}

// S_q = Q_q K^T into the S/P region of query tile q (K-major operands):
// K = 16 elements (32 bytes) per bf16 MMA, 32 elements (32 bytes) per E4M3
// MMA, stepping through the 128-byte swizzle rows.
template <bool kF8>
__device__ __forceinline__ void issue_s(uint32_t tmem, uint64_t dQ, uint64_t dK, int q, int st) {
  using G = Lay<kF8>;
  const uint32_t dS = tmem + (uint32_t)(q * BN);
  const uint64_t aq = desc_at(dQ, q * G::kTile), bk = desc_at(dK, st * G::kTile);
  if constexpr (kF8) {
    constexpr uint32_t idS = idesc_e4m3_f32(BM, BN, 0, 0);
#pragma unroll
    for (int kk = 0; kk < HD / 32; ++kk)
      tc_mma_ss_f8(dS, desc_at(aq, kk * 32), desc_at(bk, kk * 32), idS, kk > 0);
  } else {
    constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
      tc_mma_ss(dS, desc_at(aq, off), desc_at(bk, off), idS, kk > 0);
    }
  }
}

// O_q (+)= P_q V for one 128-key tile: P from tensor memory (aP), V from the
// ring stage at descriptor bv (MN-major).  P fills the first columns of the
// S/P region in key order, 2 keys per column for bf16 and 4 for E4M3.
template <bool kF8>
__device__ __forceinline__ void issue_pv(uint32_t dO, uint32_t aP, uint64_t bv, bool acc0) {
  if constexpr (kF8) {
    constexpr uint32_t idPV = idesc_e4m3_f32(BM, HD, 0, 1);
#pragma unroll
    for (int kk = 0; kk < BN / 32; ++kk)  // 32 keys = 8 columns of P, 4 KB of V
      tc_mma_ts_f8(dO, aP + (uint32_t)(kk * 8), desc_at(bv, kk * 32 * HD), idPV,
                   (acc0 || kk > 0) ? 1u : 0u);
  } else {
    constexpr uint32_t idPV = idesc_bf16_f32(BM, HD, 0, 1);
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk)  // 16 keys = 8 columns of P, 2 KB of each half of V
      tc_mma_ts(dO, aP + (uint32_t)(kk * 8), desc_at(bv, kk * 16 * 128), idPV,
                (acc0 || kk > 0) ? 1u : 0u);
  }
}

// One tile of 128 rows (HD elements each) of a [rows, heads, HD] tensor:
// one copy for E4M3 (128-byte rows), two 64-element halves for bf16.
template <bool kF8>
__device__ __forceinline__ void load_rows(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                          int head, int row0) {
  tma_load_3d(dst, map, bar, 0, head, row0);
  if constexpr (!kF8) tma_load_3d(dst + kHalf, map, bar, 64, head, row0);
}

// One 128-key tile of K (v = 0) or V (v = 1) into ring stage j % kStages.
template <bool kF8>
__device__ __forceinline__ bool load_kv(Barriers* bars, uint8_t* smem, int j, int v, int k_begin,
                                        int np, int p0, int b, int C, int g,
                                        const CUtensorMap* tmKp, const CUtensorMap* tmVp,
                                        const CUtensorMap* tmKc, const CUtensorMap* tmVc,
                                        volatile int* abort_flag, uint64_t wait_ns) {
  using G = Lay<kF8>;
  const int st = j % G::kStages, rd = j / G::kStages;
  uint64_t* empty = v ? &bars->v_empty[st] : &bars->k_empty[st];
  uint64_t* full = v ? &bars->v_full[st] : &bars->k_full[st];
  if (rd > 0 && !mbar_wait_bounded(empty, (rd - 1) & 1, abort_flag, wait_ns)) return false;
  const int k = k_begin + j;
  const CUtensorMap* map = k < np ? (v ? tmVp : tmKp) : (v ? tmVc : tmKc);
  const int row0 = k < np ? p0 + k * BN : b * C + (k - np) * BN;
  uint8_t* dst = smem + (v ? G::kOffV : G::kOffK) + st * G::kTile;
  mbar_arrive_expect_tx(full, G::kTile);
  load_rows<kF8>(dst, map, full, g, row0);
  return true;
}

template <bool kF8>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmKp,
                   const __grid_constant__ CUtensorMap tmVp,
                   const __grid_constant__ CUtensorMap tmKc,
                   const __grid_constant__ CUtensorMap tmVc, const TcParams p,
                   const __grid_constant__ RowPlan rp) {
  using G = Lay<kF8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + G::kOffBar);
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < G::kStages; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    for (int q = 0; q < kQT; ++q) {
      mbar_init(&bars->s_full[q], 1);
      mbar_init(&bars->p_full[q], 8);
      mbar_init(&bars->o_done[q], 1);
      mbar_init(&bars->staged[q], 8);
    }
    mbar_init(&bars->mma_final, 1);
    mbar_init(&bars->never, 1);
    bars->abort = 0;
    fence_mbar_init();
    resolve_unit(p, rp, bars);
  }
  if (warp == kWarpMMA) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = bars->tmem_base;
  const int b = bars->unit_b, g = bars->unit_g, tp = bars->unit_tp, s = bars->unit_s;
  const bool unit_ok = bars->unit_valid != 0;
  const int nsplit = bars->unit_nsplit, slot0 = bars->unit_slot0;
  const int p0 = !unit_ok ? 0 : rp.n > 0 ? rp.p0[b] : p.cu_prefix[b];
  const int L = !unit_ok ? 0 : rp.n > 0 ? rp.len[b] : p.cu_prefix[b + 1] - p0;
  const int np = cdiv(L, BN), nc = cdiv(p.C, BN);
  const int ntiles = np + nc;
  // split s of nsplit takes tiles [s T / nsplit, (s + 1) T / nsplit) of T
  const int k_begin = (int)((int64_t)s * ntiles / nsplit);
  const int n = unit_ok ? (int)((int64_t)(s + 1) * ntiles / nsplit) - k_begin : 0;
  const int nq = min(kQT, p.T - tp * kQT);  // query tiles in this CTA (1 or 2)

  if (warp == kWarpTMA) {
    if (lane == 0 && n > 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmKp);
      prefetch_tensormap(&tmKc);
      prefetch_tensormap(&tmVp);
      prefetch_tensormap(&tmVc);
      mbar_arrive_expect_tx(&bars->q_full, nq * G::kTile);
      for (int q = 0; q < nq; ++q) {
        const int qpos = b * p.C + (tp * kQT + q) * (BM / p.group);
        load_rows<kF8>(smem + G::kOffQ + q * G::kTile, &tmQ, &bars->q_full, g * p.group, qpos);
      }
      // in the order the MMAs consume them: K0, then V_j, K_{j+1}
      int kiss = 0, viss = 0;
      if (load_kv<kF8>(bars, smem, 0, 0, k_begin, np, p0, b, p.C, g, &tmKp, &tmVp, &tmKc, &tmVc,
                  abort_flag, p.wait_ns)) {
        kiss = 1;
        for (int j = 0; j < n; ++j) {
          if (!load_kv<kF8>(bars, smem, j, 1, k_begin, np, p0, b, p.C, g, &tmKp, &tmVp, &tmKc, &tmVc,
                       abort_flag, p.wait_ns))
            break;
          viss = j + 1;
          if (j + 1 < n) {
            if (!load_kv<kF8>(bars, smem, j + 1, 0, k_begin, np, p0, b, p.C, g, &tmKp, &tmVp, &tmKc,
                         &tmVc, abort_flag, p.wait_ns))
              break;
            kiss = j + 2;
          }
        }
      }
      // drain: loads still in flight must land before the CTA exits
      for (int j = max(0, kiss - G::kStages); j < kiss; ++j)
        mbar_wait_bounded(&bars->k_full[j % G::kStages], (j / G::kStages) & 1, nullptr,
                          kWaitLimitNs);
      for (int j = max(0, viss - G::kStages); j < viss; ++j)
        mbar_wait_bounded(&bars->v_full[j % G::kStages], (j / G::kStages) & 1, nullptr,
                          kWaitLimitNs);
      mbar_wait_bounded(&bars->q_full, 0, nullptr, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp == kWarpMMA) {
    if (n > 0) {
      // The whole warp runs this loop, so every MMA operand is warp-uniform
      // (computed once per warp rather than moved out of one lane's
      // registers before each MMA); one elected lane issues the MMAs and
      // their commits (a commit tracks the MMAs of the thread issuing it).
      const bool leader = elect_one_sync();
      // K-major Q and K (the leading offset is unused with 128-byte
      // swizzling); MN-major V: 8-key groups 1024 bytes apart along K,
      // 128-byte atoms along d kHalf apart (bf16; E4M3 rows are one atom)
      const uint64_t dQ = smem_desc_sw128(smem_u32(smem + G::kOffQ), 16, 1024);
      const uint64_t dK = smem_desc_sw128(smem_u32(smem + G::kOffK), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(smem + G::kOffV), kF8 ? G::kTile : kHalf, 1024);
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, abort_flag, p.wait_ns));
      };
      auto commit = [&](uint64_t* bar) {
        if (leader) tc_commit(bar);
        __syncwarp();
      };
      bool ok = wait(&bars->q_full, 0) && wait(&bars->k_full[0], 0);
      tc_fence_after();
      if (ok) {
        for (int q = 0; q < nq; ++q) {
          if (leader) {
            issue_s<kF8>(tmem, dQ, dK, q, 0);
            tc_commit(&bars->s_full[q]);
          }
          __syncwarp();
        }
        commit(&bars->k_empty[0]);
        // test stall: a wait nothing completes, with the first S MMAs in flight
        if (p.stall) ok = wait(&bars->never, 0);
      }
      for (int j = 0; ok && j < n; ++j) {
        const int vst = j % G::kStages;
        const bool more = j + 1 < n;
        const int kst = (j + 1) % G::kStages;
        if (!wait(&bars->v_full[vst], (j / G::kStages) & 1)) {
          ok = false;
          break;
        }
        for (int q = 0; q < nq; ++q) {
          if (!wait(&bars->p_full[q], j & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // O_q += P_q(j) V_j, P_q from TMEM
          const uint32_t dO = tmem + kTmemO + (uint32_t)(q * HD), aP = tmem + (uint32_t)(q * BN);
          const uint64_t bv = desc_at(dV, vst * G::kTile);
          if (leader) issue_pv<kF8>(dO, aP, bv, j > 0);
          __syncwarp();
          if (more) {
            if (q == 0 && !wait(&bars->k_full[kst], ((j + 1) / G::kStages) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (leader) {
              issue_s<kF8>(tmem, dQ, dK, q, kst);
              tc_commit(&bars->s_full[q]);
            }
            __syncwarp();
          }
        }
        if (!ok) break;
        commit(&bars->v_empty[vst]);
        if (more) commit(&bars->k_empty[kst]);
      }
      if (ok)
        for (int q = 0; q < nq; ++q) commit(&bars->o_done[q]);
      // every MMA issued above has completed before TMEM is released
      commit(&bars->mma_final);
      mbar_wait_bounded(&bars->mma_final, 0, nullptr, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp < kSoftmaxWarps && n > 0 && (warp >> 3) < nq) {
    // ------------------------------------------------------------ softmax
    // Warp (q, hv, wl) of query tile q reaches TMEM lane quarter wl (=
    // warp % 4) and takes its 16-lane half hv.  Through the 16x256b shape,
    // thread t holds rows A = 32 wl + 16 hv + t/4 and B = A + 8 and, of
    // every 8 key columns, the two at 2 (t % 4): 32 keys of each row.  The
    // four threads of a row reduce it with two shuffles, so the row max is
    // known before P is formed.
    const int q = warp >> 3, wl = warp & 3, hv = (warp >> 2) & 1;
    const int t4 = lane & 3;
    const int rbase = wl * 32 + hv * 16;
    const int rA = rbase + (lane >> 2), rB = rA + 8;  // query rows in tile q
    const uint32_t lane_base = (uint32_t)rbase << 16;  // TMEM lane field
    const uint32_t tS = tmem + lane_base + (uint32_t)(q * BN);
    const uint32_t tO = tmem + lane_base + kTmemO + (uint32_t)(q * HD);
    const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
    float mrefA = -INFINITY, mrefB = -INFINITY, lA = 0.f, lB = 0.f;
    bool ok = true;
    auto quad_max = [](float v) {
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
      return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
    };
    auto quad_sum = [](float v) {
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      return v + __shfl_xor_sync(0xffffffffu, v, 2);
    };
    // P = 2^(s scale_log2 - mref) for the thread's 64 scores, packed into
    // the first BN / 2 (bf16 pairs) or BN / 4 (E4M3 quads) columns of the
    // S/P region, where the P.V MMA reads it: this warp has loaded all of
    // its rows' S already.  Adds the rows' partial sums of the unrounded P.
    auto emit_p = [&](const uint32_t (&sv)[64], float ma, float mb) {
      const float2 na = make_float2(-ma, -ma), nb = make_float2(-mb, -mb);
      float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
      if constexpr (!kF8) {
        uint32_t w[32];  // 16x128b: w[2i] row A, w[2i + 1] row B, column 4 i + t % 4
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 da = __ffma2_rn(
              make_float2(__uint_as_float(sv[4 * i]), __uint_as_float(sv[4 * i + 1])), sl2, na);
          const float2 db = __ffma2_rn(
              make_float2(__uint_as_float(sv[4 * i + 2]), __uint_as_float(sv[4 * i + 3])), sl2, nb);
          const float2 pa = make_float2(ex2_approx(da.x), ex2_approx(da.y));
          const float2 pb = make_float2(ex2_approx(db.x), ex2_approx(db.y));
          sa = __fadd2_rn(sa, pa);
          sb = __fadd2_rn(sb, pb);
          w[2 * i] = pack_bf16x2(pa.x, pa.y);
          w[2 * i + 1] = pack_bf16x2(pb.x, pb.y);
        }
        tmem_st16x128b_x16(tS, w);
      } else {
        // a 32-bit column holds 4 keys; the thread's pair and its
        // neighbour's (thread t ^ 1) make one: the even thread stores row
        // A's, the odd one row B's (16x64b: lane t/4 + 8 (t % 2), column
        // 2 i + (t % 4) / 2)
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 da = __ffma2_rn(
              make_float2(__uint_as_float(sv[4 * i]), __uint_as_float(sv[4 * i + 1])), sl2, na);
          const float2 db = __ffma2_rn(
              make_float2(__uint_as_float(sv[4 * i + 2]), __uint_as_float(sv[4 * i + 3])), sl2, nb);
          const float2 pa = make_float2(ex2_approx(da.x), ex2_approx(da.y));
          const float2 pb = make_float2(ex2_approx(db.x), ex2_approx(db.y));
          sa = __fadd2_rn(sa, pa);
          sb = __fadd2_rn(sb, pb);
          const uint32_t ha = __nv_cvt_float2_to_fp8x2(pa, __NV_SATFINITE, __NV_E4M3);
          const uint32_t hb = __nv_cvt_float2_to_fp8x2(pb, __NV_SATFINITE, __NV_E4M3);
          const uint32_t oa = __shfl_xor_sync(0xffffffffu, ha, 1);
          const uint32_t ob = __shfl_xor_sync(0xffffffffu, hb, 1);
          w[i] = (lane & 1) ? (ob | (hb << 16)) : (ha | (oa << 16));
        }
        tmem_st16x64b_x16(tS, w);
      }
      lA += sa.x + sa.y;
      lB += sb.x + sb.y;
    };
    int j = 0;
    for (; j < n && ok; ++j) {
      const int k = k_begin + j;
      const int n_valid = k < np ? min(BN, L - k * BN) : min(BN, p.C - (k - np) * BN);
      // wait outcomes are made warp-uniform: tcgen05.ld/st are .sync.aligned
      if (!__all_sync(0xffffffffu,
                      mbar_wait_bounded(&bars->s_full[q], j & 1, abort_flag, p.wait_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld16x256b_x16(tS, sv);
      if (n_valid < BN) {  // ragged last tile of the prefix or of the canvas
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = 8 * i + 2 * t4;
          if (c >= n_valid) sv[4 * i] = sv[4 * i + 2] = __float_as_uint(-INFINITY);
          if (c + 1 >= n_valid) sv[4 * i + 1] = sv[4 * i + 3] = __float_as_uint(-INFINITY);
        }
      }
      float ma = fmaxf(__uint_as_float(sv[0]), __uint_as_float(sv[1]));
      float mb = fmaxf(__uint_as_float(sv[2]), __uint_as_float(sv[3]));
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        ma = fmaxf(ma, fmaxf(__uint_as_float(sv[4 * i]), __uint_as_float(sv[4 * i + 1])));
        mb = fmaxf(mb, fmaxf(__uint_as_float(sv[4 * i + 2]), __uint_as_float(sv[4 * i + 3])));
      }
      const float xa = quad_max(ma) * p.scale_log2, xb = quad_max(mb) * p.scale_log2;
      if (j == 0) {
        // first tile: the reference is the row max (less the bias)
        mrefA = xa - G::kBias;
        mrefB = xb - G::kBias;
      } else if (__any_sync(0xffffffffu, xa > mrefA + (G::kLazy + G::kBias) ||
                                             xb > mrefB + (G::kLazy + G::kBias))) {
        // lazy rescale (rare; a warp-uniform decision so tcgen05.ld/st stay
        // converged): PV_q(j-1) is complete because S_q(j) is
        const float na = fmaxf(mrefA, xa - G::kBias), nb = fmaxf(mrefB, xb - G::kBias);
        const float alA = ex2_approx(mrefA - na), alB = ex2_approx(mrefB - nb);
        lA *= alA;
        lB *= alB;
#pragma unroll 1
        for (int c16 = 0; c16 < HD / 16; ++c16) {
          uint32_t o[8];  // 16x256b x2: o[4r], o[4r+1] row A; o[4r+2], o[4r+3] row B
          tmem_ld16x256b_x2(tO + (uint32_t)(c16 * 16), o);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            o[e] = __float_as_uint(__uint_as_float(o[e]) * ((e & 2) ? alB : alA));
          tmem_st16x256b_x2(tO + (uint32_t)(c16 * 16), o);
        }
        mrefA = na;
        mrefB = nb;
      }
      emit_p(sv, mrefA, mrefB);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[q]);
    }
    // epilogue: O / l and the log2-domain LSE of this split
    if (ok)
      ok = __all_sync(0xffffffffu,
                      mbar_wait_bounded(&bars->o_done[q], 0, abort_flag, p.wait_ns));
    const float lrowA = quad_sum(lA), lrowB = quad_sum(lB);
    if (ok) {
      // O / l in fp16 pairs, each row scaled by a power of two 2^-e that
      // puts its largest magnitude in [2^14, 2^15): 11 significant bits
      // against the row maximum, whatever V's range, in half the bytes of
      // fp32.  Staged row-wise in shared memory (free now: every MMA has
      // completed; rows 68 words apart, so a warp's 32-bit stores hit 32
      // different banks), then copied out in whole 256-byte rows.
      tc_fence_after();
      const float invA = p.out_scale / lrowA, invB = p.out_scale / lrowB;
      uint32_t* stage = reinterpret_cast<uint32_t*>(smem) + q * (BM * kStageWords);
      const size_t slot = (size_t)slot0 + (size_t)q * nsplit;
      {
        uint32_t o[64];
        tmem_ld16x256b_x16(tO, o);
        float mA = 0.f, mB = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          mA = fmaxf(mA, fmaxf(fabsf(__uint_as_float(o[4 * i])), fabsf(__uint_as_float(o[4 * i + 1]))));
          mB = fmaxf(mB, fmaxf(fabsf(__uint_as_float(o[4 * i + 2])),
                               fabsf(__uint_as_float(o[4 * i + 3]))));
        }
        mA = quad_max(mA) * invA;
        mB = quad_max(mB) * invB;
        const int eA = row_exponent(mA), eB = row_exponent(mB);
        const float sA = invA * pow2(-eA), sB = invB * pow2(-eB);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int w = 4 * i + t4;  // columns 8 i + 2 t4, + 1
          stage[rA * kStageWords + w] =
              pack_f16x2(__uint_as_float(o[4 * i]) * sA, __uint_as_float(o[4 * i + 1]) * sA);
          stage[rB * kStageWords + w] =
              pack_f16x2(__uint_as_float(o[4 * i + 2]) * sB, __uint_as_float(o[4 * i + 3]) * sB);
        }
        if (t4 == 0) {
          p.part_lse[slot * BM + rA] = make_float2(mrefA + __log2f(lrowA), pow2(eA));
          p.part_lse[slot * BM + rB] = make_float2(mrefB + __log2f(lrowB), pow2(eB));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->staged[q]);
      if (__all_sync(0xffffffffu,
                     mbar_wait_bounded(&bars->staged[q], 0, abort_flag, p.wait_ns))) {
        uint32_t* dst = p.part_o + slot * BM * (HD / 2);
        const int wq = warp & 7;  // warp index within this query tile's 8
        // two rows per warp instruction, 16 bytes per lane
        for (int row = 2 * wq + (lane >> 4); row < BM; row += 16)
          *reinterpret_cast<uint4*>(dst + row * (HD / 2) + (lane & 15) * 4) =
              *reinterpret_cast<const uint4*>(stage + row * kStageWords + (lane & 15) * 4);
      }
    }
  }

  if (*abort_flag && threadIdx.x == 0) atomicOr(p.err, kDevErrTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // this split's partials are written (by every warp, ordered before the
  // barrier): release them to the merge.  An aborted CTA counts too, so the
  // merge never waits for it (its error is latched already).
  if (p.poll && threadIdx.x == 0 && bars->unit_valid)
    red_release_add(&p.done[(bars->unit_b * p.Hkv + bars->unit_g) * cdiv(p.T, kQT) + bars->unit_tp],
                    1u);
  if (warp == kWarpMMA) tmem_dealloc(tmem, kTmemCols);
}

// Merge the splits of every (b, g, t) query tile: lse = log2 sum 2^lse_s,
// O = sum_s 2^(lse_s - lse) 2^e_s O_s, O_s the split's scaled fp16 row.
// Each warp takes kRows query rows (kCombineWarps warps per CTA); lane s
// holds split s's weight, and lane l the row's columns 4 l .. 4 l + 3.
// kMaxS bounds the splits whose rows are all requested at once (kRows x
// kMaxS 8-byte loads per lane, at most 24, so that the grid is about one
// wave); more splits take a looped path.
constexpr int kCombineWarps = 8;  // warps per CTA of the combine kernel

// Final row of the combine: O = acc / wsum (4 columns per lane) and the
// natural-log LSE.
template <typename TOut>
__device__ __forceinline__ void combine_store(const TcParams& p, TOut* __restrict__ out,
                                              float* __restrict__ lse_out, int b, int g, int pr,
                                              int lane, float4 acc, float mx, float wsum) {
  const float inv = 1.f / wsum;
  const int i = pr / p.group, h = g * p.group + (pr - i * p.group);
  TOut* orow = out + (((size_t)b * p.C + i) * p.Hq + h) * HD + lane * 4;
  if constexpr (sizeof(TOut) == 2) {
    uint2 v;
    v.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    v.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(orow) = v;
  } else {
    *reinterpret_cast<float4*>(orow) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
  if (lse_out && lane == 0)
    lse_out[((size_t)b * p.Hq + h) * p.C + i] = (mx + __log2f(wsum)) * 0.6931471805599453f;
}

template <typename TOut, int kMaxS, int kRows>
__global__ void __launch_bounds__(kCombineWarps * 32, 3)
    attn_combine_kernel(const TcParams p, const __grid_constant__ RowPlan rp, int total_units,
                        TOut* __restrict__ out, float* __restrict__ lse_out) {
  // polling: the group's counter orders these reads after its splits'
  // writes (and every kernel before the attention grid has completed: each
  // attention CTA waited for it before this grid could start)
  if (!p.poll) pdl_wait();
  pdl_trigger();
  // kRows rows per warp, all of their split rows requested at once
  static_assert(kMaxS * kRows <= 24 && BM % (kCombineWarps * kRows) == 0, "merge shape");
  constexpr int kBlocksPerTile = BM / (kCombineWarps * kRows);
  int q = blockIdx.x / kBlocksPerTile;  // (b, g, t) group
  const int groups = p.Hkv * p.T;
  int b = -1, nsplit = 0, ubase = 0;
  if (rp.n > 0) {
    if (q < p.B * groups) {
      b = q / groups;
      q -= b * groups;
      nsplit = rp.ns[b];
      ubase = rp.sbase[b];
    }
  } else {
    const int nc = cdiv(p.C, BN);
    for (int bb = 0; bb < p.B; ++bb) {
      const int L = p.cu_prefix[bb + 1] - p.cu_prefix[bb];
      const int ns = cdiv(cdiv(L, BN) + nc, p.chunk);
      if (q < groups) {
        b = bb;
        nsplit = ns;
        break;
      }
      q -= groups;
      ubase += groups * ns;
    }
  }
  if (b < 0) return;
  const int g = q / p.T, t = q % p.T;
  const int u0 = ubase + q * nsplit;
  const int grp = (b * p.Hkv + g) * cdiv(p.T, kQT) + t / kQT;
  // the group's merge CTAs (kBlocksPerTile per query tile of the pair) have
  // all seen the count once the last of them has added itself to `seen`;
  // that one clears both counters for the next call (`seen_before` is read
  // only after this CTA's loads are in flight)
  uint32_t seen_before = 0;
  auto clear_if_last = [&]() {
    const uint32_t readers = (uint32_t)(min(kQT, p.T - (t / kQT) * kQT) * kBlocksPerTile);
    if (p.poll && threadIdx.x == 0 && seen_before == readers - 1) {
      p.done[grp] = 0;
      p.seen[grp] = 0;
    }
  };
  if (p.poll) {
    __shared__ int all_done;
    if (threadIdx.x == 0) {
      const uint64_t t0 = globaltimer_ns();
      bool ok = true;
      while (ld_acquire(&p.done[grp]) < (uint32_t)nsplit) {
        if (globaltimer_ns() - t0 > p.wait_ns) {
          atomicOr(p.err, kDevErrTimeout);
          ok = false;
          break;
        }
        __nanosleep(128);
      }
      all_done = ok ? 1 : 0;
      seen_before = atomicAdd(&p.seen[grp], 1u);
    }
    __syncthreads();
    if (!all_done) {
      clear_if_last();
      return;
    }
  }
  if (u0 + nsplit > total_units) {
    if (threadIdx.x == 0) atomicOr(p.err, kDevErrBounds);
    clear_if_last();
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = (blockIdx.x % kBlocksPerTile) * (kCombineWarps * kRows) + warp * kRows;
  const int rows_valid = p.C * p.group - t * BM;  // rows of this tile that exist
  if (nsplit <= kMaxS) {
    // common case: every split row and LSE of the warp's rows requested at
    // once (one L2 round trip), then the weights and the sums
    float2 lse_l[kRows];    // lane s: split s's (LSE, row scale)
    uint2 o[kRows][kMaxS];  // 4 fp16 columns per lane
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const int r = r0 + i;
      const bool rv = r < rows_valid;
      lse_l[i] = (rv && lane < nsplit) ? __ldcg(p.part_lse + (size_t)(u0 + lane) * BM + r)
                                       : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int u = 0; u < kMaxS; ++u)
        o[i][u] = (rv && u < nsplit)
                      ? __ldcg(reinterpret_cast<const uint2*>(
                                   p.part_o + ((size_t)(u0 + u) * BM + r) * (HD / 2)) +
                               lane)
                      : make_uint2(0u, 0u);
    }
    clear_if_last();
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const int r = r0 + i;
      if (r >= rows_valid) break;
      float mx = lse_l[i].x;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float wl = lane < nsplit ? exp2f(lse_l[i].x - mx) : 0.f;
      const float wo = wl * lse_l[i].y;  // the weight of the scaled fp16 row
      float wsum = wl;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < kMaxS; ++u) {
        const float w = __shfl_sync(0xffffffffu, wo, u);  // 0 past nsplit
        const float2 a = unpack_f16x2(o[i][u].x), c = unpack_f16x2(o[i][u].y);
        acc.x = fmaf(w, a.x, acc.x);
        acc.y = fmaf(w, a.y, acc.y);
        acc.z = fmaf(w, c.x, acc.z);
        acc.w = fmaf(w, c.y, acc.w);
      }
      combine_store<TOut>(p, out, lse_out, b, g, t * BM + r, lane, acc, mx, wsum);
    }
    return;
  }
  clear_if_last();
  for (int i = 0; i < kRows; ++i) {
    const int r = r0 + i;
    if (r >= rows_valid) break;
    // split weights, 32 splits per pass
    float mx = -INFINITY;
    for (int s0 = 0; s0 < nsplit; s0 += 32) {
      const int s = s0 + lane;
      if (s < nsplit) mx = fmaxf(mx, __ldcg(p.part_lse + (size_t)(u0 + s) * BM + r).x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float wsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < nsplit; s0 += 32) {
      const int s = s0 + lane;
      const float2 ls = s < nsplit ? __ldcg(p.part_lse + (size_t)(u0 + s) * BM + r)
                                   : make_float2(-INFINITY, 0.f);
      const float wl = s < nsplit ? exp2f(ls.x - mx) : 0.f;
      const float wo = wl * ls.y;  // the weight of the scaled fp16 row
      float ws = wl;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, off);
      wsum += ws;
      const int n = min(32, nsplit - s0);
      // eight splits' rows in flight at a time (L2 latency, not bandwidth,
      // is what a one-row-at-a-time loop waits on)
      for (int j0 = 0; j0 < n; j0 += 8) {
        uint2 ov[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          ov[u] = j0 + u < n ? __ldcg(reinterpret_cast<const uint2*>(
                                   p.part_o + ((size_t)(u0 + s0 + j0 + u) * BM + r) * (HD / 2)) +
                               lane)
                             : make_uint2(0u, 0u);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float w = __shfl_sync(0xffffffffu, wo, j0 + u);  // 0 past nsplit
          const float2 a = unpack_f16x2(ov[u].x), c = unpack_f16x2(ov[u].y);
          acc.x = fmaf(w, a.x, acc.x);
          acc.y = fmaf(w, a.y, acc.y);
          acc.z = fmaf(w, c.x, acc.z);
          acc.w = fmaf(w, c.y, acc.w);
        }
      }
    }
    combine_store<TOut>(p, out, lse_out, b, g, t * BM + r, lane, acc, mx, wsum);
  }
}

// ----------------------------------------------------------------- host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
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

// 3-D map over a [rows, heads, 128] tensor of bf16 (f8 = false) or 8-bit
// elements (f8 = true, copied as bytes), box (128 bytes of a row, box_heads,
// box_rows), 128-byte swizzle; rows outside [0, rows) read as zero.
bool encode_map(CUtensorMap* m, const void* base, int64_t rows, int heads, int box_heads,
                int box_rows, bool f8) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t esz = f8 ? 1 : 2;
  const cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)heads, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)HD * esz, (cuuint64_t)heads * HD * esz};
  const cuuint32_t box[3] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

struct Plan {
  int T, chunk, units, slots, groups, max_ns;
  RowPlan rp;
};

// The attention kernel's parameters (five tensor maps, TcParams, RowPlan)
// stay within the classic 4 KB kernel-parameter space.
static_assert(5 * sizeof(CUtensorMap) + sizeof(TcParams) + sizeof(RowPlan) <= 4096,
              "kernel parameters");

// Cost model of one CTA (measured on B200 with per-CTA %globaltimer traces):
// about 8.5 us of fixed work -- set-up, the first S tile, the wait for the
// last P.V and the write of its split partials (128 KB per CTA when they
// were fp32; the fp16 partials take about 1.5 us off, which changes none of
// the plans of the workloads measured here) -- and 1.84 us per 128-key tile,
// so the fixed part weighs as much as kUnitFixed tiles.  The merge pass
// reads each partial slot once: kSlotMerge tiles per slot for the GPU (set
// for a 64 KB fp32 slot at ~5 TB/s; the fp16 slots are half that, which
// again changes none of those plans).
constexpr double kUnitFixed = 4.6;
constexpr double kSlotMerge = 0.0071;

// Makespan (in key tiles) of the units of `ns` launched row by row in
// `order`, each unit going to the SM that frees first: the hardware hands
// out CTAs in launch order as SMs free up, one attention CTA per SM.
double simulate(const std::vector<int>& tiles, const std::vector<int>& ns,
                const std::vector<int>& order, int per_split, int sms) {
  std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
  for (int i = 0; i < sms; ++i) free_at.push(0.0);
  double end = 0.0;
  for (int b : order) {
    const int t = tiles[b], n = ns[b];
    for (int lu = 0; lu < per_split * n; ++lu) {
      const int sp = lu % n;
      const int len = (int)((int64_t)(sp + 1) * t / n - (int64_t)sp * t / n);
      const double start = free_at.top();
      free_at.pop();
      const double fin = start + kUnitFixed + len;
      free_at.push(fin);
      end = std::max(end, fin);
    }
  }
  return end;
}

// Rows launched longest unit first (ties: lower batch row first).
std::vector<int> lpt_order(const std::vector<int>& tiles, const std::vector<int>& ns) {
  std::vector<int> order(tiles.size());
  for (size_t b = 0; b < order.size(); ++b) order[b] = (int)b;
  auto longest = [&](int b) { return (tiles[b] + ns[b] - 1) / ns[b]; };
  std::stable_sort(order.begin(), order.end(),
                   [&](int x, int y) { return longest(x) > longest(y); });
  return order;
}

// The split plan.  Every batch row b of tiles_b key tiles gets
// ns_b = ceil(tiles_b / target) splits, for the target length (in tiles)
// that minimises the simulated makespan plus the merge pass; rows go out
// longest unit first.  Batches wider than kMaxPlanRows use one split length
// for all rows (the kernels derive that plan themselves).
Plan plan_uncached(const AttnArgs& a) {
  Plan pl{};
  const int group = a.Hq / a.Hkv;
  pl.T = (a.C * group + BM - 1) / BM;
  const int TP = (pl.T + kQT - 1) / kQT;
  const int nc = (a.C + BN - 1) / BN;
  const int sms = num_sms();
  pl.groups = a.B * a.Hkv * pl.T;
  std::vector<int> tiles(a.B);
  int max_tiles = 1;
  int64_t total = 0;
  for (int b = 0; b < a.B; ++b) {
    const int L = a.cu_prefix_host[b + 1] - a.cu_prefix_host[b];
    tiles[b] = (L + BN - 1) / BN + nc;
    max_tiles = std::max(max_tiles, tiles[b]);
    total += (int64_t)tiles[b] * a.Hkv * TP;
  }
  if (a.B > kMaxPlanRows) {
    // uniform split length: waves(units) * (chunk + 2), plus a charge per
    // split for the merge
    double best_cost = 1e300;
    for (int chunk = 1; chunk <= max_tiles; ++chunk) {
      int64_t units = 0, slots = 0;
      int max_ns = 1;
      for (int b = 0; b < a.B; ++b) {
        const int ns = (tiles[b] + chunk - 1) / chunk;
        units += (int64_t)a.Hkv * TP * ns;
        slots += (int64_t)a.Hkv * pl.T * ns;
        max_ns = std::max(max_ns, ns);
      }
      const int64_t waves = (units + sms - 1) / sms;
      const double cost = (double)waves * (chunk + 2) + 0.25 * (double)units / sms;
      if (cost < best_cost - 1e-9) {
        best_cost = cost;
        pl.chunk = chunk;
        pl.units = (int)units;
        pl.slots = (int)slots;
        pl.max_ns = max_ns;
      }
    }
    pl.rp.n = 0;
    return pl;
  }
  // candidate target lengths: each share of the longest row, and the even
  // share of all the work over 1-4 rounds of the SMs
  std::vector<int> cand;
  for (int k = 1; k <= 32; ++k) cand.push_back((max_tiles + k - 1) / k);
  for (int w = 1; w <= 4; ++w)
    cand.push_back((int)std::max<int64_t>(1, (total + (int64_t)w * sms - 1) / ((int64_t)w * sms)));
  std::sort(cand.begin(), cand.end());
  cand.erase(std::unique(cand.begin(), cand.end()), cand.end());
  double best_cost = 1e300;
  std::vector<int> best_ns;
  for (int target : cand) {
    std::vector<int> ns(a.B);
    int64_t units = 0;
    for (int b = 0; b < a.B; ++b) {
      ns[b] = std::min(tiles[b], std::max(1, (tiles[b] + target - 1) / target));
      units += (int64_t)a.Hkv * TP * ns[b];
    }
    // more than 16 rounds of the SMs never pays; the one-split plan is
    // always a candidate
    if (units > 16 * (int64_t)sms && target != max_tiles) continue;
    int64_t slots = 0;
    for (int b = 0; b < a.B; ++b) slots += (int64_t)a.Hkv * pl.T * ns[b];
    const double cost =
        simulate(tiles, ns, lpt_order(tiles, ns), a.Hkv * TP, sms) + kSlotMerge * (double)slots;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best_ns = ns;
    }
  }
  const std::vector<int> order = lpt_order(tiles, best_ns);
  RowPlan& rp = pl.rp;
  rp.n = a.B;
  int slots = 0;
  pl.max_ns = 1;
  for (int b = 0; b < a.B; ++b) {
    rp.ns[b] = best_ns[b];
    rp.p0[b] = a.cu_prefix_host[b];
    rp.len[b] = a.cu_prefix_host[b + 1] - a.cu_prefix_host[b];
    rp.sbase[b] = slots;
    slots += a.Hkv * pl.T * best_ns[b];
    pl.max_ns = std::max(pl.max_ns, best_ns[b]);
  }
  rp.ubase[0] = 0;
  for (int i = 0; i < a.B; ++i) {
    rp.order[i] = order[i];
    rp.ubase[i + 1] = rp.ubase[i] + a.Hkv * TP * best_ns[order[i]];
  }
  pl.units = rp.ubase[a.B];
  pl.slots = slots;
  pl.chunk = max_tiles;  // unused with a row plan
  return pl;
}

// The plan depends on the shape and the prefix lengths only; the last one
// is kept per host thread (a decode loop asks for the same plan every step).
Plan make_plan(const AttnArgs& a) {
  struct Cache {
    bool valid = false;
    int B = 0, C = 0, Hq = 0, Hkv = 0, sms = 0;
    std::vector<int32_t> cu;
    Plan plan;
  };
  thread_local Cache cache;
  const int sms = num_sms();
  if (cache.valid && cache.B == a.B && cache.C == a.C && cache.Hq == a.Hq &&
      cache.Hkv == a.Hkv && cache.sms == sms &&
      std::equal(cache.cu.begin(), cache.cu.end(), a.cu_prefix_host))
    return cache.plan;
  cache.plan = plan_uncached(a);
  cache.B = a.B;
  cache.C = a.C;
  cache.Hq = a.Hq;
  cache.Hkv = a.Hkv;
  cache.sms = sms;
  cache.cu.assign(a.cu_prefix_host, a.cu_prefix_host + a.B + 1);
  cache.valid = true;
  return cache.plan;
}

}  // namespace

bool attn_tc_supported(const AttnArgs& a) {
  if (!(a.bf16 || a.e4m3) || a.D != HD) return false;
  const int group = a.Hq / a.Hkv;
  if (group < 1 || BM % group != 0) return false;
  // TMA: 16-byte aligned bases (rows of 256 bytes are always aligned)
  const uintptr_t mask = 15;
  if ((reinterpret_cast<uintptr_t>(a.q) | reinterpret_cast<uintptr_t>(a.kc) |
       reinterpret_cast<uintptr_t>(a.vc) | reinterpret_cast<uintptr_t>(a.kp) |
       reinterpret_cast<uintptr_t>(a.vp)) & mask)
    return false;
  return true;
}

// Scratch: the done/seen counters (two per (b, g, tile pair)), then the
// partial O and LSE of every slot.
size_t counter_bytes(const AttnArgs& a, const Plan& pl) {
  const size_t n = (size_t)a.B * a.Hkv * ((pl.T + kQT - 1) / kQT);
  return (2 * n * sizeof(uint32_t) + 255) & ~(size_t)255;
}

size_t attn_tc_scratch_bytes(const AttnArgs& a) {
  const Plan pl = make_plan(a);
  return counter_bytes(a, pl) + (size_t)pl.slots * BM * (HD * 2 + sizeof(float2)) + 256;
}

template <bool kF8>
cudaError_t set_smem_attr() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    err = cudaFuncSetAttribute(attn_tc_kernel<kF8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)Lay<kF8>::kSmemBytes);
  });
  return err;
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t stream) {
  const bool f8 = a.e4m3;
  cudaError_t attr_err = f8 ? set_smem_attr<true>() : set_smem_attr<false>();
  if (attr_err != cudaSuccess) return attr_err;

  const Plan pl = make_plan(a);
  const int group = a.Hq / a.Hkv;
  CUtensorMap mQ, mKp, mVp, mKc, mVc;
  bool ok = encode_map(&mQ, a.q, (int64_t)a.B * a.C, a.Hq, group, BM / group, f8) &&
            encode_map(&mKc, a.kc, (int64_t)a.B * a.C, a.Hkv, 1, BN, f8) &&
            encode_map(&mVc, a.vc, (int64_t)a.B * a.C, a.Hkv, 1, BN, f8);
  if (a.total_prefix > 0) {
    ok = ok && encode_map(&mKp, a.kp, a.total_prefix, a.Hkv, 1, BN, f8) &&
         encode_map(&mVp, a.vp, a.total_prefix, a.Hkv, 1, BN, f8);
  } else {  // no prefix rows anywhere: the prefix maps are never read
    mKp = mKc;
    mVp = mVc;
  }
  if (!ok) return cudaErrorInvalidValue;

  TcParams tp;
  tp.B = a.B;
  tp.C = a.C;
  tp.Hq = a.Hq;
  tp.Hkv = a.Hkv;
  tp.group = group;
  tp.T = pl.T;
  tp.chunk = pl.chunk;
  tp.scale_log2 = f8 ? (float)((double)a.scale * 1.4426950408889634 * (double)a.q_scale *
                               (double)a.k_scale)
                     : a.scale * 1.4426950408889634f;
  tp.out_scale = f8 ? a.v_scale : 1.0f;
  tp.cu_prefix = a.cu_prefix;
  uint8_t* scratch = static_cast<uint8_t*>(a.scratch);
  const size_t ncnt = (size_t)a.B * a.Hkv * ((pl.T + kQT - 1) / kQT);
  tp.done = reinterpret_cast<uint32_t*>(scratch);
  tp.seen = tp.done + ncnt;
  scratch += counter_bytes(a, pl);
  tp.part_o = reinterpret_cast<uint32_t*>(scratch);
  tp.part_lse = reinterpret_cast<float2*>(scratch + (size_t)pl.slots * BM * HD * 2);
  tp.err = a.err;
  tp.wait_ns = pipeline_wait_ns();
  tp.stall = pipeline_test_stall() ? 1 : 0;
  tp.poll = pl.units > num_sms() ? 1 : 0;

  cudaError_t e =
      f8 ? launch_pdl(attn_tc_kernel<true>, dim3(pl.units), dim3(kThreads), Lay<true>::kSmemBytes,
                      stream, mQ, mKp, mVp, mKc, mVc, tp, pl.rp)
         : launch_pdl(attn_tc_kernel<false>, dim3(pl.units), dim3(kThreads),
                      Lay<false>::kSmemBytes, stream, mQ, mKp, mVp, mKc, mVc, tp, pl.rp);
  note_launch();
  if (e != cudaSuccess) return e;
  // kMaxS splits of kRows rows per warp in flight (kMaxS * kRows <= 24
  // 8-byte loads per lane), so that the merge grid is about one wave
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out);
  const dim3 cblock(kCombineWarps * 32);
  auto cgrid = [&](int rows) { return dim3(pl.groups * (BM / (kCombineWarps * rows))); };
  if (pl.max_ns <= 4)
    e = launch_pdl(attn_combine_kernel<__nv_bfloat16, 4, 4>, cgrid(4), cblock, 0, stream, tp,
                   pl.rp, (int)pl.slots, out, a.lse);
  else if (pl.max_ns <= 8)
    e = launch_pdl(attn_combine_kernel<__nv_bfloat16, 8, 2>, cgrid(2), cblock, 0, stream, tp,
                   pl.rp, (int)pl.slots, out, a.lse);
  else if (pl.max_ns <= 12)
    e = launch_pdl(attn_combine_kernel<__nv_bfloat16, 12, 2>, cgrid(2), cblock, 0, stream, tp,
                   pl.rp, (int)pl.slots, out, a.lse);
  else
    e = launch_pdl(attn_combine_kernel<__nv_bfloat16, 16, 1>, cgrid(1), cblock, 0, stream, tp,
                   pl.rp, (int)pl.slots, out, a.lse);
  note_launch();
  return e;
}

}  // namespace dd
