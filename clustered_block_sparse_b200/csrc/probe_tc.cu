// Compensation-error probe on the sm_100a tensor cores (SVG-EAR §4.2 "Error
// estimation"; §1: query centroids stand in for the queries of their
// cluster; §4.4: the estimate is one streaming pass over the keys), bf16 keys.
//
//   E[a][b] = sum_{j in b} (s q̄_a·k_j - s q̄_a·k̄_b)^2
//
// is evaluated as a C_q x N_k GEMM S = q̄ K^T fused with a per-key-cluster
// reduction of (s S_aj - s μ_ab)^2, μ_ab = q̄_a·k̄_b:
//   pr_prep   q̄ (fp32) -> three bf16 parts q1 + q2 + q3 = q̄ exactly (each
//             remainder is exact in fp32 and has at most 16, then 8,
//             significant bits), rows padded to 128 per M tile; and
//             -s μ_ab in fp64, stored as an fp32 pair (hi + lo).
//   pr_tc     persistent: each CTA takes a contiguous share of the (slice,
//             128-row M tile of query centroids, key row) space and, in each
//             slice it touches, the WHOLE key clusters that start in its share
//             (so every block sum is finished in one CTA, in a fixed order: E
//             is deterministic); q̄ is reloaded when the slice changes.  A TMA warp
//             streams 128-key tiles of K_perm (or, gathered, of K in original
//             order: each lane looks up four rows' original indices in k_perm
//             and the elected lane fetches them with tile::gather4 into the
//             same swizzled tile); one elected thread issues
//             tcgen05.mma (three MMAs per k step, one per q̄ part, fp32
//             accumulation in TMEM, four accumulator buffers); four epilogue
//             warps (one TMEM lane = one centroid row each) walk the tile's
//             columns in key order: g = s S + (-s μ) (hi then lo), sum g^2,
//             and store E[a][b] when key cluster b ends.  Empty key clusters
//             and empty query clusters get E = 0.
// The keys are bf16, so each product of a q̄ part and a key is exact in fp32;
// the only rounding is the fp32 accumulation, about the same as an fp32 dot
// product.
#include <algorithm>
#include <mutex>

#include "ear_internal.cuh"
#include "sm100.cuh"

namespace ear {
namespace {

using namespace sm100;

constexpr int kM = 128;       // query centroid rows per M tile
constexpr int kN = 128;       // keys per tile
constexpr int kParts = 3;     // bf16 parts of q̄
constexpr int kAcc = 4;       // TMEM accumulator buffers (kN columns each)
constexpr int kThreads = 192; // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

constexpr int kBarAFull = 0;
constexpr int kBarAEmpty = 1;
constexpr int kBarBFull = 2;                   // + stage
constexpr int kMaxStages = 6;
constexpr int kBarBEmpty = kBarBFull + kMaxStages;   // + stage
constexpr int kBarTmFull = kBarBEmpty + kMaxStages;  // + buffer
constexpr int kBarTmEmpty = kBarTmFull + kAcc;       // + buffer
constexpr int kBarDrain = kBarTmEmpty + kAcc;
constexpr int kNumBars = kBarDrain + 1;

template <int D>
struct PLayout {
  static constexpr int kStages = D == 128 ? 3 : 6;
  static constexpr int kAHalf = kM * 128;                // 128 rows x 64 bf16
  static constexpr int kAPart = kAHalf * (D / 64);
  static constexpr int kBHalf = kN * 128;
  static constexpr int kBStage = kBHalf * (D / 64);
  static constexpr int kA = 0;
  static constexpr int kB = kA + kParts * kAPart;
  static constexpr int kGIdx = kB + kStages * kBStage;  // gather: one tile's row coordinates
  static constexpr int kBar = kGIdx + kN * 4;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 1024;  // + slack to align the base to 1024
};

struct PrParams {
  const int32_t* qn;      // [BH][C_q]
  const int32_t* koff;    // [BH][C_k + 1]
  const float2* nmu;      // [BH][C_k][mtiles * kM]: -s μ as (hi, lo)
  float* E;               // [BH][C_q][C_k]
  const int32_t* kperm;   // gather: original index of each permuted key; nullptr = K_perm given
  int64_t Nk;
  int Cq, Ck, mtiles;
  int64_t nseg;           // BH * mtiles segments of Nk key rows each
  float scale;
  int* status;
  // weight probes (EAR_PROBE_WEIGHTS / EAR_PROBE_VALUE)
  uint32_t* zmax;         // [BH][mtiles * kM] largest logit of each centroid row, ordered bits
  const float2* vst;      // [BH][N_k] per permuted key: (|v_j - v̄_b|^2, (v_j - v̄_b)·v̄_b)
  const float* vnorm;     // [BH][C_k] |v̄_b|^2
};

// Monotone map of a float onto uint32 (0 is below every float), for atomicMax.
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_ordered(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// First cluster b in [0, Ck] with koff[b] >= row (koff is non-decreasing; Ck
// if none).  Called by a whole warp: each round the 32 lanes test 32 evenly
// spaced positions of the remaining interval, so C_k = 500 takes two rounds
// of loads instead of nine dependent ones.
__device__ __forceinline__ int lower_cluster(const int32_t* koff, int Ck, int64_t row) {
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = Ck;  // answer in [lo, hi]
  while (lo < hi) {
    const int step = (hi - lo + 31) / 32;
    const int pos = lo + lane * step;
    const bool ge = pos < hi && (int64_t)koff[pos] >= row;
    const unsigned m = __ballot_sync(0xffffffffu, ge);
    if (m == 0) {
      // every tested position is below row: the answer is past the last one
      lo += min(31, (hi - 1 - lo) / step) * step + 1;
    } else {
      const int f = __ffs(m) - 1;  // first tested position with koff >= row
      hi = lo + f * step;
      lo = f == 0 ? lo : lo + (f - 1) * step + 1;
    }
  }
  return lo;
}

// One segment (slice h, M tile mt) of a CTA's range: key clusters [b0, b1),
// key rows [r0, r1), ntiles tiles of kN keys.
struct Seg {
  int64_t h;
  int mt, b0, b1;
  int32_t r0, r1;
  int ntiles;
};

// The CTA's share of the flattened (segment, key row) space is
// [lo, hi) = [cta * total / ncta, (cta + 1) * total / ncta).  Within segment
// `seg` it owns the clusters whose first row falls in its share; a segment
// whose rows lie wholly outside the share is not visited.
__device__ __forceinline__ bool seg_of(const PrParams& p, int64_t seg, int64_t lo, int64_t hi,
                                       Seg& g) {
  const int64_t s0 = seg * p.Nk, s1 = s0 + p.Nk;
  if (s1 <= lo || s0 >= hi) return false;
  g.h = seg / p.mtiles;
  g.mt = (int)(seg % p.mtiles);
  const int32_t* koff = p.koff + g.h * (int64_t)(p.Ck + 1);
  g.b0 = lo <= s0 ? 0 : lower_cluster(koff, p.Ck, lo - s0);
  g.b1 = hi >= s1 ? p.Ck : lower_cluster(koff, p.Ck, hi - s0);
  g.r0 = g.b0 < g.b1 ? koff[g.b0] : 0;
  g.r1 = g.b0 < g.b1 ? koff[g.b1] : 0;
  if (g.r0 < 0 || g.r1 < g.r0 || g.r1 > p.Nk) {
    latch(p.status, EAR_ERR_DEVICE);
    g.r0 = g.r1 = 0;
  }
  g.ntiles = (int)((g.r1 - g.r0 + kN - 1) / kN);
  return true;
}

// MODE 0: the logit-gap probe.  MODE 1 / 2: the weight / value-aware probes;
// with g = z_j - z̄_b, t = e^g, δ = t - 1 = expm1(g) and u_j = v_j - v̄_b, the
// block sum is w̄_b^2 * sum_j δ^2 (MODE 1) or
// w̄_b^2 * sum_j (t^2 |u_j|^2 + 2 t δ u_j·v̄_b + δ^2 |v̄_b|^2) (MODE 2), since
// w_j = w̄_b t and |t v_j - v̄_b|^2 = |t u_j + δ v̄_b|^2.  This kernel keeps the
// sums (no running maximum is needed for them) and each row's largest logit;
// pr_weigh multiplies by w̄_b^2 = e^{2 (z̄_b - m_a)} once m_a is known.
template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
pr_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmK,
      const PrParams p) {
  using L = PLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int64_t total = p.nseg * p.Nk;
  const int64_t lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  const int64_t seg0 = lo / p.Nk, seg1 = (hi + p.Nk - 1) / p.Nk;  // segments touched

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kBarAFull], 1);
    mbar_init(&bars[kBarAEmpty], 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&bars[kBarBFull + s], 1);
      mbar_init(&bars[kBarBEmpty + s], 1);
    }
    for (int b = 0; b < kAcc; ++b) {
      mbar_init(&bars[kBarTmFull + b], 1);
      mbar_init(&bars[kBarTmEmpty + b], kM);
    }
    mbar_init(&bars[kBarDrain], 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kAcc * kN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmK);
    }
    int64_t t = 0;  // tiles issued so far (ring position)
    int li = 0;     // segments with tiles so far (A buffer phase)
    bool ok = true;
    for (int64_t seg = seg0; ok && seg < seg1; ++seg) {
      Seg g;
      if (!seg_of(p, seg, lo, hi, g) || g.ntiles == 0) continue;
      // the previous segment's MMAs are done with A before it is overwritten
      if (li > 0 && !mbar_wait_warp(&bars[kBarAEmpty], (li - 1) & 1, abort)) break;
      if (leader) {
        mbar_arrive_expect_tx(&bars[kBarAFull], kParts * L::kAPart);
        const int32_t arow = (int32_t)((g.h * p.mtiles + g.mt) * kParts * kM);
        for (int sp = 0; sp < kParts; ++sp)
          for (int hf = 0; hf < D / 64; ++hf)
            tma_load_2d(smem + L::kA + sp * L::kAPart + hf * L::kAHalf, &tmA, &bars[kBarAFull],
                        64 * hf, arow + sp * kM);
      }
      ++li;
      for (int i = 0; i < g.ntiles; ++i, ++t) {
        const int s = (int)(t % L::kStages);
        int4 gi = make_int4(0, 0, 0, 0);
        if (p.kperm != nullptr) {  // rows 4 lane .. 4 lane + 3 of the tile, looked up before the wait;
                                   // rows past the segment repeat its last row
          const int64_t kb = g.h * p.Nk;
          const int32_t j = g.r0 + i * kN + 4 * lane, jl = g.r1 - 1;
          gi.x = gather_row(p.kperm, kb + min(j, jl), g.h, p.Nk, p.status);
          gi.y = gather_row(p.kperm, kb + min(j + 1, jl), g.h, p.Nk, p.status);
          gi.z = gather_row(p.kperm, kb + min(j + 2, jl), g.h, p.Nk, p.status);
          gi.w = gather_row(p.kperm, kb + min(j + 3, jl), g.h, p.Nk, p.status);
        }
        if (t >= L::kStages &&
            !mbar_wait_warp(&bars[kBarBEmpty + s], (int)((t / L::kStages) - 1) & 1, abort)) {
          ok = false;
          break;
        }
        uint8_t* bdst = smem + L::kB + s * L::kBStage;
        if (p.kperm != nullptr) {
          int4* gidx = reinterpret_cast<int4*>(smem + L::kGIdx);
          gidx[lane] = gi;
          __syncwarp();
          if (leader) {
            mbar_arrive_expect_tx(&bars[kBarBFull + s], L::kBStage);
            for (int q4 = 0; q4 < kN / 4; ++q4) {
              const int4 rr = gidx[q4];
              for (int hf = 0; hf < D / 64; ++hf)
                tma_gather4(bdst + hf * L::kBHalf + q4 * 4 * 128, &tmK, &bars[kBarBFull + s],
                            64 * hf, rr);
            }
          }
        } else if (leader) {
          mbar_arrive_expect_tx(&bars[kBarBFull + s], L::kBStage);
          const int32_t row = (int32_t)(g.h * p.Nk + g.r0 + (int64_t)i * kN);
          for (int hf = 0; hf < D / 64; ++hf)
            tma_load_2d(bdst + hf * L::kBHalf, &tmK, &bars[kBarBFull + s], 64 * hf, row);
        }
        __syncwarp();
      }
    }
    if (*abort && leader) {  // let issued loads land before the CTA exits
      if (li > 0) mbar_wait_drain(&bars[kBarAFull], (li - 1) & 1);
      for (int64_t u = t - 1; u >= 0 && u >= t - L::kStages; --u)
        mbar_wait_drain(&bars[kBarBFull + u % L::kStages], (int)(u / L::kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = elect_one();
    const uint32_t idesc = idesc_bf16(kM, kN, false);
    const uint32_t abase = smem_u32(smem + L::kA);
    int64_t t = 0;
    int li = 0;
    bool ok = true;
    for (int64_t seg = seg0; ok && seg < seg1; ++seg) {
      Seg g;
      if (!seg_of(p, seg, lo, hi, g) || g.ntiles == 0) continue;
      ok = mbar_wait_warp(&bars[kBarAFull], li & 1, abort);
      ++li;
      for (int i = 0; ok && i < g.ntiles; ++i, ++t) {
        const int s = (int)(t % L::kStages), buf = (int)(t % kAcc);
        ok = mbar_wait_warp(&bars[kBarBFull + s], (int)(t / L::kStages) & 1, abort);
        if (ok && t >= kAcc)
          ok = mbar_wait_warp(&bars[kBarTmEmpty + buf], (int)((t / kAcc) - 1) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        const uint32_t bbase = smem_u32(smem + L::kB + s * L::kBStage);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * L::kAHalf + (kk % 4) * 32;
          const uint32_t boff = (kk / 4) * L::kBHalf + (kk % 4) * 32;
#pragma unroll
          for (int sp = 0; sp < kParts; ++sp) {
            if (leader)
              mma_ss(tmem + buf * kN, desc_sw128(abase + sp * L::kAPart + off, 16, 1024),
                     desc_sw128(bbase + boff, 16, 1024), idesc, (kk > 0 || sp > 0) ? 1u : 0u);
          }
        }
        if (leader) {
          mma_commit(&bars[kBarTmFull + buf]);
          mma_commit(&bars[kBarBEmpty + s]);
        }
        __syncwarp();
      }
      if (ok && leader) mma_commit(&bars[kBarAEmpty]);  // A free once these MMAs finish
      __syncwarp();
    }
    if (leader) {
      mma_commit(&bars[kBarDrain]);
      mbar_wait_drain(&bars[kBarDrain], 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                // TMEM lane quadrant this warp may read
    const int r = q * 32 + lane;           // centroid row within the M tile
    const uint32_t lane_bits = (uint32_t)(q * 32) << 16;
    const int apad = p.mtiles * kM;
    const float scale = p.scale;
    int64_t t = 0;
    bool ok = true;
    for (int64_t seg = seg0; ok && seg < seg1; ++seg) {
      Seg g;
      if (!seg_of(p, seg, lo, hi, g)) continue;
      const int a = g.mt * kM + r;
      const bool live_a = a < p.Cq && p.qn[g.h * p.Cq + a] > 0;
      const int32_t* koff = p.koff + g.h * (int64_t)(p.Ck + 1);
      const float2* nmu_h = p.nmu + g.h * (int64_t)p.Ck * apad + g.mt * kM + r;
      float* Erow = p.E + (g.h * p.Cq + (a < p.Cq ? a : 0)) * (int64_t)p.Ck;
      // walk state: current cluster cb, its end row, its -s μ (hi, lo), running
      // sum; the next cluster's end and -s μ are loaded one cluster ahead, so
      // moving to it waits on no memory
      int cb = g.b0;
      int32_t cend = cb < g.b1 ? koff[cb + 1] : 0;
      float2 nm = cb < g.b1 ? nmu_h[(int64_t)cb * apad] : make_float2(0.f, 0.f);
      int32_t cend_n = cb + 1 < g.b1 ? koff[cb + 2] : 0;
      float2 nm_n = cb + 1 < g.b1 ? nmu_h[(int64_t)(cb + 1) * apad] : make_float2(0.f, 0.f);
      float acc = 0.f;
      float zm = -INFINITY;  // largest logit of this row seen here (MODE > 0)
      const float2* vst_h = MODE == 2 ? p.vst + g.h * p.Nk : nullptr;
      const float* vn_h = MODE == 2 ? p.vnorm + g.h * p.Ck : nullptr;
      float vn = MODE == 2 && cb < g.b1 ? vn_h[cb] : 0.f;
      float vn_n = MODE == 2 && cb + 1 < g.b1 ? vn_h[cb + 1] : 0.f;
      auto flush = [&]() {  // cluster cb is complete
        if (a < p.Cq) Erow[cb] = live_a ? acc : 0.f;
        acc = 0.f;
        ++cb;
        cend = cend_n;
        nm = nm_n;
        vn = vn_n;
        if (cb + 1 < g.b1) {
          cend_n = koff[cb + 2];
          nm_n = nmu_h[(int64_t)(cb + 1) * apad];
          if (MODE == 2) vn_n = vn_h[cb + 1];
        }
      };
      // one term of the block sum for score value sv (raw S) of key row `row`;
      // st = (|u|^2, u·v̄) of that key (MODE 2)
      auto term = [&](float sv, float2 st) {
        const float gg = fmaf(sv, scale, nm.x) + nm.y;
        if (MODE == 0) return gg * gg;
        zm = fmaxf(zm, sv * scale);
        const float dl = expm1f(gg);
        if (MODE == 1) return dl * dl;
        const float tt = dl + 1.f;
        return fmaf(tt * tt, st.x, fmaf(2.f * tt * dl, st.y, dl * dl * vn));
      };
      for (int i = 0; ok && i < g.ntiles; ++i, ++t) {
        const int buf = (int)(t % kAcc);
        ok = mbar_wait_warp(&bars[kBarTmFull + buf], (int)(t / kAcc) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        const int32_t trow = g.r0 + i * kN;
#pragma unroll 1
        for (int gq = 0; gq < kN / 32; ++gq) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_bits + buf * kN + 32 * gq, v);
          tmem_ld_wait();
          const int32_t gr = trow + 32 * gq;
          if (gr >= g.r1) break;
          // MODE 2: lane l holds key gr + l's statistics, broadcast per column
          float2 stl = make_float2(0.f, 0.f);
          if (MODE == 2 && gr + lane < g.r1) stl = vst_h[gr + lane];
          if (gr + 32 <= cend) {  // the whole group lies in cluster cb (warp-uniform)
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              float2 st0 = make_float2(0.f, 0.f), st1 = st0;
              if (MODE == 2) {
                st0 = make_float2(__shfl_sync(0xffffffffu, stl.x, j), __shfl_sync(0xffffffffu, stl.y, j));
                st1 = make_float2(__shfl_sync(0xffffffffu, stl.x, j + 1),
                                  __shfl_sync(0xffffffffu, stl.y, j + 1));
              }
              s0 += term(__uint_as_float(v[j]), st0);
              s1 += term(__uint_as_float(v[j + 1]), st1);
            }
            acc += s0 + s1;
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              float2 st = make_float2(0.f, 0.f);
              if (MODE == 2)  // every lane joins the shuffle before any break
                st = make_float2(__shfl_sync(0xffffffffu, stl.x, j), __shfl_sync(0xffffffffu, stl.y, j));
              const int32_t row = gr + j;
              if (row >= g.r1) break;
              while (row >= cend && cb < g.b1) flush();  // empty clusters flush as 0
              acc += term(__uint_as_float(v[j]), st);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bars[kBarTmEmpty + buf]);
      }
      if (ok)
        while (cb < g.b1) flush();  // the last cluster, then empty trailing clusters
      if (MODE > 0 && a < p.Cq && zm > -INFINITY)
        atomicMax(p.zmax + g.h * apad + a, ordered_bits(zm));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kAcc * kN);
    if (lane == 0 && *abort) latch(p.status, EAR_ERR_TIMEOUT);
  }
}

// q̄ -> three bf16 parts per element, rows padded to mtiles * 128 with zeros.
// Layout [BH][mtiles][part][128][D].
__global__ void pr_split(const float* __restrict__ qc, uint16_t* __restrict__ out, int Cq,
                         int mtiles, int D, int64_t total) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const int k = (int)(e % D);
  const int64_t rowg = e / D;                 // (h, mt, part, r)
  const int r = (int)(rowg % kM);
  const int sp = (int)((rowg / kM) % kParts);
  const int64_t hm = rowg / ((int64_t)kM * kParts);
  const int mt = (int)(hm % mtiles);
  const int64_t h = hm / mtiles;
  const int a = mt * kM + r;
  float x = a < Cq ? qc[(h * Cq + a) * (int64_t)D + k] : 0.f;
  uint16_t part = 0;
  for (int i = 0; i <= sp; ++i) {
    part = f32_to_bf16(x);
    x -= bf16_to_f32(part);  // exact: the remainder keeps the bits bf16 dropped
  }
  out[e] = part;
}

// -s μ_ab = -s q̄_a·k̄_b in fp64, stored as hi = fp32(value), lo = fp32(value - hi).
// Block = (16 key clusters, a tile of 128 centroid rows, slice); thread = row a.
// Layout [BH][C_k][mtiles * 128] (a fastest), so an epilogue warp reads it
// coalesced.  k̄ is held in shared memory already widened to fp64 (one
// conversion per value and block, not per value and thread); q̄'s rows are
// padded to kM + 1 floats so its transposing stores do not share banks.
constexpr int kMuB = 16;
constexpr int kMuQS = kM + 1;
template <int D>
__global__ void __launch_bounds__(kM)
pr_mu(const float* __restrict__ qc, const float* __restrict__ kc, int Cq, int Ck, int mtiles,
      double scale, float2* __restrict__ nmu) {
  extern __shared__ double mu_smem[];
  double (*ks)[D] = reinterpret_cast<double (*)[D]>(mu_smem);                    // [kMuB][D]
  float (*qs)[kMuQS] = reinterpret_cast<float (*)[kMuQS]>(mu_smem + kMuB * D);  // [D][kM + 1]
  const int b0 = blockIdx.x * kMuB;
  const int mt = blockIdx.y;
  const int64_t h = blockIdx.z;
  const int r = threadIdx.x, a = mt * kM + r;
  for (int e = threadIdx.x; e < kM * D; e += kM) {
    const int rr = e / D, k = e % D, aa = mt * kM + rr;
    qs[k][rr] = aa < Cq ? qc[(h * Cq + aa) * (int64_t)D + k] : 0.f;
  }
  for (int e = threadIdx.x; e < kMuB * D; e += kM) {
    const int bb = b0 + e / D;
    ks[e / D][e % D] = bb < Ck ? (double)kc[(h * Ck + bb) * (int64_t)D + e % D] : 0.0;
  }
  __syncthreads();
  double acc[kMuB];
#pragma unroll
  for (int i = 0; i < kMuB; ++i) acc[i] = 0.0;
  for (int k = 0; k < D; ++k) {
    const double qv = (double)qs[k][r];
#pragma unroll
    for (int i = 0; i < kMuB; ++i) acc[i] = fma(qv, ks[i][k], acc[i]);
  }
  const int apad = mtiles * kM;
#pragma unroll
  for (int i = 0; i < kMuB; ++i) {
    const int b = b0 + i;
    if (b < Ck) {
      const double v = -scale * acc[i];
      const float hi = (float)v;
      nmu[(h * Ck + b) * (int64_t)apad + a] = make_float2(hi, (float)(v - (double)hi));
    }
  }
}

// Weight probes: E[a][b] *= e^{2 (z̄_ab - m_a)}, m_a = the row's largest logit
// over every key of the slice.  Block = (centroid row a, slice).
__global__ void pr_weigh(float* __restrict__ E, const float2* __restrict__ nmu,
                         const uint32_t* __restrict__ zmax, int Cq, int Ck, int apad) {
  const int a = blockIdx.x;
  const int64_t h = blockIdx.y;
  const uint32_t mb = zmax[h * apad + a];
  const float m = from_ordered(mb);
  float* row = E + (h * Cq + a) * (int64_t)Ck;
  for (int b = threadIdx.x; b < Ck; b += blockDim.x) {
    const float2 nm = nmu[(h * Ck + b) * (int64_t)apad + a];
    const float zbar = -(nm.x + nm.y);
    row[b] = mb == 0 ? 0.f : row[b] * expf(2.f * (zbar - m));
  }
}

// Per permuted key j of cluster b: (|v_j - v̄_b|^2, (v_j - v̄_b)·v̄_b), and
// |v̄_b|^2.  Block = (key cluster, slice); a warp per key row, lanes over d.
// perm != nullptr: V is in original order and permuted row j is V[perm[j]].
template <int D>
__global__ void pr_vstats(const uint16_t* __restrict__ V, const int32_t* __restrict__ perm,
                          const float* __restrict__ vc, const int32_t* __restrict__ koff,
                          int64_t Nk, int Ck, float2* __restrict__ vst,
                          float* __restrict__ vnorm, int* status) {
  constexpr int kPer = D / 32;
  const int b = blockIdx.x;
  const int64_t h = blockIdx.y;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int32_t* oh = koff + h * (int64_t)(Ck + 1);
  int32_t r0 = oh[b], r1 = oh[b + 1];
  if (r0 < 0 || r1 < r0 || r1 > Nk) {
    if (threadIdx.x == 0) latch(status, EAR_ERR_DEVICE);
    r0 = r1 = 0;
  }
  float cb[kPer];
  float nv = 0.f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    cb[i] = vc[(h * Ck + b) * (int64_t)D + lane * kPer + i];
    nv = fmaf(cb[i], cb[i], nv);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) nv += __shfl_xor_sync(0xffffffffu, nv, off);
  if (threadIdx.x == 0) vnorm[h * Ck + b] = nv;
  for (int32_t j = r0 + w; j < r1; j += nw) {
    const int64_t src = perm != nullptr ? gather_row(perm, h * Nk + j, h, Nk, status) : h * Nk + j;
    const uint16_t* row = V + src * D + lane * kPer;
    float uu = 0.f, uv = 0.f;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const float u = bf16_to_f32(row[i]) - cb[i];
      uu = fmaf(u, u, uu);
      uv = fmaf(u, cb[i], uv);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      uu += __shfl_xor_sync(0xffffffffu, uu, off);
      uv += __shfl_xor_sync(0xffffffffu, uv, off);
    }
    if (lane == 0) vst[h * Nk + j] = make_float2(uu, uv);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D bf16 map over [rows][d], 64-column x box_rows boxes, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int mtiles_of(int32_t c_q) { return (int)ceil_div(c_q, kM); }

struct PrWs {
  uint16_t* qsplit;
  float2* nmu;
  uint32_t* zmax;
  float2* vst;
  float* vnorm;
};

PrWs carve(Carver& cv, int64_t bh, int64_t n_k, int32_t d, int32_t c_q, int32_t c_k) {
  const int mt = mtiles_of(c_q);
  PrWs w;
  w.qsplit = cv.take<uint16_t>((size_t)bh * mt * kParts * kM * d);
  w.nmu = cv.take<float2>((size_t)bh * c_k * mt * kM);
  w.zmax = cv.take<uint32_t>((size_t)bh * mt * kM);
  w.vst = cv.take<float2>((size_t)bh * n_k);
  w.vnorm = cv.take<float>((size_t)bh * c_k);
  return w;
}

template <int D, int MODE>
ear_status run_tc(const float* qc, const int32_t* qn, const float* kc, const void* K,
                  const int32_t* kperm, const int32_t* koff, int64_t bh, int64_t n_k, int32_t c_q,
                  int32_t c_k,
                  float scale, const void* V, const float* vc, float* E, void* ws,
                  cudaStream_t s) {
  using L = PLayout<D>;
  Carver cv(ws);
  PrWs w = carve(cv, bh, n_k, D, c_q, c_k);
  const int mt = mtiles_of(c_q);
  const int64_t total = bh * mt * kParts * kM * D;
  pr_split<<<(unsigned)ceil_div(total, 256), 256, 0, s>>>(qc, w.qsplit, c_q, mt, D, total);
  EAR_TRY(after_launch());
  const int mu_smem = kMuB * D * (int)sizeof(double) + D * kMuQS * (int)sizeof(float);
  EAR_CUDA(cudaFuncSetAttribute(pr_mu<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, mu_smem));
  pr_mu<D><<<dim3((unsigned)ceil_div(c_k, kMuB), (unsigned)mt, (unsigned)bh), kM, mu_smem, s>>>(
      qc, kc, c_q, c_k, mt, (double)scale, w.nmu);
  EAR_TRY(after_launch());
  CUtensorMap ma, mk;
  if (!make_map(&ma, w.qsplit, bh * mt * kParts * kM, D, kM) ||
      !make_map(&mk, K, bh * n_k, D, kperm != nullptr ? 1 : kN))
    return EAR_ERR_CUDA;
  // Persistent: one CTA per SM (at most), each a contiguous share of the
  // (slice, M tile, key row) space, about 2048 key rows at least.
  const int64_t nseg = bh * mt;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(148, nseg * n_k / 2048));
  PrParams p;
  p.qn = qn;
  p.koff = koff;
  p.nmu = w.nmu;
  p.E = E;
  p.kperm = kperm;
  p.Nk = n_k;
  p.Cq = c_q;
  p.Ck = c_k;
  p.mtiles = mt;
  p.nseg = nseg;
  p.scale = scale;
  p.status = device_status_word();
  p.zmax = w.zmax;
  p.vst = w.vst;
  p.vnorm = w.vnorm;
  if (MODE > 0) EAR_CUDA(cudaMemsetAsync(w.zmax, 0, sizeof(uint32_t) * bh * mt * kM, s));
  if (MODE == 2) {
    pr_vstats<D><<<dim3((unsigned)c_k, (unsigned)bh), 128, 0, s>>>(
        static_cast<const uint16_t*>(V), kperm, vc, koff, n_k, c_k, w.vst, w.vnorm, p.status);
    EAR_TRY(after_launch());
  }
  EAR_CUDA(cudaFuncSetAttribute(pr_tc<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                L::kBytes));
  pr_tc<D, MODE><<<grid, kThreads, L::kBytes, s>>>(ma, mk, p);
  EAR_TRY(after_launch());
  if (MODE > 0) {
    pr_weigh<<<dim3((unsigned)c_q, (unsigned)bh), 128, 0, s>>>(E, w.nmu, w.zmax, c_q, c_k,
                                                              mt * kM);
    EAR_TRY(after_launch());
  }
  return after_launch();
}

}  // namespace

size_t probe_tc_workspace(int64_t bh, int64_t n_k, int32_t d, int32_t c_q, int32_t c_k) {
  Carver cv(nullptr);
  carve(cv, bh, n_k, d, c_q, c_k);
  return cv.used;
}

ear_status probe_tc_run(const float* qc, const int32_t* qn, const float* kc, const void* K,
                        const int32_t* kperm, const int32_t* koff, int64_t bh, int64_t n_k,
                        int32_t d, int32_t c_q, int32_t c_k, float scale, int32_t mode,
                        const void* V, const float* vc, float* E, void* ws, cudaStream_t s) {
  if (bh * n_k > INT32_MAX) return EAR_ERR_UNSUPPORTED;  // TMA row coordinates are int32
#define EAR_PR(DD, MM) \
  run_tc<DD, MM>(qc, qn, kc, K, kperm, koff, bh, n_k, c_q, c_k, scale, V, vc, E, ws, s)
  if (d == 64)
    return mode == 0 ? EAR_PR(64, 0) : mode == 1 ? EAR_PR(64, 1) : EAR_PR(64, 2);
  return mode == 0 ? EAR_PR(128, 0) : mode == 1 ? EAR_PR(128, 1) : EAR_PR(128, 2);
#undef EAR_PR
}

}  // namespace ear
