// Lloyd k-means on the sm_100a tensor cores (SVG-EAR §4.1: Q and K are
// clustered and each token is represented by the mean token of its cluster).
// Used for bf16 inputs with C <= 2048 centroids; labels are exact.  Up to 512
// centroids sit in shared memory at a time: beyond that km_tc runs in passes
// of 512 centroids, each row's candidate state carried between passes in
// global memory, and only the last pass decides.
//
// Per call:
//   km_xprep     X (bf16) -> fp16 copy Xh plus ||x|| per row.  A row with a
//                value beyond the fp16 range gets ||x|| = +inf (always re-decided).
//   km_cprep     centroids -> fp16 copy, fp32 ||c||^2 (+inf on padding
//                columns), per-slice max ||c||.
// Per iteration:
//   km_tc        one CTA = up to 16 tiles of 128 rows of one slice.  The
//                slice's fp16 centroids stay in shared memory; a TMA warp
//                streams X tiles, one thread issues tcgen05.mma
//                (S = X C^T, fp32, 256-column chunks, two TMEM buffers) and
//                two epilogue warpgroups scan each chunk (alternate 32-column
//                groups; with one chunk per tile and one pass, C <= 256,
//                alternate tiles instead, one TMEM buffer each, so two tiles
//                are decided at once and no merge is needed) in one pass:
//                the minimum of d~_c = ||c||^2 - 2 x.c^ is taken group by
//                group, and a group whose minimum lies within the rounding
//                margin of the running minimum is searched for candidates
//                from the same registers.  Each warpgroup
//                keeps its four best candidates by distance and the smallest
//                distance it had to drop.  One candidate within the margin of
//                the row's minimum = a certain label; 2-4 go to an fp64
//                decision among them; more (a dropped candidate within the
//                margin, or a row / centroid without an exact fp16 copy) go
//                to a full fp64 decision.  Each row's outcome is a
//                byte of its own (moved / pick with n candidates / full), the
//                candidates and the old label go to per-row slots: plain
//                coalesced stores, no list counters.
//   km_resolve   one warp per 32-row window of those bytes: moves (sums[new]
//                += x, sums[old] -= x, counts likewise, vector fp32 atomics),
//                picks (fp64 distances of the 2-4 candidates in the order
//                sum_k (x_k - c_k)^2, k = 0..d-1, ties to the lowest index;
//                eight rows per warp) and full decisions (the same over all C
//                centroids, four per lane at a time), each followed by its
//                move.  After the first iteration only moved rows cost atomics.
//   km_finalize  centroid = sum / count (empty clusters keep theirs), and the
//                fp16 copy / norms / max norm for the next iteration.
//
// Rounding bound of the approximate distance d~_c = ||c||^2 - 2 x.c^ (c^ =
// fp16(c), products exact, fp32 accumulation over d terms, ||c||^2 in fp32):
//   |d~_c - (||x - c||^2 - ||x||^2)| <= a ||x|| Cmax + b Cmax^2
//                                            + s (||x|| + Cmax)
//   a = 2 (2^-11 + (d + 1) 2^-23)(1 + 2^-11) (1 + 2^-20),  b = 2^-16,
//   s = 2 sqrt(d) 2^-25 (centroid or x values in the fp16 subnormal range
//   round with absolute error <= 2^-25)
// (Cauchy-Schwarz turns sum |x_k c_k| into ||x|| ||c||, Cmax = max ||c||.)
// A centroid value beyond the fp16 range makes its slice fall back to fp64
// for every row; an X row with a value beyond it always does.
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "ear_internal.cuh"
#include "sm100.cuh"

namespace ear {
namespace {

using namespace sm100;

constexpr int kTileRows = 128;
constexpr int kTilesPerCta = 16;
constexpr int kColChunk = 256;
constexpr int kMaxCPad = 512;     // centroids of one km_tc pass
constexpr int kMaxCTotal = 2048;  // centroids over all passes
constexpr int kXStages = 2;
constexpr int kThreads = 384;  // warp 0 TMA, warp 1 MMA, warps 4-11 epilogue

constexpr int kBarXFull = 0;    // + stage
constexpr int kBarXEmpty = 2;   // + stage
constexpr int kBarCFull = 4;
constexpr int kBarTmFull = 5;   // + buffer
constexpr int kBarTmEmpty = 7;  // + buffer
constexpr int kBarDrain = 9;
constexpr int kNumBars = 10;

__host__ __device__ constexpr uint32_t idesc_f16(uint32_t m, uint32_t n) {
  return (1u << 4) | ((n >> 3) << 17) | ((m >> 4) << 24);  // D f32, A/B f16, K-major
}

template <int D>
struct KLayout {
  static constexpr int kXHalf = kTileRows * 128;
  static constexpr int kXTile = kXHalf * (D / 64);
  static constexpr int kCHalf = kMaxCPad * 128;
  static constexpr int kC = 0;
  static constexpr int kX = kC + kCHalf * (D / 64);
  static constexpr int kNorm = kX + kXStages * kXTile;
  static constexpr int kXchg = kNorm + kMaxCPad * 4;   // [2][128] x 10 words
  static constexpr int kBar = kXchg + 2 * kTileRows * 40;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16 + 1024;
};

// per-row outcome byte: bits 0-1 kind, bits 2-4 pick candidate count
constexpr uint8_t kKindNone = 0;    // certain, label unchanged
constexpr uint8_t kKindMove = 1;    // certain, label changed (old label in `from`)
constexpr uint8_t kKindPick = 2;    // 2-4 candidates in `cand`
constexpr uint8_t kKindFull = 3;    // fp64 decision over every centroid

struct KmTcParams {
  const float* xnorm;       // [BH*N]
  const float* cnorm;       // [BH*C_pad]
  const float* cmax;        // [BH]
  const int* cbad;          // [BH] a centroid of the slice has no finite fp16 copy
  int32_t* labels;          // [BH*N]
  uint8_t* kind;            // [BH*N] outcome byte
  int4* cand;               // [BH*N] pick candidates
  int32_t* from;            // [BH*N] old label of a moved row
  int64_t N;
  int C, C_pad, first;
  int c_box;  // rows per centroid TMA box (min(256, C_pad))
  int c0, cp_pass;             // this pass: centroids [c0, c0 + cp_pass) of the padded C_pad
  int carry_in, carry_out;     // read / write the row state of earlier / later passes
  float* st_run;               // [BH*N] smallest d~ so far
  float* st_drop;              // [BH*N] smallest d~ pushed out of a candidate list
  int4* st_cand;               // [BH*N] up to four candidates (global centroid index, -1 = none)
  float4* st_dist;             // [BH*N] their d~
  float a_coef, b_coef, s_coef;
};

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// min over 32 columns of d~ = cn - 2 v, four independent chains of
// three-input minima; the norms come in as 16-byte loads
__device__ __forceinline__ float group_min(const uint32_t (&v)[32], const float* cn) {
  const unsigned long long m2 = 0xC0000000C0000000ull;  // (-2.f, -2.f)
  const float4* c4 = reinterpret_cast<const float4*>(cn);
  float m[4] = {__int_as_float(0x7f800000), __int_as_float(0x7f800000),
                __int_as_float(0x7f800000), __int_as_float(0x7f800000)};
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    const float4 cc = c4[k / 4];
    const unsigned long long c01 =
        (unsigned long long)__float_as_uint(cc.x) | ((unsigned long long)__float_as_uint(cc.y) << 32);
    const unsigned long long c23 =
        (unsigned long long)__float_as_uint(cc.z) | ((unsigned long long)__float_as_uint(cc.w) << 32);
    const unsigned long long v01 = (unsigned long long)v[k] | ((unsigned long long)v[k + 1] << 32);
    const unsigned long long v23 =
        (unsigned long long)v[k + 2] | ((unsigned long long)v[k + 3] << 32);
    unsigned long long d01, d23;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d01) : "l"(v01), "l"(m2), "l"(c01));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d23) : "l"(v23), "l"(m2), "l"(c23));
    const int a = (k / 4) & 3;
    m[a] = min3f(m[a], __uint_as_float((uint32_t)d01), __uint_as_float((uint32_t)(d01 >> 32)));
    m[a] = min3f(m[a], __uint_as_float((uint32_t)d23), __uint_as_float((uint32_t)(d23 >> 32)));
  }
  return fminf(fminf(m[0], m[1]), fminf(m[2], m[3]));
}

// bit k set where d~ of column k is <= thr (the same packed fma as group_min,
// so a column's d~ is bit-identical in both)
__device__ __forceinline__ uint32_t group_hits(const uint32_t (&v)[32], const float* cn, float thr) {
  const unsigned long long m2 = 0xC0000000C0000000ull;  // (-2.f, -2.f)
  const float4* c4 = reinterpret_cast<const float4*>(cn);
  uint32_t hit = 0;
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    const float4 cc = c4[k / 4];
    const unsigned long long c01 =
        (unsigned long long)__float_as_uint(cc.x) | ((unsigned long long)__float_as_uint(cc.y) << 32);
    const unsigned long long c23 =
        (unsigned long long)__float_as_uint(cc.z) | ((unsigned long long)__float_as_uint(cc.w) << 32);
    const unsigned long long v01 = (unsigned long long)v[k] | ((unsigned long long)v[k + 1] << 32);
    const unsigned long long v23 =
        (unsigned long long)v[k + 2] | ((unsigned long long)v[k + 3] << 32);
    unsigned long long d01, d23;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d01) : "l"(v01), "l"(m2), "l"(c01));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d23) : "l"(v23), "l"(m2), "l"(c23));
    hit |= (__uint_as_float((uint32_t)d01) <= thr ? 1u : 0u) << k;
    hit |= (__uint_as_float((uint32_t)(d01 >> 32)) <= thr ? 1u : 0u) << (k + 1);
    hit |= (__uint_as_float((uint32_t)d23) <= thr ? 1u : 0u) << (k + 2);
    hit |= (__uint_as_float((uint32_t)(d23 >> 32)) <= thr ? 1u : 0u) << (k + 3);
  }
  return hit;
}

// TP: tile-parallel epilogue (one 256-column chunk per tile and one pass:
// the launcher picks it only then).
template <int D, bool TP>
__global__ void __launch_bounds__(kThreads, 1)
km_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
      const KmTcParams p, int* status) {
  using L = KLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int64_t h = blockIdx.y;
  const int64_t tile0 = (int64_t)blockIdx.x * kTilesPerCta;
  const int64_t ntiles_slice = (p.N + kTileRows - 1) / kTileRows;
  const int64_t left = ntiles_slice - tile0;
  const int ntiles = (int)(left < kTilesPerCta ? left : kTilesPerCta);
  if (ntiles <= 0) return;
  const int nch = (p.cp_pass + kColChunk - 1) / kColChunk;
  // tile-parallel epilogue: each warpgroup decides every other tile on its own
  constexpr bool tp = TP;
  constexpr int kNg = TP ? 8 : 4;  // column groups of a chunk one warpgroup scans
  if (TP && (nch != 1 || p.carry_in || p.carry_out)) {
    if (threadIdx.x == 0) latch(status, EAR_ERR_DEVICE);
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  float* cn = reinterpret_cast<float*>(smem + L::kNorm);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(&bars[kBarXFull + s], 1);
      mbar_init(&bars[kBarXEmpty + s], 1);
    }
    mbar_init(&bars[kBarCFull], 1);
    mbar_init(&bars[kBarDrain], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[kBarTmFull + b], 1);
      mbar_init(&bars[kBarTmEmpty + b], tp ? 128 : 256);
    }
    *abort = 0;
    fence_barrier_init();
  }
  for (int c = threadIdx.x; c < kMaxCPad; c += kThreads)
    cn[c] = c < p.cp_pass ? p.cnorm[h * p.C_pad + p.c0 + c] : __int_as_float(0x7f800000);
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmC);
      // whole boxes land (rows past the pass see cn = +inf and never win)
      const int nbox = (p.cp_pass + p.c_box - 1) / p.c_box;
      mbar_arrive_expect_tx(&bars[kBarCFull], nbox * p.c_box * D * 2);
      for (int r = 0; r < nbox * p.c_box; r += p.c_box)
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_2d(smem + L::kC + hf * L::kCHalf + r * 128, &tmC, &bars[kBarCFull], 64 * hf,
                      (int32_t)(h * p.C_pad + p.c0) + r);
    }
    int issued = 0;
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % kXStages;
      if (t >= kXStages && !mbar_wait(&bars[kBarXEmpty + s], ((t / kXStages) - 1) & 1, abort))
        break;
      issued = t + 1;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars[kBarXFull + s], L::kXTile);
        const int32_t row = (int32_t)(h * p.N + (tile0 + t) * kTileRows);
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_2d(smem + L::kX + s * L::kXTile + hf * L::kXHalf, &tmX, &bars[kBarXFull + s],
                      64 * hf, row);
      }
      __syncwarp();
    }
    if (*abort) {
      mbar_wait_drain(&bars[kBarCFull], 0);
      for (int t = issued - 1; t >= 0 && t >= issued - kXStages; --t)
        mbar_wait_drain(&bars[kBarXFull + t % kXStages], (t / kXStages) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&bars[kBarCFull], 0, abort);
      const uint32_t cb = smem_u32(smem + L::kC);
      for (int t = 0; ok && t < ntiles; ++t) {
        const int s = t % kXStages;
        ok = mbar_wait(&bars[kBarXFull + s], (t / kXStages) & 1, abort);
        if (!ok) break;
        const uint32_t xb = smem_u32(smem + L::kX + s * L::kXTile);
        for (int j = 0; j < nch; ++j) {
          const int i = t * nch + j, b = i & 1;
          if (i >= 2) {
            ok = mbar_wait(&bars[kBarTmEmpty + b], ((i >> 1) - 1) & 1, abort);
            if (!ok) break;
          }
          tc_fence_after();
          const int n = min(kColChunk, p.cp_pass - j * kColChunk);
          const uint32_t idesc = idesc_f16(128, (uint32_t)n);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t xo = (kk / 4) * L::kXHalf + (kk % 4) * 32;
            const uint32_t co = (kk / 4) * L::kCHalf + j * kColChunk * 128 + (kk % 4) * 32;
            mma_ss(tmem + b * kColChunk, desc_sw128(xb + xo, 16, 1024),
                   desc_sw128(cb + co, 16, 1024), idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars[kBarTmFull + b]);
        }
        if (ok) mma_commit(&bars[kBarXEmpty + s]);
      }
      mma_commit(&bars[kBarDrain]);
      mbar_wait_drain(&bars[kBarDrain], 0);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue
    const int w = (warp - 4) >> 2;       // warpgroup: column groups g with g % 2 == w
    const int q = warp & 3;
    const int r = q * 32 + lane;         // row within the tile = TMEM lane
    const uint32_t lane_bits = (uint32_t)(q * 32) << 16;
    // exchange [2 tiles][128 rows]: running min, count, 4 candidates, 4 distances
    float* xrun = reinterpret_cast<float*>(smem + L::kXchg);
    int* xcnt = reinterpret_cast<int*>(xrun + 2 * kTileRows);
    int* xcand = xcnt + 2 * kTileRows;                                    // [.][4]
    float* xdist = reinterpret_cast<float*>(xcand + 8 * kTileRows);       // [.][4]
    const float inf = __int_as_float(0x7f800000);
    const float cmax = p.cmax[h];
    const bool cbad = p.cbad[h] != 0;
    bool ok = true;
    // ||x|| and the old label of the next tile's row are loaded a tile ahead
    auto row_of = [&](int t) { return (tile0 + t) * kTileRows + r; };
    // tp: this warpgroup's tiles are w, w + 2, ...; it decides them alone
    const int t_first = tp ? w : 0, t_step = tp ? 2 : 1;
    const bool decider = tp || w == 0;
    float xn_next = 0.f;
    int old_next = -1;
    if (t_first < ntiles) {
      const int64_t r0 = row_of(t_first);
      xn_next = r0 < p.N ? p.xnorm[h * p.N + r0] : 0.f;
      old_next = (decider && !p.first && r0 < p.N) ? p.labels[h * p.N + r0] : -1;
    }
    for (int t = t_first; t < ntiles; t += t_step) {
      const int64_t row = row_of(t);
      const bool valid = row < p.N;
      const int64_t g = h * p.N + row;
      const float xn = xn_next;
      const int old_pre = old_next;
      if (t + t_step < ntiles) {
        const int64_t rn = row_of(t + t_step);
        xn_next = rn < p.N ? p.xnorm[h * p.N + rn] : 0.f;
        old_next = (decider && !p.first && rn < p.N) ? p.labels[h * p.N + rn] : -1;
      }
      const float margin =
          2.f * (p.a_coef * xn * cmax + p.b_coef * cmax * cmax + p.s_coef * (xn + cmax));
      float run = inf;
      // the four best candidates so far, ascending d~ (inf = empty), and the
      // smallest d~ of any candidate pushed out of them
      int c0 = -1, c1 = -1, c2 = -1, c3 = -1;
      float d0 = inf, d1 = inf, d2 = inf, d3 = inf, dropped = inf;
      auto insert = [&](int c, float dv) {
        dropped = fminf(dropped, fmaxf(dv, d3));  // inf while a slot is free
        if (dv < d3) {
          if (dv < d2) {
            c3 = c2; d3 = d2;
            if (dv < d1) {
              c2 = c1; d2 = d1;
              if (dv < d0) { c1 = c0; d1 = d0; c0 = c; d0 = dv; } else { c1 = c; d1 = dv; }
            } else { c2 = c; d2 = dv; }
          } else { c3 = c; d3 = dv; }
        }
      };
      for (int j = 0; j < nch && ok; ++j) {
        const int i = t * nch + j, b = i & 1;
        ok = mbar_wait_warp(&bars[kBarTmFull + b], (i >> 1) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        const int n = min(kColChunk, p.cp_pass - j * kColChunk);
        const uint32_t tbuf = tmem + lane_bits + b * kColChunk;
        // This warpgroup's column groups of the chunk: gg = w + 2u, u = 0..3
        // (tp: all eight, gg = u), two per TMEM wait, each minimum in four
        // independent chains.  Columns past C_pad see cn = +inf; stale TMEM
        // there turns into +inf or NaN, and NaN never wins a comparison.
        // One pass: each pair of groups is read from TMEM once; the running
        // minimum moves group by group and a group whose minimum lies within
        // the margin of it is searched for candidates from the same registers
        // (the running threshold is never below the row's final minimum +
        // margin, so every final candidate is inserted or counted as dropped).
        auto scan = [&](const uint32_t (&v)[32], float gm, int gg) {
          run = fminf(run, gm);
          const float thr = run + margin;
          if (!__any_sync(0xffffffffu, gm <= thr)) return;
          if (gm > thr) return;
          const int cbase = j * kColChunk + 32 * gg;
          uint32_t hit = group_hits(v, cn + cbase, thr);
          if ((hit & (hit - 1)) == 0) {
            if (hit) insert(p.c0 + cbase + __ffs(hit) - 1, gm);
            hit = 0;
          }
          while (hit) {
            const int k = __ffs(hit) - 1;
            hit &= hit - 1;
            uint32_t vk = 0;
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) vk = kk == k ? v[kk] : vk;
            insert(p.c0 + cbase + k, fmaf(-2.f, __uint_as_float(vk), cn[cbase + k]));
          }
        };
#pragma unroll
        for (int u = 0; u < kNg; u += 2) {
          const int ga = tp ? u : w + 2 * u, gb = tp ? u + 1 : w + 2 * (u + 1);
          uint32_t va[32], vb[32];
          const bool has_a = ga * 32 < n, has_b = gb * 32 < n;
          if (has_a) tmem_ld32(tbuf + 32 * ga, va);
          if (has_b) tmem_ld32(tbuf + 32 * gb, vb);
          tmem_ld_wait();
          if (has_a) scan(va, group_min(va, cn + j * kColChunk + 32 * ga), ga);
          if (has_b) scan(vb, group_min(vb, cn + j * kColChunk + 32 * gb), gb);
        }
        tc_fence_before();
        mbar_arrive(&bars[kBarTmEmpty + b]);
      }
      const int xo = (t & 1) * kTileRows + r;
      if (w == 1 && !tp) {
        xrun[xo] = run;
        reinterpret_cast<float*>(xcnt)[xo] = dropped;
        xcand[4 * xo + 0] = c0; xcand[4 * xo + 1] = c1; xcand[4 * xo + 2] = c2; xcand[4 * xo + 3] = c3;
        xdist[4 * xo + 0] = d0; xdist[4 * xo + 1] = d1; xdist[4 * xo + 2] = d2; xdist[4 * xo + 3] = d3;
      }
      if (!tp) named_bar(1, 256);
      if (decider && ok && valid) {
        // this warpgroup's list, the other warpgroup's, and (after the first
        // pass) the state earlier passes carried for the row
        float best = run;
        float drop = dropped;
        int cs[12];
        float ds[12];
        cs[0] = c0; cs[1] = c1; cs[2] = c2; cs[3] = c3;
        ds[0] = d0; ds[1] = d1; ds[2] = d2; ds[3] = d3;
        if (!tp) {  // the other warpgroup's list
          best = fminf(run, xrun[xo]);
          drop = fminf(dropped, reinterpret_cast<const float*>(xcnt)[xo]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          cs[4 + u] = tp ? -1 : xcand[4 * xo + u];
          ds[4 + u] = tp ? inf : xdist[4 * xo + u];
          cs[8 + u] = -1;
          ds[8 + u] = inf;
        }
        if (p.carry_in) {
          best = fminf(best, p.st_run[g]);
          drop = fminf(drop, p.st_drop[g]);
          const int4 cc = p.st_cand[g];
          const float4 dd = p.st_dist[g];
          cs[8] = cc.x; cs[9] = cc.y; cs[10] = cc.z; cs[11] = cc.w;
          ds[8] = dd.x; ds[9] = dd.y; ds[10] = dd.z; ds[11] = dd.w;
        }
        const float lim = best + margin;
        if (p.carry_out) {
          // the four smallest candidates within the margin go on; the
          // smallest one pushed out joins the dropped minimum
          c0 = c1 = c2 = c3 = -1;
          d0 = d1 = d2 = d3 = dropped = inf;
#pragma unroll
          for (int u = 0; u < 12; ++u)
            if (cs[u] >= 0 && ds[u] <= lim) insert(cs[u], ds[u]);
          p.st_run[g] = best;
          p.st_drop[g] = fminf(drop, dropped);
          p.st_cand[g] = make_int4(c0, c1, c2, c3);
          p.st_dist[g] = make_float4(d0, d1, d2, d3);
        }
        int keep = 0, kc[4] = {0, 0, 0, 0};
        // a candidate pushed out of any list that is still within the
        // margin of the row's minimum forces the full decision
        bool full = cbad || !(margin < inf) || drop <= lim;
#pragma unroll
        for (int u = 0; u < 12; ++u) {
          const bool live = cs[u] >= 0 && ds[u] <= lim;
          if (live) {
            if (keep < 4) {
              kc[0] = keep == 0 ? cs[u] : kc[0];
              kc[1] = keep == 1 ? cs[u] : kc[1];
              kc[2] = keep == 2 ? cs[u] : kc[2];
              kc[3] = keep == 3 ? cs[u] : kc[3];
            }
            ++keep;
          }
        }
        full = full || keep == 0 || keep > 4;
        if (!p.carry_out) {
          const int old = old_pre;
          uint8_t kind = kKindFull;
          if (!full && keep == 1) {
            p.labels[g] = kc[0];
            kind = kc[0] != old ? kKindMove : kKindNone;
            if (kind == kKindMove) p.from[g] = old;
          } else if (!full) {
            kind = (uint8_t)(kKindPick | (keep << 2));
            p.cand[g] = make_int4(kc[0], kc[1], kc[2], kc[3]);
          }
          p.kind[g] = kind;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort) latch(status, EAR_ERR_TIMEOUT);
}

// X -> fp16 copy and ||x|| (fp32, rounded up); +inf if the copy overflows.
// (Below the fp16 normal range the copy rounds with absolute error <= 2^-25,
// which the certification margin covers.)
// A row is D/8 lanes of 8 values (16-byte loads and stores).
template <int D>
__global__ void km_xprep(const uint16_t* __restrict__ X, __half* __restrict__ Xh,
                         float* __restrict__ xnorm, int64_t rows) {
  constexpr int kLanes = D / 8;
  constexpr int kRowsPerWarp = 32 / kLanes;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanes, part = lane % kLanes;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t g0 = warp * kRowsPerWarp; g0 < rows; g0 += nw * kRowsPerWarp) {
    const int64_t g = g0 + sub;
    float ss = 0.f;
    bool exact = true;
    if (g < rows) {
      const uint4 raw = reinterpret_cast<const uint4*>(X + g * D)[part];
      const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
      uint32_t out[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float lo = __uint_as_float(w4[u] << 16), hi = __uint_as_float(w4[u] & 0xFFFF0000u);
        const __half hl = __float2half_rn(lo), hh = __float2half_rn(hi);
        exact &= fabsf(lo) <= 65504.f && fabsf(hi) <= 65504.f;  // else the copy overflows
        ss = fmaf(lo, lo, fmaf(hi, hi, ss));
        out[u] = (uint32_t)__half_as_ushort(hl) | ((uint32_t)__half_as_ushort(hh) << 16);
      }
      reinterpret_cast<uint4*>(Xh + g * D)[part] = make_uint4(out[0], out[1], out[2], out[3]);
    }
#pragma unroll
    for (int off = kLanes / 2; off >= 1; off >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, off);
      exact = __shfl_xor_sync(0xffffffffu, (int)exact, off) && exact;
    }
    if (part == 0 && g < rows)
      xnorm[g] = exact ? sqrtf(ss) * (1.f + 1.0e-6f) : __int_as_float(0x7f800000);
  }
}

// A centroid value beyond the fp16 range has no finite copy: the slice is
// flagged (every row then takes the fp64 decision) and the copy is zeroed.
__device__ __forceinline__ void prep_row(const float* __restrict__ c, __half* __restrict__ ch,
                                         float* __restrict__ cnorm, float* __restrict__ cmax,
                                         int* __restrict__ cbad, int D, bool real) {
  const int lane = threadIdx.x & 31;
  float ss = 0.f;
  bool finite = true;
  for (int k = lane; k < D; k += 32) {
    const float v = real ? c[k] : 0.f;
    finite &= fabsf(v) <= 65504.f;
    ss = fmaf(v, v, ss);
  }
  finite = __all_sync(0xffffffffu, finite);
  for (int k = lane; k < D; k += 32) ch[k] = __float2half_rn(finite && real ? c[k] : 0.f);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (lane == 0) {
    *cnorm = real ? ss : __int_as_float(0x7f800000);
    if (real) atomicMax(reinterpret_cast<int*>(cmax), __float_as_int(sqrtf(ss) * (1.f + 1.0e-6f)));
    if (!finite) atomicOr(cbad, 1);
  }
}

__global__ void km_cprep(const float* __restrict__ cent, __half* __restrict__ ch,
                         float* __restrict__ cnorm, float* __restrict__ cmax,
                         int* __restrict__ cbad, int C, int C_pad, int D, int64_t rows_pad) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp >= rows_pad) return;
  const int64_t h = warp / C_pad;
  const int c = (int)(warp % C_pad);
  prep_row(cent + (h * C + (c < C ? c : 0)) * D, ch + warp * D, cnorm + warp, cmax + h, cbad + h,
           D, c < C);
}

// sums[to] += x, sums[from] -= x (no old cluster when !has_from) for one row;
// the `gs` lanes of a group (rank `u`) take 4-value slices.
template <typename T, int D>
__device__ __forceinline__ void move_row(const T* __restrict__ x, float* __restrict__ sums,
                                         int32_t* __restrict__ cnt, int64_t hc_to,
                                         int64_t hc_from, bool has_from, int u, int gs) {
  for (int k = u * 4; k < D; k += 4 * gs) {
    const float4 v = make_float4(Elem<T>::load(x, k), Elem<T>::load(x, k + 1),
                                 Elem<T>::load(x, k + 2), Elem<T>::load(x, k + 3));
    atomicAdd(reinterpret_cast<float4*>(sums + hc_to * D + k), v);
    if (has_from)
      atomicAdd(reinterpret_cast<float4*>(sums + hc_from * D + k),
                make_float4(-v.x, -v.y, -v.z, -v.w));
  }
  if (u == 0) {
    atomicAdd(cnt + hc_to, 1);
    if (has_from) atomicAdd(cnt + hc_from, -1);
  }
}

// four consecutive bf16 values of a row (k a multiple of 4) as one 8-byte load
__device__ __forceinline__ float4 load4(const uint16_t* x, int k) {
  const uint2 w = *reinterpret_cast<const uint2*>(x + k);
  return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u),
                     __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u));
}

// fp64 squared distance in the oracle's order: sum_k (x_k - c_k)^2, k = 0..D-1,
// one rounding per operation (no contraction)
template <typename T, int D>
__device__ __forceinline__ double dist64(const T* __restrict__ x, const float* __restrict__ c) {
  double dist = 0.0;
  for (int k = 0; k < D; ++k) {
    const double diff = __dsub_rn((double)Elem<T>::load(x, k), (double)c[k]);
    dist = __dadd_rn(dist, __dmul_rn(diff, diff));
  }
  return dist;
}

// (best, index) across the lanes xor-reachable with offsets < `width`; ties
// go to the lower index
__device__ __forceinline__ void argmin_lanes(double& best, int& bidx, int width) {
  for (int off = width / 2; off >= 1; off >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, best, off);
    const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
    if (ob < best || (ob == best && oi < bidx)) {
      best = ob;
      bidx = oi;
    }
  }
}

// Resolves every row decided in km_tc: one warp per window of 32 rows.
template <typename T, int D>
__global__ void km_resolve(const T* __restrict__ X, const float* __restrict__ cent, int64_t N,
                           int C, int64_t rows, int32_t* __restrict__ labels, int first,
                           const uint8_t* __restrict__ kind, const int4* __restrict__ cand,
                           const int32_t* __restrict__ from, float* __restrict__ sums,
                           int32_t* __restrict__ cnt) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t nwin = (rows + 31) / 32;
  for (int64_t win = warp; win < nwin; win += nw) {
    const int64_t gl = win * 32 + lane;
    const uint8_t kd = gl < rows ? kind[gl] : kKindNone;
    // moves of certain rows: each lane reads its own row's labels, then the
    // warp moves up to four rows per round with their loads issued together
    const bool mv = (kd & 3) == kKindMove;
    int my_to = 0, my_from = -1;
    if (mv) {
      my_to = labels[gl];
      my_from = from[gl];
    }
    const int my_h = (int)(gl / N);
    unsigned m = __ballot_sync(0xffffffffu, mv);
    const bool part = lane * 4 < D;  // this lane's 4-value slice exists
    while (m) {
      int ri[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        ri[j] = m ? __ffs(m) - 1 : -1;
        if (m) m &= m - 1;
      }
      float4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (ri[j] >= 0 && part) v[j] = load4(X + (win * 32 + ri[j]) * D, lane * 4);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (ri[j] < 0) break;
        const int64_t hb = (int64_t)__shfl_sync(0xffffffffu, my_h, ri[j]) * C;
        const int to = __shfl_sync(0xffffffffu, my_to, ri[j]);
        const int old = __shfl_sync(0xffffffffu, my_from, ri[j]);
        if (part) {
          atomicAdd(reinterpret_cast<float4*>(sums + (hb + to) * D + lane * 4), v[j]);
          if (old >= 0)
            atomicAdd(reinterpret_cast<float4*>(sums + (hb + old) * D + lane * 4),
                      make_float4(-v[j].x, -v[j].y, -v[j].z, -v[j].w));
        }
        if (lane == 0) {
          atomicAdd(cnt + hb + to, 1);
          if (old >= 0) atomicAdd(cnt + hb + old, -1);
        }
      }
    }
    // picks: eight rows at a time, lane 4r + u takes candidate u of row r
    unsigned pm = __ballot_sync(0xffffffffu, (kd & 3) == kKindPick);
    while (pm) {
      int myrow = -1;
      for (int r = 0; r < 8 && pm; ++r) {  // the r-th of the next eight rows
        const int i = __ffs(pm) - 1;
        pm &= pm - 1;
        if ((lane >> 2) == r) myrow = i;
      }
      const int r = lane >> 2, u = lane & 3;
      const bool live = myrow >= 0;
      const int64_t g = win * 32 + (live ? myrow : 0);
      const int64_t h = g / N;
      const T* x = X + g * D;
      double best = __longlong_as_double(0x7ff0000000000000ll);
      int bidx = C;
      if (live) {
        const int n = (kind[g] >> 2) & 7;
        if (u < n) {
          const int4 cc = cand[g];
          const int c = u == 0 ? cc.x : u == 1 ? cc.y : u == 2 ? cc.z : cc.w;
          best = dist64<T, D>(x, cent + (h * C + c) * (int64_t)D);
          bidx = c;
        }
      }
      argmin_lanes(best, bidx, 4);
      int old = -1;
      if (live) old = first ? -1 : labels[g];
      __syncwarp();
      if (live && u == 0) labels[g] = bidx;
      if (live && bidx != old)
        move_row<T, D>(x, sums, cnt, h * C + bidx, h * C + old, old >= 0, u, 4);
      (void)r;
    }
    // full fp64 decisions: a lane carries centroids c, c+32, c+64, c+96 (four
    // independent chains, compared in increasing index order)
    unsigned fm = __ballot_sync(0xffffffffu, (kd & 3) == kKindFull);
    while (fm) {
      const int i = __ffs(fm) - 1;
      fm &= fm - 1;
      const int64_t g = win * 32 + i;
      const int64_t h = g / N;
      const T* x = X + g * D;
      const float* ch = cent + h * (int64_t)C * D;
      double best = __longlong_as_double(0x7ff0000000000000ll);
      int bidx = 0;
      for (int c0 = lane; c0 < C; c0 += 128) {
        const int c1 = c0 + 32, c2 = c0 + 64, c3 = c0 + 96;
        const float* p0 = ch + (int64_t)c0 * D;
        const float* p1 = ch + (int64_t)(c1 < C ? c1 : c0) * D;
        const float* p2 = ch + (int64_t)(c2 < C ? c2 : c0) * D;
        const float* p3 = ch + (int64_t)(c3 < C ? c3 : c0) * D;
        double d0 = 0.0, d1 = 0.0, d2 = 0.0, d3 = 0.0;
        for (int k = 0; k < D; ++k) {
          const double xv = (double)Elem<T>::load(x, k);
          const double e0 = __dsub_rn(xv, (double)p0[k]), e1 = __dsub_rn(xv, (double)p1[k]);
          const double e2 = __dsub_rn(xv, (double)p2[k]), e3 = __dsub_rn(xv, (double)p3[k]);
          d0 = __dadd_rn(d0, __dmul_rn(e0, e0));
          d1 = __dadd_rn(d1, __dmul_rn(e1, e1));
          d2 = __dadd_rn(d2, __dmul_rn(e2, e2));
          d3 = __dadd_rn(d3, __dmul_rn(e3, e3));
        }
        if (d0 < best) { best = d0; bidx = c0; }
        if (c1 < C && d1 < best) { best = d1; bidx = c1; }
        if (c2 < C && d2 < best) { best = d2; bidx = c2; }
        if (c3 < C && d3 < best) { best = d3; bidx = c3; }
      }
      argmin_lanes(best, bidx, 32);
      const int old = first ? -1 : labels[g];
      __syncwarp();
      if (lane == 0) labels[g] = bidx;
      if (bidx != old) move_row<T, D>(x, sums, cnt, h * C + bidx, h * C + old, old >= 0, lane, 32);
    }
  }
}

// new centroids from the running sums, then the fp16 / norm copies
__global__ void km_finalize(const float* __restrict__ sums, const int32_t* __restrict__ cnt,
                            float* __restrict__ cent, int32_t* __restrict__ counts,
                            __half* __restrict__ ch, float* __restrict__ cnorm,
                            float* __restrict__ cmax, int* __restrict__ cbad, int C, int C_pad,
                            int D, int64_t rows) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp >= rows) return;  // rows = BH * C
  const int64_t h = warp / C;
  const int c = (int)(warp % C);
  const int n = cnt[warp];
  float* cr = cent + warp * D;
  if (n > 0)
    for (int k = lane; k < D; k += 32) cr[k] = sums[warp * D + k] / (float)n;
  if (lane == 0) counts[warp] = n;
  __syncwarp();
  prep_row(cr, ch + (h * C_pad + c) * D, cnorm + h * C_pad + c, cmax + h, cbad + h, D, true);
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

bool make_map_f16(CUtensorMap* map, const void* base, int64_t rows, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct TcWs {
  float* sums;
  int32_t* cnt;
  uint8_t* kind;
  int4* cand;
  int32_t* from;
  __half* xh;
  float* xnorm;
  __half* ch;
  float* cnorm;
  float* cmax;  // [BH] floats, then [BH] ints (cbad): cleared together
  int* cbad;
  float* st_run;  // row state between passes (C_pad > 512 only)
  float* st_drop;
  int4* st_cand;
  float4* st_dist;
};

int c_pad_of(int32_t c) { return (int)ceil_div(c, 16) * 16; }

TcWs carve(Carver& cv, int64_t bh, int64_t n, int32_t d, int32_t c) {
  TcWs w;
  const int cp = c_pad_of(c);
  w.sums = cv.take<float>((size_t)bh * c * d);
  w.cnt = cv.take<int32_t>((size_t)bh * c);
  w.cand = cv.take<int4>((size_t)bh * n);
  w.from = cv.take<int32_t>((size_t)bh * n);
  w.kind = cv.take<uint8_t>((size_t)bh * n);
  w.xh = cv.take<__half>((size_t)bh * n * d);
  w.xnorm = cv.take<float>((size_t)bh * n);
  w.ch = cv.take<__half>((size_t)bh * cp * d);
  w.cnorm = cv.take<float>((size_t)bh * cp);
  w.cmax = cv.take<float>((size_t)bh * 2);
  w.cbad = reinterpret_cast<int*>(w.cmax + bh);
  const bool passes = cp > kMaxCPad;
  w.st_cand = passes ? cv.take<int4>((size_t)bh * n) : nullptr;
  w.st_dist = passes ? cv.take<float4>((size_t)bh * n) : nullptr;
  w.st_run = passes ? cv.take<float>((size_t)bh * n) : nullptr;
  w.st_drop = passes ? cv.take<float>((size_t)bh * n) : nullptr;
  return w;
}

template <int D>
ear_status run_tc(const uint16_t* X, int64_t bh, int64_t n, int32_t c, int32_t iters,
                  const float* init, float* cent, int32_t* labels, int32_t* counts, void* ws,
                  cudaStream_t s) {
  using L = KLayout<D>;
  Carver cv(ws);
  TcWs w = carve(cv, bh, n, D, c);
  const int cp = c_pad_of(c);
  int* status = device_status_word();
  const int64_t rows = bh * n;
  const unsigned wgrid = (unsigned)std::min<int64_t>(ceil_div(rows, 8), 148 * 32);
  const unsigned rgrid = (unsigned)std::min<int64_t>(ceil_div(ceil_div(rows, 32), 8), 148 * 32);

  if (cent != init)
    EAR_CUDA(cudaMemcpyAsync(cent, init, sizeof(float) * bh * c * D, cudaMemcpyDeviceToDevice, s));
  EAR_CUDA(cudaMemsetAsync(w.sums, 0, sizeof(float) * bh * c * D, s));
  EAR_CUDA(cudaMemsetAsync(w.cnt, 0, sizeof(int32_t) * bh * c, s));
  km_xprep<D><<<wgrid, 256, 0, s>>>(X, w.xh, w.xnorm, rows);
  EAR_TRY(after_launch());
  EAR_CUDA(cudaMemsetAsync(w.cmax, 0, sizeof(float) * bh * 2, s));
  const int64_t prow = bh * cp;
  km_cprep<<<(unsigned)ceil_div(prow, 8), 256, 0, s>>>(cent, w.ch, w.cnorm, w.cmax, w.cbad, c, cp,
                                                        D, prow);
  EAR_TRY(after_launch());

  CUtensorMap mx, mc;
  const int c_box = std::min(cp, kColChunk);
  if (!make_map_f16(&mx, w.xh, rows, D, kTileRows) || !make_map_f16(&mc, w.ch, bh * cp, D, c_box))
    return EAR_ERR_CUDA;
  KmTcParams p;
  p.xnorm = w.xnorm;
  p.cnorm = w.cnorm;
  p.cmax = w.cmax;
  p.cbad = w.cbad;
  p.labels = labels;
  p.kind = w.kind;
  p.cand = w.cand;
  p.from = w.from;
  p.N = n;
  p.C = c;
  p.C_pad = cp;
  p.c_box = c_box;
  p.st_run = w.st_run;
  p.st_drop = w.st_drop;
  p.st_cand = w.st_cand;
  p.st_dist = w.st_dist;
  const int npass = (int)ceil_div(cp, kMaxCPad);
  const double a = 2.0 * (std::ldexp(1.0, -11) + (D + 1) * std::ldexp(1.0, -23)) *
                   (1.0 + std::ldexp(1.0, -11)) * (1.0 + std::ldexp(1.0, -20));
  p.a_coef = (float)(a * (1.0 + 1e-6));
  p.b_coef = (float)std::ldexp(1.0, -16);
  // centroid values in the fp16 subnormal range round with absolute error
  // <= 2^-25: at most sqrt(d) 2^-25 ||x|| on x.c, doubled in d~
  p.s_coef = (float)(2.0 * std::sqrt((double)D) * std::ldexp(1.0, -25) * 1.01);
  EAR_CUDA(cudaFuncSetAttribute(km_tc<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                L::kBytes));
  EAR_CUDA(cudaFuncSetAttribute(km_tc<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                L::kBytes));
  const dim3 grid((unsigned)ceil_div(ceil_div(n, kTileRows), kTilesPerCta), (unsigned)bh);
  const int64_t crow = bh * (int64_t)c;
  for (int t = 0; t < iters; ++t) {
    p.first = t == 0 ? 1 : 0;
    for (int pass = 0; pass < npass; ++pass) {  // 512 centroids per pass
      p.c0 = pass * kMaxCPad;
      p.cp_pass = std::min(kMaxCPad, cp - p.c0);
      p.carry_in = pass > 0 ? 1 : 0;
      p.carry_out = pass + 1 < npass ? 1 : 0;
      if (npass == 1 && cp <= kColChunk)  // one chunk per tile: tile-parallel epilogue
        km_tc<D, true><<<grid, kThreads, L::kBytes, s>>>(mx, mc, p, status);
      else
        km_tc<D, false><<<grid, kThreads, L::kBytes, s>>>(mx, mc, p, status);
      EAR_TRY(after_launch());
    }
    km_resolve<uint16_t, D><<<rgrid, 256, 0, s>>>(X, cent, n, c, rows, labels, p.first, w.kind,
                                                  w.cand, w.from, w.sums, w.cnt);
    EAR_TRY(after_launch());
    EAR_CUDA(cudaMemsetAsync(w.cmax, 0, sizeof(float) * bh * 2, s));
    km_finalize<<<(unsigned)ceil_div(crow, 8), 256, 0, s>>>(w.sums, w.cnt, cent, counts, w.ch,
                                                           w.cnorm, w.cmax, w.cbad, c, cp, D,
                                                           crow);
    EAR_TRY(after_launch());
  }
  return EAR_OK;
}

}  // namespace

bool kmeans_tc_supported(ear_dtype dt, int32_t d, int32_t c) {
  return dt == EAR_BF16 && (d == 64 || d == 128) && c_pad_of(c) <= kMaxCTotal;
}

size_t kmeans_tc_workspace(int64_t bh, int64_t n, int32_t d, int32_t c) {
  Carver cv(nullptr);
  carve(cv, bh, n, d, c);
  return cv.used;
}

ear_status kmeans_tc_run(const void* X, int64_t bh, int64_t n, int32_t d, int32_t c,
                         int32_t iters, const float* init, float* cent, int32_t* labels,
                         int32_t* counts, void* ws, cudaStream_t s) {
  const uint16_t* x = static_cast<const uint16_t*>(X);
  return d == 64 ? run_tc<64>(x, bh, n, c, iters, init, cent, labels, counts, ws, s)
                 : run_tc<128>(x, bh, n, c, iters, init, cent, labels, counts, ws, s);
}

}  // namespace ear
