// Cluster-contiguous permutation (SVG-EAR §3.1: tokens of a cluster are laid
// out contiguously so the attention map splits into cluster x cluster blocks).
//
// A stable counting sort per slice, in 1024-token tiles:
//  * pm_tile_hist: per (slice, tile, cluster) member counts (cluster fastest,
//                  so the scan below reads them coalesced).
//  * pm_scan:      one block per slice turns them into the first output
//                  position of every (cluster, tile) and writes offsets.
//  * pm_scatter:   each tile walks its 32 warps in order; a warp groups equal
//                  labels with __match_any_sync, so a token's position is the
//                  (cluster, tile) cursor plus the number of earlier tokens of
//                  its cluster - the order within a cluster is token order.
//  * pm_gather:    X_perm[r] = X[perm[r]], 16-byte vector copies; a warp
//                  moves several rows at once (lanes split per row) with four
//                  row groups in flight per thread.
//  * pm_gather_mean: when the per-cluster means are asked for (v̄, §4.3): one
//                  block per cluster gathers the cluster's rows into place and
//                  sums them in a fixed order (per thread over its rows, then
//                  across the block's row groups), X read once.
#include "ear_internal.cuh"

namespace ear {
namespace {

constexpr int kTile = 1024;

__global__ void __launch_bounds__(kTile)
pm_tile_hist(const int32_t* __restrict__ labels, int64_t N, int C, int ntiles,
             int32_t* __restrict__ hist, int* status) {
  const int64_t h = blockIdx.y;
  const int64_t i = (int64_t)blockIdx.x * kTile + threadIdx.x;
  if (i >= N) return;
  int c = labels[h * N + i];
  if (c < 0 || c >= C) {
    latch(status, EAR_ERR_DEVICE);
    return;
  }
  atomicAdd(hist + ((h * ntiles + blockIdx.x) * C + c), 1);
}

__global__ void __launch_bounds__(1024)
pm_scan(int32_t* __restrict__ hist, int32_t* __restrict__ totals, int C, int ntiles,
        int32_t* __restrict__ offsets) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  const int64_t h = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  int32_t* hh = hist + h * (int64_t)C * ntiles;  // [tile][cluster]
  int32_t* th = totals + h * (int64_t)C;
  // per cluster: exclusive prefix over tiles, total in `totals` (consecutive
  // threads read consecutive clusters of one tile; 16 tiles' counts are
  // loaded before they are summed)
  for (int c = tid; c < C; c += 1024) {
    int32_t run = 0;
    for (int t0 = 0; t0 < ntiles; t0 += 16) {
      int32_t v[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = t0 + k < ntiles ? hh[(int64_t)(t0 + k) * C + c] : 0;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if (t0 + k < ntiles) hh[(int64_t)(t0 + k) * C + c] = run;
        run += v[k];
      }
    }
    th[c] = run;
  }
  if (tid == 0) carry = 0;
  __syncthreads();
  // exclusive scan of totals over clusters -> offsets
  int32_t* oh = offsets + h * (int64_t)(C + 1);
  for (int base = 0; base < C; base += 1024) {
    int c = base + tid;
    int32_t v = c < C ? th[c] : 0;
    int32_t x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int32_t w = warp_sums[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        int32_t y = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += y;
      }
      warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    int32_t incl = x + (wid > 0 ? warp_sums[wid - 1] : 0) + carry;
    if (c < C) oh[c] = incl - v;
    __syncthreads();
    if (tid == 1023) carry = incl;
    __syncthreads();
  }
  if (tid == 0) oh[C] = carry;
  // the cursor of (cluster, tile) is offsets[cluster] + hist[tile][cluster]:
  // pm_scatter adds the offset
}

// Stable scatter of one tile: the tile's 32 warps take turns; a warp's rows
// of one cluster go to consecutive places after those of earlier warps and
// tiles.  SHARED: the tile's cursors (offset + earlier tiles' members) live in
// shared memory, else in the global cursor table.
template <bool SHARED>
__global__ void __launch_bounds__(kTile)
pm_scatter(const int32_t* __restrict__ labels, int64_t N, int C, int ntiles,
           int32_t* __restrict__ cursor, const int32_t* __restrict__ offsets,
           int32_t* __restrict__ perm) {
  extern __shared__ int32_t scur[];
  const int64_t h = blockIdx.y;
  const int tile = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (SHARED) {
    for (int k = tid; k < C; k += kTile)
      scur[k] = offsets[h * (int64_t)(C + 1) + k] + cursor[(h * ntiles + tile) * (int64_t)C + k];
    __syncthreads();
  }
  const int64_t i = (int64_t)tile * kTile + tid;
  int c = -1;
  if (i < N) {
    c = labels[h * N + i];
    if (c < 0 || c >= C) c = -1;
  }
  const unsigned group = __match_any_sync(0xffffffffu, c);
  const int leader = __ffs(group) - 1;
  const int before = __popc(group & ((1u << lane) - 1u));
  int32_t* cur = SHARED ? scur + (c < 0 ? 0 : c)
                        : cursor + (h * ntiles + tile) * (int64_t)C + (c < 0 ? 0 : c);
  const int32_t off = (!SHARED && c >= 0) ? offsets[h * (int64_t)(C + 1) + c] : 0;
  for (int w = 0; w < 32; ++w) {
    if (wid == w) {
      int32_t base = 0;
      if (lane == leader && c >= 0) base = *cur;
      base = __shfl_sync(0xffffffffu, base, leader);
      if (c >= 0) {
        perm[h * N + off + base + before] = (int32_t)i;
        if (lane == leader) *cur = base + __popc(group);
      }
    }
    __syncthreads();
  }
}

// row_vecs (16-byte vectors per row) divides 32: 8, 16 or 32
__global__ void pm_gather(const uint4* __restrict__ X, uint4* __restrict__ Xp,
                          const int32_t* __restrict__ perm, int64_t N, int row_vecs,
                          int64_t rows_total, int* status) {
  constexpr int kDepth = 4;  // row groups in flight per thread
  const int lane = threadIdx.x & 31;
  const int groups = 32 / row_vecs;  // rows a warp moves per group
  const int gi = lane / row_vecs, u = lane % row_vecs;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t step = (int64_t)groups * kDepth;
  for (int64_t base = warp * step; base < rows_total; base += nwarps * step) {
    uint4 v[kDepth];
    int64_t dst[kDepth];
#pragma unroll
    for (int k = 0; k < kDepth; ++k) {
      const int64_t g = base + (int64_t)k * groups + gi;
      dst[k] = -1;
      if (g < rows_total) {
        const int32_t src = perm[g];
        if (src >= 0 && src < N) {
          v[k] = X[((g / N) * N + src) * row_vecs + u];
          dst[k] = g * row_vecs + u;
        } else if (u == 0) {
          latch(status, EAR_ERR_DEVICE);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kDepth; ++k)
      if (dst[k] >= 0) Xp[dst[k]] = v[k];
  }
}

// one 16-byte piece of a row: its values as floats
__device__ __forceinline__ void unpack16(const uint4 w, float (&f)[8], const uint16_t*) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(u[k] << 16);
    f[2 * k + 1] = __uint_as_float(u[k] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void unpack16(const uint4 w, float (&f)[8], const float*) {
  f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
  f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
#pragma unroll
  for (int k = 4; k < 8; ++k) f[k] = 0.f;
}

// X_perm rows of cluster c = X[perm[r]] for r in [offsets[c], offsets[c+1])
// (skipped when Xp is null: the means alone), and their fp32 mean in a fixed
// order.  The offsets must partition [0, N)
// (offsets[0] = 0, offsets[C] = N, non-decreasing), as ear_permute writes
// them; a table that does not is latched as an error.  A thread moves one
// 16-byte piece of a row (kPer values) for every kGroups-th row of the
// cluster, two rows in flight.
template <typename T, int D>
__global__ void __launch_bounds__(256)
pm_gather_mean(const T* __restrict__ X, T* __restrict__ Xp, const int32_t* __restrict__ perm,
               const int32_t* __restrict__ offsets, int64_t N, int C, float* __restrict__ mean,
               int* status) {
  constexpr int kPer = 16 / (int)sizeof(T);  // values per 16-byte piece
  constexpr int kPieces = D / kPer;          // pieces per row
  constexpr int kGroups = 256 / kPieces;     // rows in flight per block step
  __shared__ float part[kGroups][D];
  const int64_t h = blockIdx.y;
  const int c = blockIdx.x;
  const int q = threadIdx.x % kPieces, g = threadIdx.x / kPieces;
  const int32_t* oh = offsets + h * (int64_t)(C + 1);
  int32_t r0 = oh[c], r1 = oh[c + 1];
  const bool ends_ok = (c > 0 || r0 == 0) && (c < C - 1 || r1 == N);
  if (r0 < 0 || r1 < r0 || r1 > N || !ends_ok) {
    if (threadIdx.x == 0) latch(status, EAR_ERR_DEVICE);
    if (r0 < 0 || r1 < r0 || r1 > N) r0 = r1 = 0;
  }
  float acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
  const uint4* xh = reinterpret_cast<const uint4*>(X + h * N * D);
  uint4* ph = Xp != nullptr ? reinterpret_cast<uint4*>(Xp + h * N * D) : nullptr;
  const int32_t* pp = perm + h * N;
  for (int64_t r = r0 + g; r < r1; r += 2 * kGroups) {
    const int64_t ra = r, rb = r + kGroups;
    const int32_t sa = pp[ra];
    const int32_t sb = rb < r1 ? pp[rb] : 0;
    const bool oka = sa >= 0 && sa < N, okb = rb < r1 && sb >= 0 && sb < N;
    if ((!oka || (rb < r1 && !okb)) && q == 0) latch(status, EAR_ERR_DEVICE);
    uint4 wa = make_uint4(0u, 0u, 0u, 0u), wb = wa;
    if (oka) wa = xh[(int64_t)sa * kPieces + q];
    if (okb) wb = xh[(int64_t)sb * kPieces + q];
    float f[8];
    if (oka) {
      if (ph != nullptr) ph[ra * kPieces + q] = wa;
      unpack16(wa, f, X);
#pragma unroll
      for (int k = 0; k < kPer; ++k) acc[k] += f[k];
    }
    if (okb) {
      if (ph != nullptr) ph[rb * kPieces + q] = wb;
      unpack16(wb, f, X);
#pragma unroll
      for (int k = 0; k < kPer; ++k) acc[k] += f[k];
    }
  }
#pragma unroll
  for (int k = 0; k < kPer; ++k) part[g][q * kPer + k] = acc[k];
  __syncthreads();
  for (int e = threadIdx.x; e < D; e += 256) {
    float s = part[0][e];
    for (int k = 1; k < kGroups; ++k) s += part[k][e];
    const int32_t n = r1 - r0;
    mean[(h * C + c) * (int64_t)D + e] = n > 0 ? s / (float)n : 0.f;
  }
}

template <typename T, int D>
ear_status gather_mean_t(const void* X, void* Xp, const int32_t* perm, const int32_t* offsets,
                         int64_t bh, int64_t n, int32_t c, float* mean, cudaStream_t s) {
  pm_gather_mean<T, D><<<dim3((unsigned)c, (unsigned)bh), 256, 0, s>>>(
      (const T*)X, (T*)Xp, perm, offsets, n, c, mean, device_status_word());
  return after_launch();
}

struct PmWs {
  int32_t* hist;
  int32_t* totals;
};

PmWs carve(Carver& cv, int64_t bh, int64_t n, int32_t c) {
  PmWs w;
  const int64_t ntiles = ceil_div(n, kTile);
  w.hist = cv.take<int32_t>((size_t)bh * c * ntiles);
  w.totals = cv.take<int32_t>((size_t)bh * c);
  return w;
}

}  // namespace

size_t permute_workspace(int64_t bh, int64_t n, int32_t c) {
  Carver cv(nullptr);
  carve(cv, bh, n, c);
  return cv.used;
}

ear_status permute_run(const int32_t* labels, int64_t bh, int64_t n, int32_t c, int32_t* perm,
                       int32_t* offsets, const void* X, void* X_perm, ear_dtype dt, int32_t d,
                       float* seg_mean, void* ws, cudaStream_t s) {
  Carver cv(ws);
  PmWs w = carve(cv, bh, n, c);
  int* status = device_status_word();
  const int ntiles = (int)ceil_div(n, kTile);
  const dim3 tgrid((unsigned)ntiles, (unsigned)bh);
  EAR_CUDA(cudaMemsetAsync(w.hist, 0, sizeof(int32_t) * bh * c * ntiles, s));
  EAR_CUDA(cudaMemsetAsync(perm, 0xff, sizeof(int32_t) * bh * n, s));
  pm_tile_hist<<<tgrid, kTile, 0, s>>>(labels, n, c, ntiles, w.hist, status);
  EAR_TRY(after_launch());
  pm_scan<<<(unsigned)bh, 1024, 0, s>>>(w.hist, w.totals, c, ntiles, offsets);
  EAR_TRY(after_launch());
  const size_t scur_bytes = sizeof(int32_t) * (size_t)c;
  if (scur_bytes <= 48 * 1024)
    pm_scatter<true><<<tgrid, kTile, scur_bytes, s>>>(labels, n, c, ntiles, w.hist, offsets, perm);
  else
    pm_scatter<false><<<tgrid, kTile, 0, s>>>(labels, n, c, ntiles, w.hist, offsets, perm);
  EAR_TRY(after_launch());
  if (X == nullptr) return EAR_OK;
  return permute_apply_run(perm, offsets, bh, n, c, X, X_perm, dt, d, seg_mean, s);
}

ear_status permute_apply_run(const int32_t* perm, const int32_t* offsets, int64_t bh, int64_t n,
                             int32_t c, const void* X, void* X_perm, ear_dtype dt, int32_t d,
                             float* seg_mean, cudaStream_t s) {
  int* status = device_status_word();
  if (seg_mean != nullptr) {  // gather and means in one pass over X
    if (dt == EAR_F32)
      return d == 64 ? gather_mean_t<float, 64>(X, X_perm, perm, offsets, bh, n, c, seg_mean, s)
                     : gather_mean_t<float, 128>(X, X_perm, perm, offsets, bh, n, c, seg_mean, s);
    return d == 64 ? gather_mean_t<uint16_t, 64>(X, X_perm, perm, offsets, bh, n, c, seg_mean, s)
                   : gather_mean_t<uint16_t, 128>(X, X_perm, perm, offsets, bh, n, c, seg_mean, s);
  }
  const int elem = dt == EAR_F32 ? 4 : 2;
  const int row_vecs = d * elem / 16;
  const int64_t rows_total = bh * n;
  const unsigned ggrid = (unsigned)std::min<int64_t>(ceil_div(rows_total, 8), 148 * 64);
  pm_gather<<<ggrid, 256, 0, s>>>((const uint4*)X, (uint4*)X_perm, perm, n, row_vecs, rows_total,
                                  status);
  return after_launch();
}

}  // namespace ear
