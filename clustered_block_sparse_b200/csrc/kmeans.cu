// Lloyd k-means (SVG-EAR §4.1: Q and K are clustered into C_q / C_k clusters
// and every token is represented by the mean token of its cluster).
//
// One iteration = assign, re-decide, update, finalize:
//  * km_assign: a 64-row x 64-centroid register-tiled SIMT kernel computes
//    sum_k (x_k - c_k)^2 in fp32 and keeps, per row, the best and second-best
//    distance.  With e = (d + 8) * 2^-24 bounding the relative rounding error
//    of that sum, the label is certain when second * (1 - e) > best * (1 + e).
//    Otherwise the row goes to a refine list.
//  * km_refine: one warp per listed row recomputes all C distances in fp64,
//    each step rounded separately (no fused multiply-add) so the decision is
//    the exact fp64 argmin, ties to the lowest index.
//  * km_update: member sums with vector fp32 atomics, counts with int atomics.
//  * km_finalize: centroid = sum / count; an empty cluster keeps its centroid.
#include <algorithm>

#include "ear_internal.cuh"

namespace ear {
namespace {

constexpr int kRows = 64;
constexpr int kCents = 64;
constexpr int kThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
km_assign(const T* __restrict__ X, const float* __restrict__ cent, int64_t N, int C,
          int32_t* __restrict__ labels, int64_t* __restrict__ refine_rows,
          unsigned long long* __restrict__ refine_count) {
  extern __shared__ float smem[];
  float* xs = smem;                    // [kRows][D + 1]
  float* cs = smem + kRows * (D + 1);  // [kCents][D + 1]
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t h = blockIdx.y;
  const int64_t row0 = (int64_t)blockIdx.x * kRows;
  const T* xh = X + h * N * D;
  const float* ch = cent + h * (int64_t)C * D;

  for (int e = tid; e < kRows * D; e += kThreads) {
    int r = e / D, k = e % D;
    int64_t row = row0 + r;
    xs[r * (D + 1) + k] = row < N ? Elem<T>::load(xh, row * D + k) : 0.f;
  }

  float best[4], second[4];
  int bidx[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    best[i] = __int_as_float(0x7f800000);
    second[i] = __int_as_float(0x7f800000);
    bidx[i] = 0;
  }

  for (int c0 = 0; c0 < C; c0 += kCents) {
    __syncthreads();
    for (int e = tid; e < kCents * D; e += kThreads) {
      int r = e / D, k = e % D;
      cs[r * (D + 1) + k] = (c0 + r) < C ? ch[(int64_t)(c0 + r) * D + k] : 0.f;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      float xv[4], cv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) xv[i] = xs[(ty + 16 * i) * (D + 1) + k];
#pragma unroll
      for (int j = 0; j < 4; ++j) cv[j] = cs[(tx + 16 * j) * (D + 1) + k];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float diff = xv[i] - cv[j];
          acc[i][j] = fmaf(diff, diff, acc[i][j]);
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int c = c0 + tx + 16 * j;  // increasing per thread, so ties keep the lower index
      if (c >= C) continue;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float dv = acc[i][j];
        if (dv < best[i]) {
          second[i] = best[i];
          best[i] = dv;
          bidx[i] = c;
        } else if (dv < second[i]) {
          second[i] = dv;
        }
      }
    }
  }

  // merge the 16 column threads of each row (lanes differing in bits 0..3)
  const float e_rel = (float)(D + 8) * 5.9604645e-8f;  // (d + 8) * 2^-24
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float b = best[i], s = second[i];
    int bi = bidx[i];
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) {
      float ob = __shfl_xor_sync(0xffffffffu, b, off);
      float os = __shfl_xor_sync(0xffffffffu, s, off);
      int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (ob < b || (ob == b && oi < bi)) {
        s = fminf(os, b);
        b = ob;
        bi = oi;
      } else {
        s = fminf(s, ob);
      }
    }
    int64_t row = row0 + ty + 16 * i;
    if (tx == 0 && row < N) {
      labels[h * N + row] = bi;
      bool certain = s * (1.f - e_rel) > b * (1.f + e_rel);
      if (!certain) {
        unsigned long long pos = atomicAdd(refine_count, 1ull);
        refine_rows[pos] = h * N + row;  // capacity is BH * N: every row fits
      }
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
km_refine(const T* __restrict__ X, const float* __restrict__ cent, int64_t N, int C,
          int32_t* __restrict__ labels, const int64_t* __restrict__ refine_rows,
          const unsigned long long* __restrict__ refine_count) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
  const int64_t total = (int64_t)*refine_count;
  for (int64_t e = warp; e < total; e += nwarps) {
    const int64_t g = refine_rows[e];
    const int64_t h = g / N;
    const T* x = X + g * D;
    const float* ch = cent + h * (int64_t)C * D;
    double best = __longlong_as_double(0x7ff0000000000000ll);
    int bidx = 0;
    for (int c = lane; c < C; c += 32) {
      const float* cc = ch + (int64_t)c * D;
      double dist = 0.0;
      for (int k = 0; k < D; ++k) {
        double diff = __dsub_rn((double)Elem<T>::load(x, k), (double)cc[k]);
        dist = __dadd_rn(dist, __dmul_rn(diff, diff));
      }
      if (dist < best) {
        best = dist;
        bidx = c;
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      double ob = __shfl_xor_sync(0xffffffffu, best, off);
      int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
      if (ob < best || (ob == best && oi < bidx)) {
        best = ob;
        bidx = oi;
      }
    }
    if (lane == 0) labels[g] = bidx;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
km_update(const T* __restrict__ X, int64_t N, int C, const int32_t* __restrict__ labels,
          float* __restrict__ sums, int32_t* __restrict__ cnt, int64_t rows_total) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
  for (int64_t g = warp; g < rows_total; g += nwarps) {
    const int64_t h = g / N;
    const int c = labels[g];
    float* dst = sums + (h * C + c) * D;
    const T* x = X + g * D;
    if (lane * 4 < D) {
      float4 v;
      v.x = Elem<T>::load(x, lane * 4 + 0);
      v.y = Elem<T>::load(x, lane * 4 + 1);
      v.z = Elem<T>::load(x, lane * 4 + 2);
      v.w = Elem<T>::load(x, lane * 4 + 3);
      atomicAdd(reinterpret_cast<float4*>(dst + lane * 4), v);
    }
    if (lane == 0) atomicAdd(cnt + h * C + c, 1);
  }
}

template <int D>
__global__ void km_finalize(const float* __restrict__ sums, const int32_t* __restrict__ cnt,
                            float* __restrict__ cent, int32_t* __restrict__ counts,
                            int64_t total) {
  int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= total) return;
  int64_t hc = e / D;
  int n = cnt[hc];
  if (n > 0) cent[e] = sums[e] / (float)n;
  if (e % D == 0) counts[hc] = n;
}

struct KmWs {
  float* sums;
  int32_t* cnt;
  int64_t* refine_rows;
  unsigned long long* refine_count;
};

KmWs carve(Carver& cv, int64_t bh, int64_t n, int32_t d, int32_t c) {
  KmWs w;
  w.sums = cv.take<float>((size_t)bh * c * d);
  w.cnt = cv.take<int32_t>((size_t)bh * c);
  w.refine_rows = cv.take<int64_t>((size_t)bh * n);
  w.refine_count = cv.take<unsigned long long>(1);
  return w;
}

template <typename T, int D>
ear_status run_t(const T* X, int64_t bh, int64_t n, int32_t c, int32_t iters, const float* init,
                 float* cent, int32_t* labels, int32_t* counts, void* ws, cudaStream_t s) {
  Carver cv(ws);
  KmWs w = carve(cv, bh, n, D, c);
  const size_t smem = (size_t)(kRows + kCents) * (D + 1) * sizeof(float);
  EAR_CUDA(cudaFuncSetAttribute(km_assign<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem));
  if (cent != init)
    EAR_CUDA(cudaMemcpyAsync(cent, init, sizeof(float) * bh * c * D, cudaMemcpyDeviceToDevice, s));
  const int64_t rows_total = bh * n;
  const dim3 agrid((unsigned)ceil_div(n, kRows), (unsigned)bh);
  const unsigned wgrid = (unsigned)std::min<int64_t>(ceil_div(rows_total, kThreads / 32), 148 * 16);
  const int64_t cent_total = bh * (int64_t)c * D;
  for (int t = 0; t < iters; ++t) {
    EAR_CUDA(cudaMemsetAsync(w.refine_count, 0, sizeof(unsigned long long), s));
    km_assign<T, D><<<agrid, kThreads, smem, s>>>(X, cent, n, c, labels, w.refine_rows,
                                                  w.refine_count);
    EAR_TRY(after_launch());
    km_refine<T, D><<<wgrid, kThreads, 0, s>>>(X, cent, n, c, labels, w.refine_rows,
                                               w.refine_count);
    EAR_TRY(after_launch());
    EAR_CUDA(cudaMemsetAsync(w.sums, 0, sizeof(float) * cent_total, s));
    EAR_CUDA(cudaMemsetAsync(w.cnt, 0, sizeof(int32_t) * bh * c, s));
    km_update<T, D><<<wgrid, kThreads, 0, s>>>(X, n, c, labels, w.sums, w.cnt, rows_total);
    EAR_TRY(after_launch());
    km_finalize<D><<<(unsigned)ceil_div(cent_total, 256), 256, 0, s>>>(w.sums, w.cnt, cent,
                                                                     counts, cent_total);
    EAR_TRY(after_launch());
  }
  return EAR_OK;
}

}  // namespace

// The tensor-core path serves bf16 inputs with at most 512 centroids; the
// workspace covers whichever path the dtype selects.
size_t kmeans_workspace(int64_t bh, int64_t n, int32_t d, int32_t c) {
  Carver cv(nullptr);
  carve(cv, bh, n, d, c);
  size_t bytes = cv.used;
  if (kmeans_tc_supported(EAR_BF16, d, c)) bytes = std::max(bytes, kmeans_tc_workspace(bh, n, d, c));
  return bytes;
}

ear_status kmeans_run(const void* X, ear_dtype dt, int64_t bh, int64_t n, int32_t d, int32_t c,
                      int32_t iters, const float* init, float* cent, int32_t* labels,
                      int32_t* counts, void* ws, cudaStream_t s) {
  if (kmeans_tc_supported(dt, d, c))
    return kmeans_tc_run(X, bh, n, d, c, iters, init, cent, labels, counts, ws, s);
  if (dt == EAR_F32) {
    if (d == 64)
      return run_t<float, 64>((const float*)X, bh, n, c, iters, init, cent, labels, counts, ws, s);
    return run_t<float, 128>((const float*)X, bh, n, c, iters, init, cent, labels, counts, ws, s);
  }
  if (d == 64)
    return run_t<uint16_t, 64>((const uint16_t*)X, bh, n, c, iters, init, cent, labels, counts,
                               ws, s);
  return run_t<uint16_t, 128>((const uint16_t*)X, bh, n, c, iters, init, cent, labels, counts,
                              ws, s);
}

}  // namespace ear
