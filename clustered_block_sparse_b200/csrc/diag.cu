// Diagnostics of the approximation (SVG-EAR §4.2 after "Error estimation":
// the bound's residual 8 δ_q^2 K_max^2 / (N_k d) grows with the clustering
// error δ_q^2 and the largest key norm; §5.3 "Effect of clustering"; §5.1:
// the average relative change of the softmax normalizer).
//   dg_cluster   per slice: δ^2 = (1/N) sum_i ||x_i - c_{l_i}||^2 and
//                K_max = max_i ||x_i||.  A warp per row (lanes over d, fp32
//                within the row), fp64 sums across rows (atomics into the
//                caller's output, zeroed first); the maximum of non-negative
//                doubles by an integer atomicMax on their bits.
//   dg_norm      per slice: mean over queries of |e^{lse_s - lse_d} - 1|
//                (a query with equal lse, both -inf included, counts 0).
#include <algorithm>

#include "ear_internal.cuh"

namespace ear {
namespace {

template <typename T, int D>
__global__ void __launch_bounds__(256)
dg_cluster(const T* __restrict__ X, const int32_t* __restrict__ labels,
           const float* __restrict__ cent, int64_t N, int C, int chunks,
           double* __restrict__ sum_out, unsigned long long* __restrict__ max_out, int* status) {
  constexpr int kPer = D / 32;
  const int chunk = blockIdx.x;
  const int64_t h = blockIdx.y;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t r0 = N * chunk / chunks, r1 = N * (chunk + 1) / chunks;
  double acc = 0.0;
  float mx = 0.f;
  for (int64_t i = r0 + w; i < r1; i += 8) {
    int c = labels[h * N + i];
    if (c < 0 || c >= C) {
      if (lane == 0) latch(status, EAR_ERR_DEVICE);
      continue;
    }
    const T* x = X + (h * N + i) * D + lane * kPer;
    const float* cc = cent + (h * C + c) * (int64_t)D + lane * kPer;
    float dist = 0.f, nrm = 0.f;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const float xv = Elem<T>::load(x, k);
      const float df = xv - cc[k];
      dist = fmaf(df, df, dist);
      nrm = fmaf(xv, xv, nrm);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      dist += __shfl_xor_sync(0xffffffffu, dist, o);
      nrm += __shfl_xor_sync(0xffffffffu, nrm, o);
    }
    acc += (double)dist;
    mx = fmaxf(mx, sqrtf(nrm));
  }
  if (lane == 0) {
    atomicAdd(sum_out + h, acc);
    atomicMax(max_out + h, (unsigned long long)__double_as_longlong((double)mx));
  }
}

__global__ void dg_finish(double* __restrict__ sum_out, int64_t N, int64_t bh) {
  const int64_t h = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (h < bh) sum_out[h] /= (double)N;
}

__global__ void __launch_bounds__(256)
dg_norm(const float* __restrict__ a, const float* __restrict__ b, int64_t N,
        double* __restrict__ out) {
  const int64_t h = blockIdx.x;
  __shared__ double red[8];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < N; i += 256) {
    const double x = (double)a[h * N + i], y = (double)b[h * N + i];
    if (x == y) continue;  // also both -inf (no term on either side): no change
    acc += fabs(expm1(x - y));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < 8; ++i) t += red[i];
    out[h] = t / (double)N;
  }
}

template <typename T, int D>
ear_status cluster_t(const void* X, const int32_t* labels, const float* cent, int64_t bh,
                     int64_t n, int32_t c, double* mean_sq, double* max_norm, cudaStream_t s) {
  EAR_CUDA(cudaMemsetAsync(mean_sq, 0, sizeof(double) * bh, s));
  EAR_CUDA(cudaMemsetAsync(max_norm, 0, sizeof(double) * bh, s));
  const int chunks = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(4 * 148, bh), n / 256));
  dg_cluster<T, D><<<dim3((unsigned)chunks, (unsigned)bh), 256, 0, s>>>(
      static_cast<const T*>(X), labels, cent, n, c, chunks, mean_sq,
      reinterpret_cast<unsigned long long*>(max_norm), device_status_word());
  EAR_TRY(after_launch());
  dg_finish<<<(unsigned)ceil_div(bh, 128), 128, 0, s>>>(mean_sq, n, bh);
  return after_launch();
}

}  // namespace

ear_status cluster_stats_run(const void* X, ear_dtype dt, const int32_t* labels,
                             const float* cent, int64_t bh, int64_t n, int32_t d, int32_t c,
                             double* mean_sq, double* max_norm, cudaStream_t s) {
  if (dt == EAR_F32)
    return d == 64 ? cluster_t<float, 64>(X, labels, cent, bh, n, c, mean_sq, max_norm, s)
                   : cluster_t<float, 128>(X, labels, cent, bh, n, c, mean_sq, max_norm, s);
  return d == 64 ? cluster_t<uint16_t, 64>(X, labels, cent, bh, n, c, mean_sq, max_norm, s)
                 : cluster_t<uint16_t, 128>(X, labels, cent, bh, n, c, mean_sq, max_norm, s);
}

ear_status normalizer_change_run(const float* lse_sparse, const float* lse_dense, int64_t bh,
                                 int64_t n, double* out, cudaStream_t s) {
  dg_norm<<<(unsigned)bh, 256, 0, s>>>(lse_sparse, lse_dense, n, out);
  return after_launch();
}

}  // namespace ear
