// Compensation-error probe (SVG-EAR §4.2 "Error estimation"; §1: query
// centroids stand in for the queries of their cluster).
//
//   E[a][b] = sum_{j in b} (s q̄_a·k_j - s q̄_a·k̄_b)^2 = sum_{j in b} (s q̄_a·(k_j - k̄_b))^2
//
// The second form is the one evaluated: each key is centred on its cluster
// centroid once (one fp32 rounding per element) before the dot product, so
// the small logit gaps are not the difference of two large fp32 logits.
// Grid = (key cluster b, slice); a block walks its cluster's contiguous rows
// in 64-row chunks against 64-centroid chunks of q̄ (4x4 register tiles).
#include "ear_internal.cuh"

namespace ear {
namespace {

constexpr int kA = 64;     // query centroids per chunk
constexpr int kJ = 64;     // keys per chunk
constexpr int kThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
pr_probe(const float* __restrict__ qc, const int32_t* __restrict__ qn,
         const float* __restrict__ kc, const T* __restrict__ K,
         const int32_t* __restrict__ koff, int64_t Nk, int Cq, int Ck, float scale,
         float* __restrict__ E, int* status) {
  extern __shared__ float smem[];
  float* qs = smem;                  // [kA][D + 1]
  float* ks = smem + kA * (D + 1);   // [kJ][D + 1]
  float* kbar = ks + kJ * (D + 1);   // [D]
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t h = blockIdx.y;
  const int b = blockIdx.x;
  const int32_t* oh = koff + h * (int64_t)(Ck + 1);
  int32_t r0 = oh[b], r1 = oh[b + 1];
  if (r0 < 0 || r1 < r0 || r1 > Nk) {
    if (tid == 0) latch(status, EAR_ERR_DEVICE);
    r1 = r0 = 0;
  }
  const T* kh = K + h * Nk * D;
  for (int k = tid; k < D; k += kThreads) kbar[k] = kc[(h * Ck + b) * (int64_t)D + k];

  for (int a0 = 0; a0 < Cq; a0 += kA) {
    __syncthreads();
    for (int e = tid; e < kA * D; e += kThreads) {
      int r = e / D, k = e % D;
      qs[r * (D + 1) + k] = (a0 + r) < Cq ? qc[(h * Cq + a0 + r) * (int64_t)D + k] : 0.f;
    }
    float part[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j0 = r0; j0 < r1; j0 += kJ) {
      const int nj = min(kJ, r1 - j0);
      __syncthreads();
      for (int e = tid; e < kJ * D; e += kThreads) {
        int r = e / D, k = e % D;
        ks[r * (D + 1) + k] = r < nj ? Elem<T>::load(kh, (int64_t)(j0 + r) * D + k) - kbar[k] : 0.f;
      }
      __syncthreads();
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
      for (int k = 0; k < D; ++k) {
        float qv[4], kv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) qv[i] = qs[(ty + 16 * i) * (D + 1) + k];
#pragma unroll
        for (int j = 0; j < 4; ++j) kv[j] = ks[(tx + 16 * j) * (D + 1) + k];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qv[i], kv[j], acc[i][j]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float g = scale * acc[i][j];  // zero for padded rows (centred value 0)
          part[i] = fmaf(g, g, part[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v = part[i];
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      const int a = a0 + ty + 16 * i;
      if (tx == 0 && a < Cq) {
        const bool live = qn[h * Cq + a] > 0 && r1 > r0;
        E[(h * Cq + a) * (int64_t)Ck + b] = live ? v : 0.f;
      }
    }
  }
}

template <typename T, int D>
ear_status run_t(const float* qc, const int32_t* qn, const float* kc, const void* K,
                 const int32_t* koff, int64_t bh, int64_t n_k, int32_t c_q, int32_t c_k,
                 float scale, float* E, cudaStream_t s) {
  const size_t smem = ((size_t)(kA + kJ) * (D + 1) + D) * sizeof(float);
  EAR_CUDA(cudaFuncSetAttribute(pr_probe<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem));
  pr_probe<T, D><<<dim3((unsigned)c_k, (unsigned)bh), kThreads, smem, s>>>(
      qc, qn, kc, (const T*)K, koff, n_k, c_q, c_k, scale, E, device_status_word());
  return after_launch();
}

}  // namespace

size_t probe_workspace(int64_t, int64_t, int32_t, int32_t, int32_t) { return 0; }

ear_status probe_run(const float* qc, const int32_t* qn, const float* kc, const void* K,
                     ear_dtype dt, const int32_t* koff, int64_t bh, int64_t n_k, int32_t d,
                     int32_t c_q, int32_t c_k, float scale, float* E, void*, cudaStream_t s) {
  if (dt == EAR_F32)
    return d == 64 ? run_t<float, 64>(qc, qn, kc, K, koff, bh, n_k, c_q, c_k, scale, E, s)
                   : run_t<float, 128>(qc, qn, kc, K, koff, bh, n_k, c_q, c_k, scale, E, s);
  return d == 64 ? run_t<uint16_t, 64>(qc, qn, kc, K, koff, bh, n_k, c_q, c_k, scale, E, s)
                 : run_t<uint16_t, 128>(qc, qn, kc, K, koff, bh, n_k, c_q, c_k, scale, E, s);
}

}  // namespace ear
