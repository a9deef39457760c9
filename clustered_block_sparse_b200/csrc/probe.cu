// Compensation-error probe for fp32 keys (SVG-EAR §4.2 "Error estimation";
// §1: query centroids stand in for the queries of their cluster).  bf16 keys
// take the tensor-core kernel in probe_tc.cu.
//
//   E[a][b] = sum_{j in b} (s q̄_a·k_j - s q̄_a·k̄_b)^2 = sum_{j in b} (s q̄_a·(k_j - k̄_b))^2
//
// The second form is the one evaluated: each key is centred on its cluster
// centroid once (one fp32 rounding per element) before the dot product, so
// the small logit gaps are not the difference of two large fp32 logits.
// Grid = (group of kClusters key clusters, slice).  A block holds the
// slice's centroids q̄ transposed in shared memory ([k][a], up to 128 at a
// time) and walks each cluster's contiguous rows in 64-row chunks, centred
// and transposed ([k][j]); a thread accumulates an 8 x 4 tile (8 centroids x
// 4 keys) from one 8-wide and one 4-wide vector load per k, as packed fp32x2
// FMAs on centroid pairs (each element the same fma sequence over k).
#include "ear_internal.cuh"

namespace ear {
namespace {

constexpr int kA = 128;      // query centroids per pass
constexpr int kJ = 64;       // keys per chunk
constexpr int kClusters = 4; // key clusters per block
constexpr int kThreads = 256;

__device__ __forceinline__ unsigned long long pk2(float lo, float hi) {
  return (unsigned long long)__float_as_uint(lo) | ((unsigned long long)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
pr_probe(const float* __restrict__ qc, const int32_t* __restrict__ qn,
         const float* __restrict__ kc, const T* __restrict__ K,
         const int32_t* __restrict__ kperm, const int32_t* __restrict__ koff, int64_t Nk, int Cq,
         int Ck, float scale, float* __restrict__ E, int* status) {
  extern __shared__ float smem[];
  float* qs = smem;               // [D][kA]
  float* ks = qs + D * kA;        // [D][kJ]
  float* kbar = ks + D * kJ;      // [D]
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t h = blockIdx.y;
  const int32_t* oh = koff + h * (int64_t)(Ck + 1);
  const T* kh = K + h * Nk * D;

  for (int a0 = 0; a0 < Cq; a0 += kA) {
    __syncthreads();
    // q̄ chunk, transposed: lanes take consecutive centroids (conflict-free stores)
    for (int e = tid; e < kA * (D / 4); e += kThreads) {
      const int a = e % kA, k0 = (e / kA) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (a0 + a < Cq) v = *reinterpret_cast<const float4*>(qc + (h * Cq + a0 + a) * (int64_t)D + k0);
      qs[(k0 + 0) * kA + a] = v.x;
      qs[(k0 + 1) * kA + a] = v.y;
      qs[(k0 + 2) * kA + a] = v.z;
      qs[(k0 + 3) * kA + a] = v.w;
    }
    for (int bi = 0; bi < kClusters; ++bi) {
      const int b = blockIdx.x * kClusters + bi;
      if (b >= Ck) break;
      int32_t r0 = oh[b], r1 = oh[b + 1];
      if (r0 < 0 || r1 < r0 || r1 > Nk) {
        if (tid == 0) latch(status, EAR_ERR_DEVICE);
        r1 = r0 = 0;
      }
      __syncthreads();  // previous chunk's readers are done with ks / kbar
      for (int k = tid; k < D; k += kThreads) kbar[k] = kc[(h * Ck + b) * (int64_t)D + k];
      float part[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) part[i] = 0.f;
      for (int j0 = r0; j0 < r1; j0 += kJ) {
        const int nj = min(kJ, r1 - j0);
        __syncthreads();
        // centred keys, transposed: lanes take consecutive rows
        for (int e = tid; e < kJ * (D / 4); e += kThreads) {
          const int j = e % kJ, k0 = (e / kJ) * 4;
          float v[4] = {0.f, 0.f, 0.f, 0.f};
          // gather (kperm != nullptr): K in original order, permuted key r is row kperm[r]
          const int64_t src = j >= nj ? -1
                              : kperm == nullptr
                                  ? (int64_t)(j0 + j)
                                  : (int64_t)gather_row(kperm, h * Nk + j0 + j, h, Nk, status) - h * Nk;
          if (src >= 0) {
            const int64_t base = src * D + k0;
            float x[4];
            if constexpr (sizeof(T) == 2) {  // four bf16 in one 8-byte load
              const uint2 w = *reinterpret_cast<const uint2*>(kh + base);
              x[0] = __uint_as_float(w.x << 16);
              x[1] = __uint_as_float(w.x & 0xFFFF0000u);
              x[2] = __uint_as_float(w.y << 16);
              x[3] = __uint_as_float(w.y & 0xFFFF0000u);
            } else {
              const float4 w = *reinterpret_cast<const float4*>(kh + base);
              x[0] = w.x;
              x[1] = w.y;
              x[2] = w.z;
              x[3] = w.w;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = x[i] - kbar[k0 + i];
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) ks[(k0 + i) * kJ + j] = v[i];
        }
        __syncthreads();
        // acc2[ip][j] = (acc[2 ip][j], acc[2 ip + 1][j]): one packed fp32x2 FMA per
        // centroid pair and key, each lane the same fma sequence over k as a scalar loop
        unsigned long long acc2[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc2[i][j] = 0ull;
#pragma unroll 4
        for (int k = 0; k < D; ++k) {
          const float4 q0 = *reinterpret_cast<const float4*>(qs + k * kA + ty * 8);
          const float4 q1 = *reinterpret_cast<const float4*>(qs + k * kA + ty * 8 + 4);
          const float4 kv = *reinterpret_cast<const float4*>(ks + k * kJ + tx * 4);
          const unsigned long long qp[4] = {pk2(q0.x, q0.y), pk2(q0.z, q0.w), pk2(q1.x, q1.y),
                                            pk2(q1.z, q1.w)};
          const unsigned long long kp[4] = {pk2(kv.x, kv.x), pk2(kv.y, kv.y), pk2(kv.z, kv.z),
                                            pk2(kv.w, kv.w)};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc2[i][j] = fma2(qp[i], kp[j], acc2[i][j]);
        }
        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[2 * i][j] = __uint_as_float((uint32_t)acc2[i][j]);
            acc[2 * i + 1][j] = __uint_as_float((uint32_t)(acc2[i][j] >> 32));
          }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float g = scale * acc[i][j];  // zero for padded rows (centred value 0)
            part[i] = fmaf(g, g, part[i]);
          }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float v = part[i];
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        const int a = a0 + ty * 8 + i;
        if (tx == 0 && a < Cq) {
          const bool live = qn[h * Cq + a] > 0 && r1 > r0;
          E[(h * Cq + a) * (int64_t)Ck + b] = live ? v : 0.f;
        }
      }
    }
  }
}

template <typename T, int D>
ear_status run_t(const float* qc, const int32_t* qn, const float* kc, const void* K,
                 const int32_t* kperm, const int32_t* koff, int64_t bh, int64_t n_k, int32_t c_q,
                 int32_t c_k, float scale, float* E, cudaStream_t s) {
  const size_t smem = ((size_t)(kA + kJ) * D + D) * sizeof(float);
  EAR_CUDA(cudaFuncSetAttribute(pr_probe<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem));
  pr_probe<T, D><<<dim3((unsigned)ceil_div(c_k, kClusters), (unsigned)bh), kThreads, smem, s>>>(
      qc, qn, kc, (const T*)K, kperm, koff, n_k, c_q, c_k, scale, E, device_status_word());
  return after_launch();
}

}  // namespace

// bf16 keys run on the tensor cores (probe_tc.cu); fp32 keys here.
size_t probe_workspace(int64_t bh, int64_t n_k, int32_t d, int32_t c_q, int32_t c_k) {
  return probe_tc_workspace(bh, n_k, d, c_q, c_k);
}

// The weight probes (mode 1, 2) are built for bf16 keys only (the ABI rejects
// them for fp32 before this point).
ear_status probe_run(const float* qc, const int32_t* qn, const float* kc, const void* K,
                     const int32_t* kperm, ear_dtype dt, const int32_t* koff, int64_t bh,
                     int64_t n_k, int32_t d, int32_t c_q, int32_t c_k, float scale, int32_t mode,
                     const void* V, const float* vc, float* E, void* ws, cudaStream_t s) {
  if (dt == EAR_BF16)
    return probe_tc_run(qc, qn, kc, K, kperm, koff, bh, n_k, d, c_q, c_k, scale, mode, V, vc, E,
                        ws, s);
  return d == 64 ? run_t<float, 64>(qc, qn, kc, K, kperm, koff, bh, n_k, c_q, c_k, scale, E, s)
                 : run_t<float, 128>(qc, qn, kc, K, kperm, koff, bh, n_k, c_q, c_k, scale, E, s);
}

}  // namespace ear
