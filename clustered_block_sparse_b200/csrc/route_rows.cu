// Routing inside each query cluster under its own budget (SVG-EAR §5
// "Implementation": SVG2 gives every query cluster an adaptive budget, so
// SVG-EAR's routing runs per query cluster), and SVG2-style top-p budgets.
//
// Both run one CTA per (query cluster a, slice) with the row's C_k keys in
// shared memory, and place every block in the row's order by counting the
// blocks that precede it (O(C_k^2) comparisons per row, no sort):
//   rr_route   order = ratio E[a][b] / |b| descending (fp64, correctly
//              rounded), ties to the lower b.  A block is exact iff the cost
//              of the blocks before it plus its own fits the row's budget,
//              which is the greedy walk that stops at the first block that
//              does not fit (costs are positive, so the running cost only
//              grows).  Writes the exact row, its count and its pairs.
//   rr_lists   per slice: offsets = exclusive scan of the row counts, the
//              slice's pair total, and each row's list in ascending b.
//   rr_topp    centroid attention mass w_b = |b| e^{s q̄_a·k̄_b - max} in fp64
//              (the dot products summed in index order without contraction);
//              a key cluster is in the top-p set iff the mass of the clusters
//              before it (w descending, ties to the lower b) is below p times
//              the total; budget = |a| x the keys of the set.
#include <cmath>

#include "ear_internal.cuh"

namespace ear {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
rr_route(const float* __restrict__ E, const int32_t* __restrict__ qn_all,
         const int32_t* __restrict__ kn_all, int Cq, int Ck, const int64_t* __restrict__ budget,
         uint8_t* __restrict__ exact_all, int32_t* __restrict__ rcount,
         int64_t* __restrict__ rpairs) {
  extern __shared__ double sr[];                                        // [Ck] ratio (-1: none)
  long long* sc = reinterpret_cast<long long*>(sr + Ck);               // [Ck] cost
  __shared__ int s_cnt;
  __shared__ unsigned long long s_pairs;
  const int a = blockIdx.x;
  const int64_t h = blockIdx.y;
  const int64_t qa = qn_all[h * Cq + a];
  const int32_t* kn = kn_all + h * (int64_t)Ck;
  const float* Er = E + (h * Cq + a) * (int64_t)Ck;
  const int64_t B = budget[h * Cq + a];
  if (threadIdx.x == 0) {
    s_cnt = 0;
    s_pairs = 0;
  }
  for (int b = threadIdx.x; b < Ck; b += kThreads) {
    const long long cost = qa * (long long)kn[b];
    double r = -1.0;
    if (cost > 0) {
      r = (double)Er[b] / (double)kn[b];
      if (!(r > 0.0)) r = 0.0;  // folds -0 and non-finite values onto +0
    }
    sr[b] = r;
    sc[b] = cost;
  }
  __syncthreads();
  uint8_t* ex = exact_all + (h * Cq + a) * (int64_t)Ck;
  int cnt = 0;
  unsigned long long pairs = 0;
  for (int b = threadIdx.x; b < Ck; b += kThreads) {
    const double r = sr[b];
    const long long c = sc[b];
    bool take = false;
    if (c > 0) {
      long long before = 0;  // cost of the blocks that come before b
      for (int o = 0; o < Ck; ++o) {
        const double ro = sr[o];
        if (sc[o] > 0 && (ro > r || (ro == r && o < b))) before += sc[o];
      }
      take = before + c <= B;
    }
    ex[b] = take ? 1 : 0;
    if (take) {
      ++cnt;
      pairs += (unsigned long long)c;
    }
  }
  atomicAdd(&s_cnt, cnt);
  atomicAdd(&s_pairs, pairs);
  __syncthreads();
  if (threadIdx.x == 0) {
    rcount[h * Cq + a] = s_cnt;
    rpairs[h * Cq + a] = (int64_t)s_pairs;
  }
}

__global__ void __launch_bounds__(1024)
rr_lists(const uint8_t* __restrict__ exact_all, const int32_t* __restrict__ rcount,
         const int64_t* __restrict__ rpairs, int Cq, int Ck, int32_t* __restrict__ blk_off_all,
         int32_t* __restrict__ blk_list_all, int64_t* __restrict__ pairs_all) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t s_carry;
  __shared__ unsigned long long s_pairs;
  const int64_t h = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  int32_t* off = blk_off_all + h * (int64_t)(Cq + 1);
  if (tid == 0) {
    s_carry = 0;
    s_pairs = 0;
  }
  __syncthreads();
  unsigned long long mypairs = 0;
  for (int base = 0; base < Cq; base += 1024) {
    const int a = base + tid;
    const int32_t v = a < Cq ? rcount[h * Cq + a] : 0;
    if (a < Cq) mypairs += (unsigned long long)rpairs[h * Cq + a];
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int32_t w = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int32_t incl = x + (wid > 0 ? warp_sums[wid - 1] : 0) + s_carry;
    if (a < Cq) off[a] = incl - v;
    __syncthreads();
    if (tid == 1023) s_carry = incl;
    __syncthreads();
  }
  atomicAdd(&s_pairs, mypairs);
  __syncthreads();
  if (tid == 0) {
    off[Cq] = s_carry;
    pairs_all[h] = (int64_t)s_pairs;
  }
  __syncthreads();
  // lists: a warp per query cluster, ascending b
  const uint8_t* ex = exact_all + h * (int64_t)Cq * Ck;
  int32_t* lst = blk_list_all + h * (int64_t)Cq * Ck;
  for (int a = wid; a < Cq; a += 32) {
    int32_t pos = off[a];
    for (int b0 = 0; b0 < Ck; b0 += 32) {
      const int b = b0 + lane;
      const bool e = b < Ck && ex[(int64_t)a * Ck + b];
      const unsigned m = __ballot_sync(0xffffffffu, e);
      if (e) lst[pos + __popc(m & ((1u << lane) - 1u))] = b;
      pos += __popc(m);
    }
  }
}

__global__ void __launch_bounds__(kThreads)
rr_topp(const float* __restrict__ qc, const int32_t* __restrict__ qn_all,
        const float* __restrict__ kc, const int32_t* __restrict__ kn_all, int D, int Cq, int Ck,
        double scale, double p, int64_t* __restrict__ budget) {
  extern __shared__ double sw[];                 // [Ck] mass (-1: empty cluster)
  double* sq = sw + Ck;                          // [D] q̄_a
  __shared__ double s_red[kThreads / 32];
  __shared__ unsigned long long s_keys;
  const int a = blockIdx.x;
  const int64_t h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int64_t qa = qn_all[h * Cq + a];
  const int32_t* kn = kn_all + h * (int64_t)Ck;
  if (tid == 0) s_keys = 0;
  for (int k = tid; k < D; k += kThreads) sq[k] = (double)qc[(h * Cq + a) * (int64_t)D + k];
  __syncthreads();
  // logits, then their maximum
  double zmax = -INFINITY;
  for (int b = tid; b < Ck; b += kThreads) {
    double z = -INFINITY;
    if (kn[b] > 0) {
      const float* kb = kc + (h * Ck + b) * (int64_t)D;
      double dot = 0.0;
      for (int k = 0; k < D; ++k) dot = __dadd_rn(dot, __dmul_rn(sq[k], (double)kb[k]));
      z = __dmul_rn(scale, dot);
    }
    sw[b] = z;
    zmax = fmax(zmax, z);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) zmax = fmax(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
  if (lane == 0) s_red[wid] = zmax;
  __syncthreads();
  zmax = s_red[0];
  for (int i = 1; i < kThreads / 32; ++i) zmax = fmax(zmax, s_red[i]);
  __syncthreads();
  // masses and their total
  double tot = 0.0;
  for (int b = tid; b < Ck; b += kThreads) {
    const double w = kn[b] > 0 ? (double)kn[b] * exp(sw[b] - zmax) : -1.0;
    sw[b] = w;
    if (w > 0.0) tot += w;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  __syncthreads();
  if (lane == 0) s_red[wid] = tot;
  __syncthreads();
  tot = 0.0;
  for (int i = 0; i < kThreads / 32; ++i) tot += s_red[i];
  const double target = p * tot;
  unsigned long long keys = 0;
  for (int b = tid; b < Ck; b += kThreads) {
    const double w = sw[b];
    if (!(w >= 0.0)) continue;
    double before = 0.0;  // mass of the clusters that come before b
    for (int o = 0; o < Ck; ++o) {
      const double wo = sw[o];
      if (wo >= 0.0 && (wo > w || (wo == w && o < b))) before += wo;
    }
    if (before < target) keys += (unsigned long long)kn[b];
  }
  atomicAdd(&s_keys, keys);
  __syncthreads();
  if (tid == 0) budget[h * Cq + a] = qa > 0 ? qa * (int64_t)s_keys : 0;
}

__global__ void rr_uniform(const int32_t* __restrict__ qn, int64_t rows, int64_t n_k,
                           double density, int64_t* __restrict__ budget) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < rows) budget[i] = (int64_t)floor(density * (double)((int64_t)qn[i] * n_k));
}

}  // namespace

size_t route_rows_workspace(int64_t bh, int32_t c_q) {
  Carver cv(nullptr);
  cv.take<int32_t>((size_t)bh * c_q);
  cv.take<int64_t>((size_t)bh * c_q);
  return cv.used;
}

ear_status route_rows_run(const float* E, const int32_t* qn, const int32_t* kn, int64_t bh,
                          int32_t c_q, int32_t c_k, const int64_t* row_budget, uint8_t* exact,
                          int32_t* blk_off, int32_t* blk_list, int64_t* pairs, void* ws,
                          cudaStream_t s) {
  Carver cv(ws);
  int32_t* rcount = cv.take<int32_t>((size_t)bh * c_q);
  int64_t* rpairs = cv.take<int64_t>((size_t)bh * c_q);
  const size_t smem = (size_t)c_k * (sizeof(double) + sizeof(long long));
  EAR_CUDA(cudaFuncSetAttribute(rr_route, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  rr_route<<<dim3((unsigned)c_q, (unsigned)bh), kThreads, smem, s>>>(
      E, qn, kn, c_q, c_k, row_budget, exact, rcount, rpairs);
  EAR_TRY(after_launch());
  rr_lists<<<(unsigned)bh, 1024, 0, s>>>(exact, rcount, rpairs, c_q, c_k, blk_off, blk_list, pairs);
  return after_launch();
}

ear_status topp_budget_run(const float* qc, const int32_t* qn, const float* kc, const int32_t* kn,
                           int64_t bh, int32_t d, int32_t c_q, int32_t c_k, float scale, double p,
                           int64_t* budget, cudaStream_t s) {
  const size_t smem = ((size_t)c_k + d) * sizeof(double);
  EAR_CUDA(cudaFuncSetAttribute(rr_topp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  rr_topp<<<dim3((unsigned)c_q, (unsigned)bh), kThreads, smem, s>>>(qc, qn, kc, kn, d, c_q, c_k,
                                                                  (double)scale, p, budget);
  return after_launch();
}

ear_status uniform_budget_run(const int32_t* qn, int64_t bh, int32_t c_q, int64_t n_k,
                              double density, int64_t* budget, cudaStream_t s) {
  const int64_t rows = bh * c_q;
  rr_uniform<<<(unsigned)ceil_div(rows, 256), 256, 0, s>>>(qn, rows, n_k, density, budget);
  return after_launch();
}

}  // namespace ear
