// Greedy error-to-cost routing (SVG-EAR §4.2 "Error estimation": blocks are
// computed exactly in decreasing order of error-to-size ratio until the
// budget is spent; §4.1: the budget is rho N_q N_k pairs).
//
// The greedy walk over the sorted blocks accepts block i exactly when the
// running cost up to and including i is <= B (costs are positive, so the
// running cost only grows).  So the exact set is every block whose sort key
// is below K*, the key of the first block whose running cost exceeds B.  K*
// is found without sorting by a cost-weighted radix select: the 96-bit key
// (bit-inverted fp64 ratio, then block index) is scanned 8 bits at a time
// from the top; in each pass a 256-bucket histogram of block COSTS picks the
// digit at which the running cost crosses the remaining budget.  Ratios are
// correctly rounded fp64 divisions, so the order matches a host fp64 sort.
//
// Main path (C_q <= 512 and C_q C_k <= 8 x kKeysPerCta): one cluster of 8 CTAs of 512 threads
// per slice.
// Each CTA keeps the keys of its eighth of the blocks in shared memory; in
// each pass every CTA adds its costs into the histogram of CTA 0 through
// distributed shared memory (a warp whose lanes share one digit adds them in
// registers first), the cluster synchronises, warp 0 of CTA 0 picks the digit,
// and the cluster synchronises again.  Then every CTA marks its blocks,
// counts and scans per query cluster, and emits the lists of its share of the
// query clusters.  Larger problems use one 1024-thread block per slice with
// the keys in the workspace.
#include <cooperative_groups.h>

#include "ear_internal.cuh"

namespace ear {
namespace {

constexpr int kThreads = 1024;

struct Key {
  uint64_t hi;  // ~bits(ratio): a larger ratio gives a smaller key
  uint32_t lo;  // linear block index a*C_k + b: ties to the lower index
};

__device__ __forceinline__ bool block_key(const float* __restrict__ Eh,
                                          const int32_t* __restrict__ qn,
                                          const int32_t* __restrict__ kn, int Ck, int mode,
                                          int idx, Key& key, unsigned long long& cost) {
  const int a = idx / Ck, b = idx - (idx / Ck) * Ck;
  const int64_t c = (int64_t)qn[a] * (int64_t)kn[b];
  if (c <= 0) return false;
  const double e = (double)Eh[idx];
  double r = mode == 0 ? e / (double)kn[b] : e / (double)c;
  if (!(r > 0.0)) r = 0.0;  // folds -0 (and any non-finite garbage) onto +0
  key.hi = ~(uint64_t)__double_as_longlong(r);
  key.lo = (uint32_t)idx;
  cost = (unsigned long long)c;
  return true;
}

__device__ __forceinline__ int digit_of(const Key& k, int pass) {
  return pass < 8 ? (int)((k.hi >> (56 - 8 * pass)) & 0xFF)
                  : (int)((k.lo >> (24 - 8 * (pass - 8))) & 0xFF);
}

__device__ __forceinline__ bool prefix_match(const Key& k, int pass, uint64_t phi, uint32_t plo) {
  if (pass <= 8) {
    const uint64_t mask = pass == 0 ? 0ull : (~0ull << (64 - 8 * pass));
    return (k.hi & mask) == phi;
  }
  const uint32_t mask = ~0u << (32 - 8 * (pass - 8));
  return k.hi == phi && (k.lo & mask) == plo;
}

__device__ __forceinline__ bool key_less(const Key& k, uint64_t hi, uint32_t lo) {
  return k.hi < hi || (k.hi == hi && k.lo < lo);
}

__global__ void __launch_bounds__(kThreads)
rt_route(const float* __restrict__ E, const int32_t* __restrict__ qn_all,
         const int32_t* __restrict__ kn_all, int Cq, int Ck, int64_t budget, int mode,
         uint8_t* __restrict__ exact_all, int32_t* __restrict__ blk_off_all,
         int32_t* __restrict__ blk_list_all, int64_t* __restrict__ pairs,
         uint64_t* __restrict__ khi_ws, unsigned long long* __restrict__ cost_ws) {
  __shared__ unsigned long long hist[256];
  __shared__ uint64_t s_phi;
  __shared__ uint32_t s_plo;
  __shared__ long long s_rem;
  __shared__ int s_all_fit;
  __shared__ unsigned long long s_total;
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t s_carry;

  const int64_t h = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nblk = Cq * Ck;
  const float* Eh = E + h * (int64_t)nblk;
  const int32_t* qn = qn_all + h * (int64_t)Cq;
  const int32_t* kn = kn_all + h * (int64_t)Ck;
  uint8_t* exact = exact_all + h * (int64_t)nblk;
  int32_t* blk_off = blk_off_all + h * (int64_t)(Cq + 1);
  int32_t* blk_list = blk_list_all + h * (int64_t)nblk;
  uint64_t* khi = khi_ws + h * (int64_t)nblk;
  unsigned long long* cost = cost_ws + h * (int64_t)nblk;

  if (tid == 0) {
    s_phi = 0;
    s_plo = 0;
    s_rem = budget;
    s_all_fit = 0;
    s_total = 0;
  }
  // keys once (cost 0 = never exact)
  for (int idx = tid; idx < nblk; idx += kThreads) {
    Key k;
    unsigned long long c = 0;
    if (!block_key(Eh, qn, kn, Ck, mode, idx, k, c)) {
      k.hi = 0;
      c = 0;
    }
    khi[idx] = k.hi;
    cost[idx] = c;
  }
  for (int pass = 0; pass < 12; ++pass) {
    for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    const uint64_t phi = s_phi;
    const uint32_t plo = s_plo;
    for (int base = 0; base < nblk; base += kThreads) {
      const int idx = base + tid;
      Key k;
      unsigned long long c = 0;
      if (idx < nblk) {
        k.hi = khi[idx];
        k.lo = (uint32_t)idx;
        c = cost[idx];
      }
      const bool want = c > 0 && prefix_match(k, pass, phi, plo);
      const int d = want ? digit_of(k, pass) : -1;
      // the early passes see one digit across the warp: add in registers
      if (__all_sync(0xffffffffu, d == __shfl_sync(0xffffffffu, d, 0) && want)) {
        unsigned long long sum = c;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) atomicAdd(&hist[d], sum);
      } else if (want) {
        atomicAdd(&hist[d], c);
      }
    }
    __syncthreads();
    if (wid == 0) {
      // first digit u with (costs below u) + hist[u] > remaining budget
      const unsigned long long rem = (unsigned long long)s_rem;
      unsigned long long v[8], loc = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] = hist[lane * 8 + i];
        loc += v[i];
      }
      unsigned long long incl = loc;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const unsigned long long excl = incl - loc;
      const bool mine = excl <= rem && incl > rem;
      const unsigned m = __ballot_sync(0xffffffffu, mine);
      const unsigned long long total = __shfl_sync(0xffffffffu, incl, 31);
      if (m == 0) {
        if (lane == 0) {
          s_all_fit = 1;  // everything fits: only possible in the first pass
          if (pass == 0) s_total = total;
        }
      } else if (mine) {
        unsigned long long cum = excl;
        int t = lane * 8 + 7;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (cum + v[i] > rem) {
            t = lane * 8 + i;
            break;
          }
          cum += v[i];
        }
        s_rem = (long long)(rem - cum);
        if (pass < 8)
          s_phi |= (uint64_t)t << (56 - 8 * pass);
        else
          s_plo |= (uint32_t)t << (24 - 8 * (pass - 8));
      }
    }
    __syncthreads();
    if (s_all_fit) break;
  }
  const bool all_fit = s_all_fit != 0;
  const uint64_t kstar_hi = s_phi;
  const uint32_t kstar_lo = s_plo;

  // mark
  for (int idx = tid; idx < nblk; idx += kThreads) {
    Key k;
    k.hi = khi[idx];
    k.lo = (uint32_t)idx;
    const bool ex = cost[idx] > 0 && (all_fit || key_less(k, kstar_hi, kstar_lo));
    exact[idx] = ex ? 1 : 0;
  }
  if (tid == 0) pairs[h] = all_fit ? (int64_t)s_total : (int64_t)(budget - s_rem);
  __syncthreads();

  // exact key clusters per query cluster
  for (int a = wid; a < Cq; a += kThreads / 32) {
    int cnt = 0;
    for (int b = lane; b < Ck; b += 32) cnt += exact[(int64_t)a * Ck + b];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if (lane == 0) blk_off[a] = cnt;
  }
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < Cq; base += kThreads) {
    const int a = base + tid;
    const int32_t v = a < Cq ? blk_off[a] : 0;
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
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int32_t incl = x + (wid > 0 ? warp_sums[wid - 1] : 0) + s_carry;
    __syncthreads();
    if (a < Cq) blk_off[a] = incl - v;
    if (tid == kThreads - 1) s_carry = incl;
    __syncthreads();
  }
  if (tid == 0) blk_off[Cq] = s_carry;
  __syncthreads();
  for (int a = wid; a < Cq; a += kThreads / 32) {
    int32_t pos = blk_off[a];
    for (int b0 = 0; b0 < Ck; b0 += 32) {
      const int b = b0 + lane;
      const bool ex = b < Ck && exact[(int64_t)a * Ck + b];
      const unsigned m = __ballot_sync(0xffffffffu, ex);
      if (ex) blk_list[pos + __popc(m & ((1u << lane) - 1u))] = b;
      pos += __popc(m);
    }
  }
}

constexpr int kCluster = 8;
constexpr int kKeysPerCta = 16384;  // 128 KB of keys per CTA
constexpr int kCThreads = 512;      // threads of a cluster CTA: two CTAs fit one SM

namespace cg = cooperative_groups;

// dynamic shared memory of one CTA: keys, then q / k counts, then per-query-
// cluster counts and offsets
size_t cluster_smem(int Cq, int Ck, int64_t per) {
  return (size_t)per * 8 + (size_t)(Cq + Ck) * 4 + (size_t)(Cq + 1) * 8;
}

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kCThreads)
rt_route_cluster(const float* __restrict__ E, const int32_t* __restrict__ qn_all,
                 const int32_t* __restrict__ kn_all, int Cq, int Ck, int64_t budget, int mode,
                 uint8_t* __restrict__ exact_all, int32_t* __restrict__ blk_off_all,
                 int32_t* __restrict__ blk_list_all, int64_t* __restrict__ pairs) {
  extern __shared__ uint64_t dyn[];
  __shared__ unsigned long long hist[256];  // CTA 0's is the cluster's
  __shared__ uint64_t s_phi;
  __shared__ uint32_t s_plo;
  __shared__ long long s_rem;
  __shared__ int s_all_fit;
  __shared__ unsigned long long s_total;
  __shared__ int32_t warp_sums[32];

  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int64_t h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nblk = Cq * Ck;
  const int per = (nblk + kCluster - 1) / kCluster;
  const int i0 = rank * per;
  const int i1 = min(nblk, i0 + per);
  uint64_t* skey = dyn;                                          // [per]
  int32_t* sqn = reinterpret_cast<int32_t*>(skey + per);          // [Cq]
  int32_t* skn = sqn + Cq;                                       // [Ck]
  int32_t* scnt = skn + Ck;                                      // [Cq + 1]
  int32_t* soff = scnt + Cq + 1;                                 // [Cq + 1]
  const float* Eh = E + h * (int64_t)nblk;
  uint8_t* exact = exact_all + h * (int64_t)nblk;
  int32_t* blk_off = blk_off_all + h * (int64_t)(Cq + 1);
  int32_t* blk_list = blk_list_all + h * (int64_t)nblk;

  for (int i = tid; i < Cq; i += kCThreads) sqn[i] = qn_all[h * Cq + i];
  for (int i = tid; i < Ck; i += kCThreads) skn[i] = kn_all[h * Ck + i];
  for (int i = tid; i < 256; i += kCThreads) hist[i] = 0;
  if (tid == 0) {
    s_phi = 0;
    s_plo = 0;
    s_rem = budget;
    s_all_fit = 0;
    s_total = 0;
  }
  __syncthreads();
  for (int idx = i0 + tid; idx < i1; idx += kCThreads) {
    Key k;
    unsigned long long c = 0;
    skey[idx - i0] = block_key(Eh, sqn, skn, Ck, mode, idx, k, c) ? k.hi : 0ull;
  }
  cl.sync();
  unsigned long long* hist0 = cl.map_shared_rank(hist, 0);
  uint64_t* phi0 = cl.map_shared_rank(&s_phi, 0);
  uint32_t* plo0 = cl.map_shared_rank(&s_plo, 0);
  int* fit0 = cl.map_shared_rank(&s_all_fit, 0);
  for (int pass = 0; pass < 12; ++pass) {
    const uint64_t phi = *phi0;
    const uint32_t plo = *plo0;
    for (int base = i0; base < i1; base += kCThreads) {
      const int idx = base + tid;
      Key k;
      unsigned long long c = 0;
      if (idx < i1) {
        const int a = idx / Ck, b = idx - a * Ck;
        c = (unsigned long long)((int64_t)sqn[a] * (int64_t)skn[b]);
        k.hi = skey[idx - i0];
        k.lo = (uint32_t)idx;
      }
      const bool want = c > 0 && prefix_match(k, pass, phi, plo);
      const int d = want ? digit_of(k, pass) : -1;
      if (__all_sync(0xffffffffu, d == __shfl_sync(0xffffffffu, d, 0) && want)) {
        unsigned long long sum = c;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) atomicAdd(&hist0[d], sum);
      } else if (want) {
        atomicAdd(&hist0[d], c);
      }
    }
    cl.sync();
    if (rank == 0 && wid == 0) {
      // first digit u with (costs below u) + hist[u] > remaining budget
      const unsigned long long rem = (unsigned long long)s_rem;
      unsigned long long v[8], loc = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] = hist[lane * 8 + i];
        hist[lane * 8 + i] = 0;  // ready for the next pass
        loc += v[i];
      }
      unsigned long long incl = loc;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const unsigned long long excl = incl - loc;
      const bool mine = excl <= rem && incl > rem;
      const unsigned m = __ballot_sync(0xffffffffu, mine);
      const unsigned long long total = __shfl_sync(0xffffffffu, incl, 31);
      if (m == 0) {
        if (lane == 0) {
          s_all_fit = 1;  // everything fits: only possible in the first pass
          if (pass == 0) s_total = total;
        }
      } else if (mine) {
        unsigned long long cum = excl;
        int t = lane * 8 + 7;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (cum + v[i] > rem) {
            t = lane * 8 + i;
            break;
          }
          cum += v[i];
        }
        s_rem = (long long)(rem - cum);
        if (pass < 8)
          s_phi |= (uint64_t)t << (56 - 8 * pass);
        else
          s_plo |= (uint32_t)t << (24 - 8 * (pass - 8));
      }
    }
    cl.sync();
    if (*fit0) break;
  }
  const bool all_fit = *fit0 != 0;
  const uint64_t kstar_hi = *phi0;
  const uint32_t kstar_lo = *plo0;
  // mark this CTA's blocks
  for (int idx = i0 + tid; idx < i1; idx += kCThreads) {
    const int a = idx / Ck, b = idx - a * Ck;
    const bool live = (int64_t)sqn[a] * (int64_t)skn[b] > 0;
    Key k;
    k.hi = skey[idx - i0];
    k.lo = (uint32_t)idx;
    exact[idx] = live && (all_fit || key_less(k, kstar_hi, kstar_lo)) ? 1 : 0;
  }
  if (rank == 0 && tid == 0)
    pairs[h] = all_fit ? (int64_t)s_total : (int64_t)(budget - s_rem);
  cl.sync();  // every CTA's marks are visible to the cluster
  // exact key clusters per query cluster, and their offsets (every CTA)
  for (int a = wid; a < Cq; a += kCThreads / 32) {
    int cnt = 0;
    for (int b = lane; b < Ck; b += 32) cnt += exact[(int64_t)a * Ck + b];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if (lane == 0) scnt[a] = cnt;
  }
  __syncthreads();
  {  // exclusive scan of the counts (the cluster path has C_q <= kCThreads)
    const int a = tid;
    const int32_t v = a < Cq ? scnt[a] : 0;
    int32_t x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int32_t w = warp_sums[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += y;
      }
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int32_t incl = x + (wid > 0 ? warp_sums[wid - 1] : 0);
    if (a < Cq) soff[a] = incl - v;
    if (a == Cq - 1) soff[Cq] = incl;
    __syncthreads();
  }
  if (rank == 0)
    for (int a = tid; a <= Cq; a += kCThreads) blk_off[a] = soff[a];
  // lists of this CTA's share of the query clusters (a = rank, rank + 8, ...)
  for (int a = rank + kCluster * wid; a < Cq; a += kCluster * (kCThreads / 32)) {
    int32_t pos = soff[a];
    for (int b0 = 0; b0 < Ck; b0 += 32) {
      const int b = b0 + lane;
      const bool ex = b < Ck && exact[(int64_t)a * Ck + b];
      const unsigned m = __ballot_sync(0xffffffffu, ex);
      if (ex) blk_list[pos + __popc(m & ((1u << lane) - 1u))] = b;
      pos += __popc(m);
    }
  }
  cl.sync();  // no CTA leaves while others may still read its shared memory
}

}  // namespace

namespace {
constexpr size_t kClusterSmemMax = 200 * 1024;

bool use_cluster(int32_t c_q, int32_t c_k) {
  const int64_t nblk = (int64_t)c_q * c_k;
  const int64_t per = (nblk + kCluster - 1) / kCluster;
  return c_q <= kCThreads && per <= kKeysPerCta && cluster_smem(c_q, c_k, per) <= kClusterSmemMax;
}
}  // namespace

// cluster path: nothing; otherwise the keys (fp64 ratio bits) and costs of
// every block, 8 + 8 bytes each
size_t route_workspace(int64_t bh, int32_t c_q, int32_t c_k) {
  return use_cluster(c_q, c_k) ? 0 : (size_t)bh * c_q * c_k * 16;
}

ear_status route_run(const float* E, const int32_t* qn, const int32_t* kn, int64_t bh,
                     int64_t budget, int32_t c_q, int32_t c_k, int32_t mode, uint8_t* exact,
                     int32_t* blk_off, int32_t* blk_list, int64_t* pairs, void* ws,
                     cudaStream_t s) {
  if (use_cluster(c_q, c_k)) {
    const int64_t per = ((int64_t)c_q * c_k + kCluster - 1) / kCluster;
    const size_t smem = cluster_smem(c_q, c_k, per);
    EAR_CUDA(cudaFuncSetAttribute(rt_route_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem));
    rt_route_cluster<<<dim3(kCluster, (unsigned)bh), kCThreads, smem, s>>>(
        E, qn, kn, c_q, c_k, budget, mode, exact, blk_off, blk_list, pairs);
    return after_launch();
  }
  uint64_t* khi = static_cast<uint64_t*>(ws);
  unsigned long long* cost = reinterpret_cast<unsigned long long*>(khi + bh * c_q * c_k);
  rt_route<<<(unsigned)bh, kThreads, 0, s>>>(E, qn, kn, c_q, c_k, budget, mode, exact, blk_off,
                                             blk_list, pairs, khi, cost);
  return after_launch();
}

}  // namespace ear
