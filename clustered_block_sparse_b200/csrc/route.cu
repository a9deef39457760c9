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
// One 1024-thread block per slice: keys and costs once into the workspace,
// select (each pass: a warp whose lanes share one digit adds the costs in
// registers and makes one shared-memory atomic; warp 0 scans the histogram),
// mark, count per query cluster, scan, and emit each query cluster's exact
// key clusters in ascending order.
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

}  // namespace

// keys (fp64 ratio bits) and costs of every block, 8 + 8 bytes each
size_t route_workspace(int64_t bh, int32_t c_q, int32_t c_k) {
  return (size_t)bh * c_q * c_k * 16;
}

ear_status route_run(const float* E, const int32_t* qn, const int32_t* kn, int64_t bh,
                     int64_t budget, int32_t c_q, int32_t c_k, int32_t mode, uint8_t* exact,
                     int32_t* blk_off, int32_t* blk_list, int64_t* pairs, void* ws,
                     cudaStream_t s) {
  uint64_t* khi = static_cast<uint64_t*>(ws);
  unsigned long long* cost = reinterpret_cast<unsigned long long*>(khi + bh * c_q * c_k);
  rt_route<<<(unsigned)bh, kThreads, 0, s>>>(E, qn, kn, c_q, c_k, budget, mode, exact, blk_off,
                                             blk_list, pairs, khi, cost);
  return after_launch();
}

}  // namespace ear
