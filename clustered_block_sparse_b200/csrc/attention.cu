// Block-sparse attention with linear compensation (SVG-EAR §4.1 routing mask,
// §4.3 Linear Compensation) - work planning, the fp32 SIMT kernel and the
// dispatch between it and the tensor-core kernel.
//
// For query i of cluster a, one softmax (base 2, logits pre-scaled by
// s log2 e) runs over
//   exact terms:        s q_i·k_j, value v_j, keys j of every b in blk_list[a]
//   compensated terms:  s q_i·k̄_b + log2|b| (i.e. weight |b|), value v̄_b,
//                       for every b with exact[a][b] = 0 and |b| > 0.
// O is written at the query's original index (q_perm), lse = m + ln(l).
#include <cmath>

#include "ear_internal.cuh"

namespace ear {

// Query tiles of `tile` rows that never straddle two query clusters:
// items[h][slot] = (a, first permuted row), count[h] = number of items.
__global__ void __launch_bounds__(1024)
at_plan(const int32_t* __restrict__ q_off_all, int Cq, int tile, int64_t max_items,
        int2* __restrict__ items_all, int32_t* __restrict__ count_all) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t s_carry;
  const int64_t h = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int32_t* q_off = q_off_all + h * (int64_t)(Cq + 1);
  int2* items = items_all + h * max_items;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < Cq; base += 1024) {
    const int a = base + tid;
    int32_t r0 = 0, r1 = 0, v = 0;
    if (a < Cq) {
      r0 = q_off[a];
      r1 = q_off[a + 1];
      v = r1 > r0 ? (r1 - r0 + tile - 1) / tile : 0;
    }
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
    const int32_t first = incl - v;
    for (int t = 0; t < v && first + t < max_items; ++t) items[first + t] = make_int2(a, r0 + t * tile);
    __syncthreads();
    if (tid == 1023) s_carry = incl;
    __syncthreads();
  }
  if (tid == 0) count_all[h] = (int32_t)(s_carry < max_items ? s_carry : max_items);
}

namespace {

constexpr int kTile = kAttnTileRows;  // 64 queries per block
constexpr int kKeys = 64;             // keys (or centroids) per chunk
constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// thread (r = tid / 4, part = tid % 4): query row r; logits of keys part + 4*jj;
// output dims part + 4*i.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
at_simt(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
        const int32_t* __restrict__ q_off_all, const int32_t* __restrict__ k_off_all,
        const int32_t* __restrict__ q_perm_all, const int32_t* __restrict__ k_perm_all,
        const float* __restrict__ kc_all,
        const float* __restrict__ vc_all, const uint8_t* __restrict__ exact_all,
        const int32_t* __restrict__ blk_off_all, const int32_t* __restrict__ blk_list_all,
        const int2* __restrict__ items_all, const int32_t* __restrict__ count_all,
        int64_t max_items, int64_t Nq, int64_t Nk, int Cq, int Ck, float scale, int compensate,
        T* __restrict__ O, float* __restrict__ lse_out, int* status) {
  constexpr int QS = D + 4;  // padded strides (see the index maps above)
  constexpr int KS = D + 1;
  constexpr int PS = kKeys + 1;
  extern __shared__ float smem[];
  float* qs = smem;                 // [kTile][QS]
  float* ks = qs + kTile * QS;      // [kKeys][KS]
  float* vs = ks + kKeys * KS;      // [kKeys][KS]
  float* ps = vs + kKeys * KS;      // [kTile][PS]
  float* bias = ps + kTile * PS;    // [kKeys]

  const int64_t h = blockIdx.y;
  const int64_t slot = blockIdx.x;
  if (slot >= count_all[h]) return;
  const int2 item = items_all[h * max_items + slot];
  const int a = item.x;
  const int32_t* q_off = q_off_all + h * (int64_t)(Cq + 1);
  const int32_t* k_off = k_off_all + h * (int64_t)(Ck + 1);
  const int32_t row0 = item.y;
  if (row0 < 0 || q_off[a + 1] > Nq) {
    if (threadIdx.x == 0) latch(status, EAR_ERR_DEVICE);
    return;
  }
  const int nrows = min(kTile, q_off[a + 1] - row0);
  const int tid = threadIdx.x, r = tid >> 2, part = tid & 3;
  const T* Qh = Q + h * Nq * D;
  const T* Kh = K + h * Nk * D;
  const T* Vh = V + h * Nk * D;
  const float qscale = scale * kLog2e;

  // k_perm_all != nullptr (gather): Q, K and V are in original token order;
  // permuted row r is original row q_perm[r] / k_perm[r].
  const int32_t* qp = k_perm_all != nullptr ? q_perm_all + h * Nq : nullptr;
  const int32_t* kp = k_perm_all != nullptr ? k_perm_all + h * Nk : nullptr;
  auto src_row = [&](const int32_t* perm, int64_t r, int64_t n) -> int64_t {
    if (perm == nullptr) return r;
    const int32_t o = perm[r];
    if (o < 0 || o >= n) {
      latch(status, EAR_ERR_DEVICE);
      return -1;
    }
    return o;
  };
  for (int e = tid; e < kTile * D; e += kThreads) {
    const int rr = e / D, k = e % D;
    const int64_t src = rr < nrows ? src_row(qp, row0 + rr, Nq) : -1;
    qs[rr * QS + k] = src >= 0 ? Elem<T>::load(Qh, src * D + k) * qscale : 0.f;
  }

  float m = -INFINITY, l = 0.f;
  float o[D / 4];
#pragma unroll
  for (int i = 0; i < D / 4; ++i) o[i] = 0.f;

  // One chunk of up to kKeys keys already staged in ks / vs / bias.
  auto consume = [&](int nvalid) {
    __syncthreads();
    float sv[kKeys / 4];
#pragma unroll
    for (int jj = 0; jj < kKeys / 4; ++jj) sv[jj] = 0.f;
#pragma unroll 2
    for (int k = 0; k < D; ++k) {
      const float qv = qs[r * QS + k];
#pragma unroll
      for (int jj = 0; jj < kKeys / 4; ++jj) sv[jj] = fmaf(qv, ks[(part + 4 * jj) * KS + k], sv[jj]);
    }
    float cmax = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < kKeys / 4; ++jj) {
      const int j = part + 4 * jj;
      sv[jj] = j < nvalid ? sv[jj] + bias[j] : -INFINITY;
      cmax = fmaxf(cmax, sv[jj]);
    }
    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 2));
    const float mnew = fmaxf(m, cmax);
    const float corr = mnew == -INFINITY ? 1.f : exp2f(m - mnew);
    float psum = 0.f;
#pragma unroll
    for (int jj = 0; jj < kKeys / 4; ++jj) {
      const float p = mnew == -INFINITY ? 0.f : exp2f(sv[jj] - mnew);
      psum += p;
      ps[r * PS + part + 4 * jj] = p;
    }
    psum += __shfl_xor_sync(0xffffffffu, psum, 1);
    psum += __shfl_xor_sync(0xffffffffu, psum, 2);
    l = l * corr + psum;
    m = mnew;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < D / 4; ++i) o[i] *= corr;
    for (int j = 0; j < nvalid; ++j) {
      const float p = ps[r * PS + j];
#pragma unroll
      for (int i = 0; i < D / 4; ++i) o[i] = fmaf(p, vs[j * KS + part + 4 * i], o[i]);
    }
  };

  // exact blocks
  const int32_t* blk_off = blk_off_all + h * (int64_t)(Cq + 1);
  const int32_t* blk_list = blk_list_all + h * (int64_t)Cq * Ck;
  const int32_t e0 = blk_off[a], e1 = blk_off[a + 1];
  for (int32_t e = e0; e < e1; ++e) {
    const int b = blk_list[e];
    if (b < 0 || b >= Ck) {
      if (tid == 0) latch(status, EAR_ERR_DEVICE);
      continue;
    }
    const int32_t k0 = k_off[b], k1 = k_off[b + 1];
    if (k0 < 0 || k1 > Nk) {
      if (tid == 0) latch(status, EAR_ERR_DEVICE);
      continue;
    }
    for (int32_t j0 = k0; j0 < k1; j0 += kKeys) {
      const int nv = min(kKeys, k1 - j0);
      __syncthreads();
      for (int x = tid; x < kKeys * D; x += kThreads) {
        const int j = x / D, k = x % D;
        const int64_t src = j < nv ? src_row(kp, j0 + j, Nk) : -1;
        ks[j * KS + k] = src >= 0 ? Elem<T>::load(Kh, src * D + k) : 0.f;
        vs[j * KS + k] = src >= 0 ? Elem<T>::load(Vh, src * D + k) : 0.f;
      }
      if (tid < kKeys) bias[tid] = 0.f;
      consume(nv);
    }
  }
  // compensated clusters: centroid "keys" with weight |b|
  if (compensate) {
    const uint8_t* ex = exact_all + (h * Cq + a) * (int64_t)Ck;
    const float* kc = kc_all + h * (int64_t)Ck * D;
    const float* vc = vc_all + h * (int64_t)Ck * D;
    for (int c0 = 0; c0 < Ck; c0 += kKeys) {
      const int nv = min(kKeys, Ck - c0);
      __syncthreads();
      for (int x = tid; x < kKeys * D; x += kThreads) {
        const int j = x / D, k = x % D;
        const bool ok = j < nv;
        ks[j * KS + k] = ok ? kc[(int64_t)(c0 + j) * D + k] : 0.f;
        vs[j * KS + k] = ok ? vc[(int64_t)(c0 + j) * D + k] : 0.f;
      }
      if (tid < kKeys) {
        float bv = -INFINITY;
        const int b = c0 + tid;
        if (tid < nv) {
          const int32_t cnt = k_off[b + 1] - k_off[b];
          if (!ex[b] && cnt > 0) bv = log2f((float)cnt);
        }
        bias[tid] = bv;
      }
      consume(nv);
    }
  }

  if (r < nrows) {
    const int32_t orig = q_perm_all[h * Nq + row0 + r];
    if (orig < 0 || orig >= Nq) {
      latch(status, EAR_ERR_DEVICE);
      return;
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    T* orow = O + (h * Nq + orig) * D;
#pragma unroll
    for (int i = 0; i < D / 4; ++i) Elem<T>::store(orow, part + 4 * i, o[i] * inv);
    if (lse_out != nullptr && part == 0)
      lse_out[h * Nq + orig] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
  }
}

template <typename T, int D>
ear_status simt_t(const AttnArgs& a, const int2* items, const int32_t* count, int64_t max_items,
                  cudaStream_t s) {
  constexpr int QS = D + 4, KS = D + 1, PS = kKeys + 1;
  const size_t smem = (size_t)(kTile * QS + 2 * kKeys * KS + kTile * PS + kKeys) * sizeof(float);
  EAR_CUDA(cudaFuncSetAttribute(at_simt<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem));
  const dim3 grid((unsigned)max_items, (unsigned)a.bh);
  at_simt<T, D><<<grid, kThreads, smem, s>>>(
      (const T*)a.Q, (const T*)a.K, (const T*)a.V, a.q_off, a.k_off, a.q_perm, a.k_perm, a.k_cent,
      a.v_cent, a.exact, a.blk_off, a.blk_list, items, count, max_items, a.n_q, a.n_k, a.c_q,
      a.c_k, a.scale, a.flags & EAR_COMPENSATE, (T*)a.O, a.lse, device_status_word());
  return after_launch();
}

// Workspace: the unit list, plus bf16 copies of the key / value centroids
// (rows padded to the tensor-core key chunk) for the tensor-core path.
struct AtWs {
  int2* items;
  int32_t* count;
  uint16_t* kc16;
  uint16_t* vc16;
};

AtWs carve(Carver& cv, int64_t bh, int64_t n_q, int32_t d, int32_t c_q, int32_t c_k) {
  AtWs w;
  w.items = cv.take<int2>((size_t)bh * attn_items_per_slice(n_q, c_q));
  w.count = cv.take<int32_t>((size_t)bh);
  const size_t cen = (size_t)bh * attention_tc_ck_pad(c_k) * d;
  w.kc16 = cv.take<uint16_t>(cen);
  w.vc16 = cv.take<uint16_t>(cen);
  return w;
}

}  // namespace

ear_status attention_plan(const int32_t* q_off, int64_t bh, int32_t c_q, int tile,
                          int64_t max_items, int2* items, int32_t* count, cudaStream_t s) {
  at_plan<<<(unsigned)bh, 1024, 0, s>>>(q_off, c_q, tile, max_items, items, count);
  return after_launch();
}

size_t attention_workspace(int64_t bh, int64_t n_q, int32_t d, int32_t c_q, int32_t c_k) {
  Carver cv(nullptr);
  carve(cv, bh, n_q, d, c_q, c_k);
  return cv.used;
}

ear_status attention_run(const AttnArgs& a, void* ws, cudaStream_t s) {
  Carver cv(ws);
  AtWs w = carve(cv, a.bh, a.n_q, a.d, a.c_q, a.c_k);
  if (a.dtype == EAR_BF16) {
    const int64_t max_items = attention_tc_items_per_slice(a.n_q, a.c_q);
    return attention_tc_run(a, w.items, w.count, max_items, w.kc16, w.vc16, s);
  }
  const int64_t max_items = attn_items_per_slice(a.n_q, a.c_q);
  EAR_TRY(attention_plan(a.q_off, a.bh, a.c_q, kTile, max_items, w.items, w.count, s));
  return a.d == 64 ? simt_t<float, 64>(a, w.items, w.count, max_items, s)
                   : simt_t<float, 128>(a, w.items, w.count, max_items, s);
}

}  // namespace ear
