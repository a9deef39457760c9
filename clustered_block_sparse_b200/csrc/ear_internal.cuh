// Internal declarations shared by libear's CUDA translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ear.h"

namespace ear {

// ---------------------------------------------------------------- host side
// Device address of the per-device status word (resolved once per device).
int* device_status_word();
// Counts one kernel launch and checks the launch for a configuration error.
ear_status after_launch();

#define EAR_TRY(expr)                         \
  do {                                        \
    ear_status st_ = (expr);                  \
    if (st_ != EAR_OK) return st_;            \
  } while (0)

#define EAR_CUDA(expr)                        \
  do {                                        \
    if ((expr) != cudaSuccess) return EAR_ERR_CUDA; \
  } while (0)

// Carves 256-byte aligned sub-buffers out of a caller workspace; with a null
// base it only measures.
struct Carver {
  char* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    size_t off = (used + 255) & ~size_t(255);
    used = off + count * sizeof(T);
    return base ? reinterpret_cast<T*>(base + off) : nullptr;
  }
};

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Work-list geometry shared by the attention launchers.
constexpr int kAttnTileRows = 64;  // smallest query tile of any attention kernel
inline int64_t attn_items_per_slice(int64_t n_q, int32_t c_q) {
  return ceil_div(n_q, kAttnTileRows) + c_q;
}

// ---------------------------------------------------------------- launchers
// Each returns EAR_OK or EAR_ERR_CUDA; arguments were validated by the ABI.
size_t kmeans_workspace(int64_t bh, int64_t n, int32_t d, int32_t c);
ear_status kmeans_run(const void* X, ear_dtype dt, int64_t bh, int64_t n, int32_t d, int32_t c,
                      int32_t iters, const float* init, float* cent, int32_t* labels,
                      int32_t* counts, void* ws, cudaStream_t s);

bool kmeans_tc_supported(ear_dtype dt, int32_t d, int32_t c);
size_t kmeans_tc_workspace(int64_t bh, int64_t n, int32_t d, int32_t c);
ear_status kmeans_tc_run(const void* X, int64_t bh, int64_t n, int32_t d, int32_t c,
                         int32_t iters, const float* init, float* cent, int32_t* labels,
                         int32_t* counts, void* ws, cudaStream_t s);

size_t permute_workspace(int64_t bh, int64_t n, int32_t c);
ear_status permute_run(const int32_t* labels, int64_t bh, int64_t n, int32_t c, int32_t* perm,
                       int32_t* offsets, const void* X, void* X_perm, ear_dtype dt, int32_t d,
                       float* seg_mean, void* ws, cudaStream_t s);
// X_perm[r] = X[perm[r]] and the optional per-cluster means, from a given
// permutation and its offsets (no workspace).
ear_status permute_apply_run(const int32_t* perm, const int32_t* offsets, int64_t bh, int64_t n,
                             int32_t c, const void* X, void* X_perm, ear_dtype dt, int32_t d,
                             float* seg_mean, cudaStream_t s);

size_t probe_workspace(int64_t bh, int64_t n_k, int32_t d, int32_t c_q, int32_t c_k);
// Tensor-core probe (bf16 keys); mode as in ear_probe.  kperm != nullptr:
// K (and V) are in original order and permuted key j is row kperm[j].
size_t probe_tc_workspace(int64_t bh, int64_t n_k, int32_t d, int32_t c_q, int32_t c_k);
ear_status probe_tc_run(const float* qc, const int32_t* qn, const float* kc, const void* K,
                        const int32_t* kperm, const int32_t* koff, int64_t bh, int64_t n_k,
                        int32_t d, int32_t c_q, int32_t c_k, float scale, int32_t mode,
                        const void* V, const float* vc, float* E, void* ws, cudaStream_t s);
ear_status probe_run(const float* qc, const int32_t* qn, const float* kc, const void* K,
                     const int32_t* kperm, ear_dtype dt, const int32_t* koff, int64_t bh,
                     int64_t n_k, int32_t d, int32_t c_q, int32_t c_k, float scale, int32_t mode,
                     const void* V, const float* vc, float* E, void* ws, cudaStream_t s);

size_t route_workspace(int64_t bh, int32_t c_q, int32_t c_k);
ear_status route_run(const float* E, const int32_t* qn, const int32_t* kn, int64_t bh,
                     int64_t budget, int32_t c_q, int32_t c_k, int32_t mode, uint8_t* exact,
                     int32_t* blk_off, int32_t* blk_list, int64_t* pairs, void* ws,
                     cudaStream_t s);

// Per-query-cluster routing and budgets (route_rows.cu); C_k <= kRowsMaxCk.
constexpr int32_t kRowsMaxCk = 8192;
size_t route_rows_workspace(int64_t bh, int32_t c_q);
ear_status route_rows_run(const float* E, const int32_t* qn, const int32_t* kn, int64_t bh,
                          int32_t c_q, int32_t c_k, const int64_t* row_budget, uint8_t* exact,
                          int32_t* blk_off, int32_t* blk_list, int64_t* pairs, void* ws,
                          cudaStream_t s);
ear_status topp_budget_run(const float* qc, const int32_t* qn, const float* kc, const int32_t* kn,
                           int64_t bh, int32_t d, int32_t c_q, int32_t c_k, float scale, double p,
                           int64_t* budget, cudaStream_t s);
ear_status uniform_budget_run(const int32_t* qn, int64_t bh, int32_t c_q, int64_t n_k,
                              double density, int64_t* budget, cudaStream_t s);

// Diagnostics (diag.cu).
ear_status cluster_stats_run(const void* X, ear_dtype dt, const int32_t* labels,
                             const float* cent, int64_t bh, int64_t n, int32_t d, int32_t c,
                             double* mean_sq, double* max_norm, cudaStream_t s);
ear_status normalizer_change_run(const float* lse_sparse, const float* lse_dense, int64_t bh,
                                 int64_t n, double* out, cudaStream_t s);

struct AttnArgs {
  const void* Q;
  const void* K;
  const void* V;
  ear_dtype dtype;
  const int32_t* q_off;
  const int32_t* k_off;
  const int32_t* q_perm;
  const float* k_cent;
  const float* v_cent;
  const uint8_t* exact;
  const int32_t* blk_off;
  const int32_t* blk_list;
  int64_t bh, n_q, n_k;
  int32_t d, c_q, c_k;
  float scale;
  int32_t flags;
  void* O;
  float* lse;
  // Gather: Q, K, V are in original token order and K / V rows are read as
  // k_perm[r] (Q rows as q_perm[r]); nullptr = cluster-contiguous inputs.
  const int32_t* k_perm = nullptr;
};
size_t attention_workspace(int64_t bh, int64_t n_q, int32_t d, int32_t c_q, int32_t c_k);
ear_status attention_run(const AttnArgs& a, void* ws, cudaStream_t s);
// Query units of `tile` rows that never straddle two query clusters.
ear_status attention_plan(const int32_t* q_off, int64_t bh, int32_t c_q, int tile,
                          int64_t max_items, int2* items, int32_t* count, cudaStream_t s);
// Tensor-core path (bf16): centroid rows padded to a multiple of the key chunk.
int64_t attention_tc_ck_pad(int32_t c_k);
int64_t attention_tc_items_per_slice(int64_t n_q, int32_t c_q);
ear_status attention_tc_run(const AttnArgs& a, int2* items, int32_t* count, int64_t max_items,
                            uint16_t* kc16, uint16_t* vc16, cudaStream_t s);

}  // namespace ear

// ---------------------------------------------------------------- device side
#ifdef __CUDACC__
namespace ear {

__device__ __forceinline__ void latch(int* status, int code) { atomicCAS(status, 0, code); }

// Gathered loads: the TMA row coordinate of original row perm[i] of slice h
// (n rows per slice), or of the slice's row 0 with EAR_ERR_DEVICE latched when
// the entry is out of range.
__device__ __forceinline__ int32_t gather_row(const int32_t* perm, int64_t i, int64_t h,
                                              int64_t n, int* status) {
  int32_t o = perm[i];
  if (o < 0 || o >= n) {
    latch(status, EAR_ERR_DEVICE);
    o = 0;
  }
  return (int32_t)(h * n) + o;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t u) {
  return __uint_as_float(static_cast<uint32_t>(u) << 16);
}

// Round-to-nearest-even fp32 -> bf16 bits (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  __device__ __forceinline__ static float load(const float* p, int64_t i) { return p[i]; }
  __device__ __forceinline__ static void store(float* p, int64_t i, float v) { p[i] = v; }
};
template <>
struct Elem<uint16_t> {
  __device__ __forceinline__ static float load(const uint16_t* p, int64_t i) {
    return bf16_to_f32(p[i]);
  }
  __device__ __forceinline__ static void store(uint16_t* p, int64_t i, float v) {
    p[i] = f32_to_bf16(v);
  }
};

}  // namespace ear
#endif
