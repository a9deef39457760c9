// libear C ABI: host-side validation, workspace sizing, status word and
// dispatch to the kernel launchers.  Every check here runs before anything
// is enqueued, so a rejected call has no side effect.
#include <atomic>
#include <cmath>

#include "ear_internal.cuh"

namespace {

__device__ int g_status_word;  // first device-side error latched since the last read

std::atomic<uint64_t> g_launches{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_dtype(ear_dtype t) { return t == EAR_F32 || t == EAR_BF16; }
bool ok_d(int32_t d) { return d == 64 || d == 128; }
constexpr int64_t kMaxN = (int64_t(1) << 31) - 1;
constexpr int32_t kMaxC = 65536;
constexpr int64_t kMaxBH = 65535;  // slices map to grid.y

ear_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws_bytes < need) return EAR_ERR_WORKSPACE;
  if (need > 0 && (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0))
    return EAR_ERR_ARG;
  return EAR_OK;
}

}  // namespace

namespace ear {

// Looked up on every call rather than cached: after a device reset the module
// is loaded again at a new address in the new context, and a cached pointer
// would be stale.  The lookup is a host-side table read once the module is
// loaded (the first call on a device loads it; make that call before any
// stream capture begins).
int* device_status_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

ear_status after_launch() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? EAR_OK : EAR_ERR_CUDA;
}

}  // namespace ear

extern "C" {

const char* ear_status_string(ear_status s) {
  switch (s) {
    case EAR_OK: return "EAR_OK";
    case EAR_ERR_ARG: return "EAR_ERR_ARG: invalid argument";
    case EAR_ERR_UNSUPPORTED: return "EAR_ERR_UNSUPPORTED: configuration not built";
    case EAR_ERR_WORKSPACE: return "EAR_ERR_WORKSPACE: workspace too small";
    case EAR_ERR_CUDA: return "EAR_ERR_CUDA: CUDA runtime error";
    case EAR_ERR_TIMEOUT: return "EAR_ERR_TIMEOUT: device-side wait ran out";
    case EAR_ERR_DEVICE: return "EAR_ERR_DEVICE: device-side index check failed";
  }
  return "unknown ear_status";
}

uint64_t ear_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

ear_status ear_workspace_bytes(ear_op op, int64_t bh, int64_t n_q, int64_t n_k, int32_t d,
                               int32_t c_q, int32_t c_k, size_t* bytes) {
  if (bytes == nullptr || bh < 0 || n_q < 0 || n_k < 0 || d < 0 || c_q < 0 || c_k < 0)
    return EAR_ERR_ARG;
  switch (op) {
    case EAR_OP_KMEANS: *bytes = ear::kmeans_workspace(bh, n_q, d, c_q); return EAR_OK;
    case EAR_OP_PERMUTE: *bytes = ear::permute_workspace(bh, n_q, c_q); return EAR_OK;
    case EAR_OP_PROBE: *bytes = ear::probe_workspace(bh, n_k, d, c_q, c_k); return EAR_OK;
    case EAR_OP_ROUTE: *bytes = ear::route_workspace(bh, c_q, c_k); return EAR_OK;
    case EAR_OP_ATTENTION: *bytes = ear::attention_workspace(bh, n_q, d, c_q, c_k); return EAR_OK;
    case EAR_OP_ROUTE_ROWS: *bytes = ear::route_rows_workspace(bh, c_q); return EAR_OK;
  }
  return EAR_ERR_ARG;
}

ear_status ear_kmeans(const void* X, ear_dtype dtype, int64_t bh, int64_t n, int32_t d,
                      int32_t c, int32_t iters, const float* init, float* centroids,
                      int32_t* labels, int32_t* counts, void* ws, size_t ws_bytes,
                      void* stream) {
  if (!ok_dtype(dtype) || bh < 1 || n < 1 || n > kMaxN || c < 1 || c > n || iters < 1)
    return EAR_ERR_ARG;
  if (!ok_ptr(X) || !ok_ptr(init) || !ok_ptr(centroids) || !ok_ptr(labels) || !ok_ptr(counts))
    return EAR_ERR_ARG;
  if (!ok_d(d) || c > kMaxC || bh > kMaxBH) return EAR_ERR_UNSUPPORTED;
  EAR_TRY(check_ws(ws, ws_bytes, ear::kmeans_workspace(bh, n, d, c)));
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  return ear::kmeans_run(X, dtype, bh, n, d, c, iters, init, centroids, labels, counts, ws,
                         static_cast<cudaStream_t>(stream));
}

ear_status ear_permute(const int32_t* labels, int64_t bh, int64_t n, int32_t c,
                       int32_t* perm, int32_t* offsets, const void* X, void* X_perm,
                       ear_dtype dtype, int32_t d, float* seg_mean, void* ws, size_t ws_bytes,
                       void* stream) {
  if (bh < 1 || n < 1 || n > kMaxN || c < 1) return EAR_ERR_ARG;
  if (!ok_ptr(labels) || !ok_ptr(perm) || !ok_ptr(offsets)) return EAR_ERR_ARG;
  if (c > kMaxC || bh > kMaxBH) return EAR_ERR_UNSUPPORTED;
  if (X != nullptr) {
    if (!ok_ptr(X) || !ok_ptr(X_perm) || !ok_dtype(dtype)) return EAR_ERR_ARG;
    if (seg_mean != nullptr && !aligned16(seg_mean)) return EAR_ERR_ARG;
    if (!ok_d(d)) return EAR_ERR_UNSUPPORTED;
  } else if (X_perm != nullptr || seg_mean != nullptr) {
    return EAR_ERR_ARG;
  }
  EAR_TRY(check_ws(ws, ws_bytes, ear::permute_workspace(bh, n, c)));
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  return ear::permute_run(labels, bh, n, c, perm, offsets, X, X_perm, dtype, d, seg_mean, ws,
                          static_cast<cudaStream_t>(stream));
}

ear_status ear_permute_apply(const int32_t* perm, const int32_t* offsets, int64_t bh, int64_t n,
                             int32_t c, const void* X, void* X_perm, ear_dtype dtype, int32_t d,
                             float* seg_mean, void* stream) {
  if (bh < 1 || n < 1 || n > kMaxN || c < 1) return EAR_ERR_ARG;
  if (!ok_ptr(perm) || !ok_ptr(offsets) || !ok_ptr(X) || !ok_dtype(dtype)) return EAR_ERR_ARG;
  // X_perm may be NULL only when the means are asked for (means only)
  if (X_perm == nullptr ? seg_mean == nullptr : !ok_ptr(X_perm)) return EAR_ERR_ARG;
  if (seg_mean != nullptr && !aligned16(seg_mean)) return EAR_ERR_ARG;
  if (c > kMaxC || bh > kMaxBH || !ok_d(d)) return EAR_ERR_UNSUPPORTED;
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  return ear::permute_apply_run(perm, offsets, bh, n, c, X, X_perm, dtype, d, seg_mean,
                                static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// ear_probe and ear_probe_gather: k_perm == nullptr means K / V are permuted.
ear_status probe_entry(const float* q_centroids, const int32_t* q_counts,
                       const float* k_centroids, const void* K_perm, const int32_t* k_perm,
                       ear_dtype dtype, const int32_t* k_offsets, int64_t bh, int64_t n_k,
                       int32_t d, int32_t c_q, int32_t c_k, float scale, int32_t mode,
                       const void* V_perm, const float* v_centroids, float* E, void* ws,
                       size_t ws_bytes, void* stream) {
  if (!ok_dtype(dtype) || bh < 1 || n_k < 1 || n_k > kMaxN || c_q < 1 || c_k < 1 ||
      !std::isfinite(scale) || mode < EAR_PROBE_LOGIT || mode > EAR_PROBE_VALUE)
    return EAR_ERR_ARG;
  if (!ok_ptr(q_centroids) || !ok_ptr(q_counts) || !ok_ptr(k_centroids) || !ok_ptr(K_perm) ||
      !ok_ptr(k_offsets) || !ok_ptr(E))
    return EAR_ERR_ARG;
  if (mode == EAR_PROBE_VALUE && (!ok_ptr(V_perm) || !ok_ptr(v_centroids))) return EAR_ERR_ARG;
  if (!ok_d(d) || c_q > kMaxC || c_k > kMaxC || bh > kMaxBH) return EAR_ERR_UNSUPPORTED;
  if (mode != EAR_PROBE_LOGIT && dtype != EAR_BF16) return EAR_ERR_UNSUPPORTED;
  EAR_TRY(check_ws(ws, ws_bytes, ear::probe_workspace(bh, n_k, d, c_q, c_k)));
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  return ear::probe_run(q_centroids, q_counts, k_centroids, K_perm, k_perm, dtype, k_offsets, bh,
                        n_k, d, c_q, c_k, scale, mode, V_perm, v_centroids, E, ws,
                        static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

ear_status ear_probe(const float* q_centroids, const int32_t* q_counts,
                     const float* k_centroids, const void* K_perm, ear_dtype dtype,
                     const int32_t* k_offsets, int64_t bh, int64_t n_k, int32_t d,
                     int32_t c_q, int32_t c_k, float scale, int32_t mode, const void* V_perm,
                     const float* v_centroids, float* E, void* ws, size_t ws_bytes,
                     void* stream) {
  return probe_entry(q_centroids, q_counts, k_centroids, K_perm, nullptr, dtype, k_offsets, bh,
                     n_k, d, c_q, c_k, scale, mode, V_perm, v_centroids, E, ws, ws_bytes, stream);
}

ear_status ear_probe_gather(const float* q_centroids, const int32_t* q_counts,
                            const float* k_centroids, const void* K, const int32_t* k_perm,
                            ear_dtype dtype, const int32_t* k_offsets, int64_t bh, int64_t n_k,
                            int32_t d, int32_t c_q, int32_t c_k, float scale, int32_t mode,
                            const void* V, const float* v_centroids, float* E, void* ws,
                            size_t ws_bytes, void* stream) {
  if (!ok_ptr(k_perm)) return EAR_ERR_ARG;
  return probe_entry(q_centroids, q_counts, k_centroids, K, k_perm, dtype, k_offsets, bh, n_k, d,
                     c_q, c_k, scale, mode, V, v_centroids, E, ws, ws_bytes, stream);
}

ear_status ear_route(const float* E, const int32_t* q_counts, const int32_t* k_counts,
                     int64_t bh, int64_t n_q, int64_t n_k, int32_t c_q, int32_t c_k,
                     double density, int32_t ratio_mode, uint8_t* exact,
                     int32_t* blk_offsets, int32_t* blk_list, int64_t* exact_pairs,
                     void* ws, size_t ws_bytes, void* stream) {
  if (bh < 1 || n_q < 1 || n_k < 1 || n_q > kMaxN || n_k > kMaxN || c_q < 1 || c_k < 1)
    return EAR_ERR_ARG;
  if (!(density >= 0.0 && density <= 1.0) || (ratio_mode != 0 && ratio_mode != 1))
    return EAR_ERR_ARG;
  if (!ok_ptr(E) || !ok_ptr(q_counts) || !ok_ptr(k_counts) || !ok_ptr(exact) ||
      !ok_ptr(blk_offsets) || !ok_ptr(blk_list) || !ok_ptr(exact_pairs))
    return EAR_ERR_ARG;
  if (c_q > kMaxC || c_k > kMaxC || (int64_t)c_q * c_k > kMaxN || bh > kMaxBH)
    return EAR_ERR_UNSUPPORTED;
  EAR_TRY(check_ws(ws, ws_bytes, ear::route_workspace(bh, c_q, c_k)));
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  // budget B = floor(rho * (N_q * N_k)): the pair count is exact in int64 and
  // in double (< 2^53), one rounded product, then floor.
  const int64_t pairs_total = n_q * n_k;
  const int64_t budget = static_cast<int64_t>(std::floor(density * static_cast<double>(pairs_total)));
  return ear::route_run(E, q_counts, k_counts, bh, budget, c_q, c_k, ratio_mode, exact,
                        blk_offsets, blk_list, exact_pairs, ws,
                        static_cast<cudaStream_t>(stream));
}

ear_status ear_route_rows(const float* E, const int32_t* q_counts, const int32_t* k_counts,
                          int64_t bh, int32_t c_q, int32_t c_k, const int64_t* row_budget,
                          uint8_t* exact, int32_t* blk_offsets, int32_t* blk_list,
                          int64_t* exact_pairs, void* ws, size_t ws_bytes, void* stream) {
  if (bh < 1 || c_q < 1 || c_k < 1) return EAR_ERR_ARG;
  if (!ok_ptr(E) || !ok_ptr(q_counts) || !ok_ptr(k_counts) || !ok_ptr(row_budget) ||
      !ok_ptr(exact) || !ok_ptr(blk_offsets) || !ok_ptr(blk_list) || !ok_ptr(exact_pairs))
    return EAR_ERR_ARG;
  if (c_q > kMaxC || c_k > ear::kRowsMaxCk || (int64_t)c_q * c_k > kMaxN || bh > kMaxBH)
    return EAR_ERR_UNSUPPORTED;
  EAR_TRY(check_ws(ws, ws_bytes, ear::route_rows_workspace(bh, c_q)));
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  return ear::route_rows_run(E, q_counts, k_counts, bh, c_q, c_k, row_budget, exact, blk_offsets,
                             blk_list, exact_pairs, ws, static_cast<cudaStream_t>(stream));
}

ear_status ear_topp_budget(const float* q_centroids, const int32_t* q_counts,
                           const float* k_centroids, const int32_t* k_counts, int64_t bh,
                           int32_t d, int32_t c_q, int32_t c_k, float scale, double p,
                           int64_t* row_budget, void* stream) {
  if (bh < 1 || c_q < 1 || c_k < 1 || !std::isfinite(scale) || !(p >= 0.0 && p <= 1.0))
    return EAR_ERR_ARG;
  if (!ok_ptr(q_centroids) || !ok_ptr(q_counts) || !ok_ptr(k_centroids) || !ok_ptr(k_counts) ||
      !ok_ptr(row_budget))
    return EAR_ERR_ARG;
  if (!ok_d(d) || c_q > kMaxC || c_k > ear::kRowsMaxCk || bh > kMaxBH) return EAR_ERR_UNSUPPORTED;
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  return ear::topp_budget_run(q_centroids, q_counts, k_centroids, k_counts, bh, d, c_q, c_k, scale,
                              p, row_budget, static_cast<cudaStream_t>(stream));
}

ear_status ear_uniform_budget(const int32_t* q_counts, int64_t bh, int32_t c_q, int64_t n_k,
                              double density, int64_t* row_budget, void* stream) {
  if (bh < 1 || c_q < 1 || n_k < 1 || n_k > kMaxN || !(density >= 0.0 && density <= 1.0))
    return EAR_ERR_ARG;
  if (!ok_ptr(q_counts) || !ok_ptr(row_budget)) return EAR_ERR_ARG;
  if (c_q > kMaxC || bh > kMaxBH) return EAR_ERR_UNSUPPORTED;
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  return ear::uniform_budget_run(q_counts, bh, c_q, n_k, density, row_budget,
                                 static_cast<cudaStream_t>(stream));
}

ear_status ear_cluster_stats(const void* X, ear_dtype dtype, const int32_t* labels,
                             const float* centroids, int64_t bh, int64_t n, int32_t d, int32_t c,
                             double* mean_sq_dist, double* max_norm, void* stream) {
  if (!ok_dtype(dtype) || bh < 1 || n < 1 || n > kMaxN || c < 1) return EAR_ERR_ARG;
  if (!ok_ptr(X) || !ok_ptr(labels) || !ok_ptr(centroids) || !ok_ptr(mean_sq_dist) ||
      !ok_ptr(max_norm))
    return EAR_ERR_ARG;
  if (!ok_d(d) || c > kMaxC || bh > kMaxBH) return EAR_ERR_UNSUPPORTED;
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  return ear::cluster_stats_run(X, dtype, labels, centroids, bh, n, d, c, mean_sq_dist, max_norm,
                                static_cast<cudaStream_t>(stream));
}

ear_status ear_normalizer_change(const float* lse_sparse, const float* lse_dense, int64_t bh,
                                 int64_t n, double* change, void* stream) {
  if (bh < 1 || n < 1 || n > kMaxN) return EAR_ERR_ARG;
  if (!ok_ptr(lse_sparse) || !ok_ptr(lse_dense) || !ok_ptr(change)) return EAR_ERR_ARG;
  if (bh > kMaxBH) return EAR_ERR_UNSUPPORTED;
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  return ear::normalizer_change_run(lse_sparse, lse_dense, bh, n, change,
                                    static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// ear_attention and ear_attention_gather: k_perm == nullptr means Q / K / V are permuted.
ear_status attention_entry(const void* Q_perm, const void* K_perm, const void* V_perm,
                           ear_dtype dtype, const int32_t* q_offsets, const int32_t* k_offsets,
                           const int32_t* q_perm, const int32_t* k_perm,
                           const float* k_centroids, const float* v_centroids,
                           const uint8_t* exact, const int32_t* blk_offsets,
                           const int32_t* blk_list, int64_t bh, int64_t n_q, int64_t n_k,
                           int32_t d, int32_t c_q, int32_t c_k, float scale, int32_t flags,
                           void* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!ok_dtype(dtype) || bh < 1 || n_q < 1 || n_k < 1 || n_q > kMaxN || n_k > kMaxN ||
      c_q < 1 || c_k < 1 || !std::isfinite(scale) || (flags & ~EAR_COMPENSATE) != 0)
    return EAR_ERR_ARG;
  if (!ok_ptr(Q_perm) || !ok_ptr(K_perm) || !ok_ptr(V_perm) || !ok_ptr(q_offsets) ||
      !ok_ptr(k_offsets) || !ok_ptr(q_perm) || !ok_ptr(k_centroids) || !ok_ptr(v_centroids) ||
      !ok_ptr(exact) || !ok_ptr(blk_offsets) || !ok_ptr(blk_list) || !ok_ptr(O))
    return EAR_ERR_ARG;
  if (lse != nullptr && !aligned16(lse)) return EAR_ERR_ARG;
  if (!ok_d(d) || c_q > kMaxC || c_k > kMaxC || bh > kMaxBH) return EAR_ERR_UNSUPPORTED;
  EAR_TRY(check_ws(ws, ws_bytes, ear::attention_workspace(bh, n_q, d, c_q, c_k)));
  if (ear::device_status_word() == nullptr) return EAR_ERR_CUDA;
  ear::AttnArgs a{Q_perm, K_perm, V_perm, dtype, q_offsets, k_offsets, q_perm, k_centroids,
                  v_centroids, exact, blk_offsets, blk_list, bh, n_q, n_k, d, c_q, c_k, scale,
                  flags, O, lse};
  a.k_perm = k_perm;
  return ear::attention_run(a, ws, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

ear_status ear_attention(const void* Q_perm, const void* K_perm, const void* V_perm,
                         ear_dtype dtype, const int32_t* q_offsets, const int32_t* k_offsets,
                         const int32_t* q_perm, const float* k_centroids,
                         const float* v_centroids, const uint8_t* exact,
                         const int32_t* blk_offsets, const int32_t* blk_list, int64_t bh,
                         int64_t n_q, int64_t n_k, int32_t d, int32_t c_q, int32_t c_k,
                         float scale, int32_t flags, void* O, float* lse, void* ws,
                         size_t ws_bytes, void* stream) {
  return attention_entry(Q_perm, K_perm, V_perm, dtype, q_offsets, k_offsets, q_perm, nullptr,
                         k_centroids, v_centroids, exact, blk_offsets, blk_list, bh, n_q, n_k, d,
                         c_q, c_k, scale, flags, O, lse, ws, ws_bytes, stream);
}

ear_status ear_attention_gather(const void* Q, const void* K, const void* V, ear_dtype dtype,
                                const int32_t* q_offsets, const int32_t* k_offsets,
                                const int32_t* q_perm, const int32_t* k_perm,
                                const float* k_centroids, const float* v_centroids,
                                const uint8_t* exact, const int32_t* blk_offsets,
                                const int32_t* blk_list, int64_t bh, int64_t n_q, int64_t n_k,
                                int32_t d, int32_t c_q, int32_t c_k, float scale, int32_t flags,
                                void* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!ok_ptr(k_perm)) return EAR_ERR_ARG;
  return attention_entry(Q, K, V, dtype, q_offsets, k_offsets, q_perm, k_perm, k_centroids,
                         v_centroids, exact, blk_offsets, blk_list, bh, n_q, n_k, d, c_q, c_k,
                         scale, flags, O, lse, ws, ws_bytes, stream);
}

ear_status ear_get_device_status(int32_t* out, void* stream) {
  if (out == nullptr) return EAR_ERR_ARG;
  int* word = ear::device_status_word();
  if (word == nullptr) return EAR_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host = 0;
  EAR_CUDA(cudaMemcpyAsync(&host, word, sizeof(int), cudaMemcpyDeviceToHost, s));
  EAR_CUDA(cudaMemsetAsync(word, 0, sizeof(int), s));
  EAR_CUDA(cudaStreamSynchronize(s));
  *out = host;
  return EAR_OK;
}

}  // extern "C"
