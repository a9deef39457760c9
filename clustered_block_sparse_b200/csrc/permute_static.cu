// ear_permute_static: the cluster-contiguous permutation without a caller
// workspace.  Some callers cannot allocate device memory at all: a plugin
// whose host application owns every device buffer and hands the plugin only
// its inputs and outputs, or an embedded runtime with a fixed memory plan and
// no allocator.  For them the permutation's scratch (per-tile cluster counts)
// lives in one fixed-size array compiled into this library.
//
// The array is a file-scope __device__ variable, so host code cannot use its
// name as a device pointer.  Its device address on the current device is
// looked up with cudaGetSymbolAddress on every call (the first call on a
// device loads the module there, so make it before any stream capture) and
// handed to the kernels as their workspace.  It is not cached: after a device
// reset the module is loaded again at a new address.
#include "ear_internal.cuh"

namespace {

constexpr size_t kScratchBytes = EAR_PERMUTE_STATIC_MAX_BYTES;

// Kept by every device that loads the library until the process exits.
static __device__ __align__(256) unsigned char g_permute_scratch[kScratchBytes];

// Device address of g_permute_scratch on the current device.
ear_status scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr)
    return EAR_ERR_CUDA;
  *out = p;
  return EAR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

ear_status ear_permute_static(const int32_t* labels, int64_t bh, int64_t n, int32_t c,
                              int32_t* perm, int32_t* offsets, const void* X, void* X_perm,
                              ear_dtype dtype, int32_t d, float* seg_mean, void* stream) {
  // Same argument rules as ear_permute, checked before anything touches the GPU.
  if (bh < 1 || n < 1 || n > (int64_t(1) << 31) - 1 || c < 1) return EAR_ERR_ARG;
  if (labels == nullptr || perm == nullptr || offsets == nullptr || !aligned16(labels) ||
      !aligned16(perm) || !aligned16(offsets))
    return EAR_ERR_ARG;
  if (c > 65536 || bh > 65535) return EAR_ERR_UNSUPPORTED;
  if (X == nullptr && (X_perm != nullptr || seg_mean != nullptr)) return EAR_ERR_ARG;
  if (X != nullptr && (X_perm == nullptr || !aligned16(X) || !aligned16(X_perm) ||
                       (dtype != EAR_F32 && dtype != EAR_BF16) ||
                       (seg_mean != nullptr && !aligned16(seg_mean))))
    return EAR_ERR_ARG;
  if (X != nullptr && d != 64 && d != 128) return EAR_ERR_UNSUPPORTED;
  // The problem must fit the fixed scratch array.
  if (ear::permute_workspace(bh, n, c) > kScratchBytes) return EAR_ERR_WORKSPACE;
  void* scratch = nullptr;
  EAR_TRY(scratch_address(&scratch));
  return ear_permute(labels, bh, n, c, perm, offsets, X, X_perm, dtype, d, seg_mean, scratch,
                     kScratchBytes, stream);
}

}  // extern "C"
