// spark_bsa_forward_noalloc: the whole forward pass with its intermediates kept in a
// fixed-size array of device memory that belongs to this library, so that the call itself
// allocates nothing.
//
// Who needs it: code that must not allocate device memory while it runs - a caller whose
// memory budget is owned by a host framework or pool it cannot call into, a caller recording
// work into a CUDA stream capture (where cudaMalloc is not allowed), or an inference plugin
// invoked from a real-time path where an allocation could block or fail.  For them the
// caller-sized workspace of spark_bsa_forward is not an option, so this entry point uses a
// file-scope __device__ array instead.  The array is part of this file's module: it is reserved
// on every GPU where the module loads (first use under lazy loading, context creation under
// eager loading) and held until the process exits.
//
// The set-up (resolving the array's device address with cudaGetSymbolAddress) runs once per
// device, on the first call made while that device is current; the host-side name of the
// array is only a stand-in and must never be handed to a kernel.  The cached address does not
// survive a device reset (cudaDeviceReset tears the context down and the module reloads
// elsewhere); the header states that calls after one are not supported.
#include <mutex>

#include "../../include/spark_bsa.h"

namespace {

constexpr size_t kScratchBytes = SPARK_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// One static scratch area per device that loads this module; every call shares it.
static __device__ __align__(256) unsigned char g_spark_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on first use).
spark_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SPARK_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_spark_scratch) != cudaSuccess || p == nullptr)
      return SPARK_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SPARK_OK;
}

}  // namespace

extern "C" SPARK_API spark_status spark_bsa_forward_noalloc(
    const void* Q, const void* K, const void* V, int dtype, int H, int N, int d,
    const int32_t* q_perm, const int32_t* k_perm, const int32_t* q_block_offsets, int nqb,
    const int32_t* k_block_offsets, int nkb, double topk_ratio, void* out, void* stream) {
  if (!Q || !K || !V || !q_perm || !k_perm || !q_block_offsets || !k_block_offsets || !out)
    return SPARK_ERR_INVALID_ARG;
  spark_bsa_layout L;
  spark_status st = spark_bsa_workspace_layout(H, N, d, nqb, nkb, topk_ratio, &L);
  if (st != SPARK_OK) return st;
  if (L.total > kScratchBytes) return SPARK_ERR_WORKSPACE;   // problem too large for the array
  void* ws = nullptr;
  st = scratch_address(&ws);
  if (st != SPARK_OK) return st;
  // spark_bsa_forward clears the error word in the scratch before its first kernel.
  return spark_bsa_forward(Q, K, V, dtype, H, N, d, q_perm, k_perm, q_block_offsets, nqb,
                           k_block_offsets, nkb, topk_ratio, out, ws, L.total, stream);
}
