// permute_static.cu -- moe_permute_align_static: the permutation with its
// scratch space inside the library instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at all: code embedded in a host
// framework that owns every device buffer through its own allocator and
// forbids hidden allocations, plugins and foreign-function callers that can
// hand over input and output tensors but have nowhere to keep a separate
// workspace alive between calls, and latency-bounded paths that may not call
// cudaMalloc.  For them this entry point takes only inputs and outputs; the
// scratch (status header, group table, per-chunk histograms) lives in a
// file-scope device array of kStaticScratchBytes that every GPU loading the
// library holds until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;  // 1 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_permute_scratch[kStaticScratchBytes];

// Device address of g_permute_scratch for each device, looked up once per
// device (with that device current) and cached for the life of the process.
// The cache does not survive a cudaDeviceReset (or any teardown of the
// device's primary context): after one, the cached address is stale, so a
// process that resets a device must not call this entry point on it again.
void* scratch_for_current_device(int* rc) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev)) || dev < 0 || dev >= kMaxDevices) {
    *rc = MOE_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (!cuda_ok(cudaGetSymbolAddress(&p, g_permute_scratch)) || p == nullptr) {
      *rc = MOE_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  *rc = MOE_OK;
  return addr[dev];
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_permute_align_static(const moe_dims* dims, const int32_t* topk_idx,
                                        const void* x, int32_t* counts, int32_t* offsets,
                                        int32_t* sorted_ids, int32_t* row_of, void* x_perm,
                                        void* stream) {
  // the same argument and shape checks as every other entry point
  const int shape_rc = check_shape(dims, false);
  if (shape_rc != MOE_OK) return shape_rc;
  // the scratch this call needs must fit the fixed array
  if (ws_layout(*dims).bytes > kStaticScratchBytes) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!counts || !offsets || !sorted_ids) return MOE_ERR_INVALID_ARG;
  if (dims->T > 0 && (!topk_idx || !row_of || (x_perm && !x))) return MOE_ERR_INVALID_ARG;
  int rc = MOE_OK;
  void* ws = scratch_for_current_device(&rc);
  if (rc != MOE_OK) return rc;
  // The array keeps whatever the previous call left: start every call from a
  // clean header (status word and routing flags).
  if (!cuda_ok(cudaMemsetAsync(ws, 0, kHeaderWords * sizeof(int32_t),
                               reinterpret_cast<cudaStream_t>(stream))))
    return MOE_ERR_CUDA;
  return launch_permute(*dims, topk_idx, x, counts, offsets, sorted_ids, row_of, x_perm, ws,
                        stream);
}
