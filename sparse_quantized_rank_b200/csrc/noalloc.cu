// compressed_linear_forward_noalloc: the forward pass for callers that cannot
// hand the library a workspace.
//
// Some callers cannot allocate device memory: an inference-server plugin whose
// enqueue path is not allowed to allocate, a runtime that accounts for every
// device byte up front, or a binding that can only pass raw input and output
// pointers.  This entry point takes no workspace.  Its scratch memory (the
// error word, the split-K accumulator, the row-block arrival counters and the
// adapter partial sums) lives in one file-scope device array of fixed size,
// which every GPU that loads the library holds until the process exits.
//
// Set-up: the first call on a device looks up the array's device address with
// cudaGetSymbolAddress (with that device current) and clears the array.
// Every call then shares the same array and clears, on its stream, the part
// it is about to use.
// Calls whose work overlaps on the GPU (different streams, or different host
// threads without ordering) race on the array and must be avoided.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr uint64_t kNoallocScratchBytes = 4ull << 20;   // 4 MiB per device

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[64] = {nullptr};

// Device address of the scratch array on the current device (set up on first
// use: address lookup and one clear).  nullptr on failure.
void* scratch_for_current_device(cql_status* st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *st = CQL_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      *st = CQL_ERR_CUDA;
      return nullptr;
    }
    if (cudaMemset(ptr, 0, kNoallocScratchBytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
      *st = CQL_ERR_CUDA;
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  }
  *st = CQL_OK;
  return g_scratch_ptr[dev];
}

}  // namespace

namespace cql {
// The scratch array's device address on the current device, or nullptr when
// no no-workspace call has run on it yet (cql_get_device_status reads its
// error word when passed no workspace).
void* noalloc_scratch_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  return g_scratch_ptr[dev];
}
}  // namespace cql

extern "C" {

cql_status compressed_linear_forward_noalloc(const cql_desc* desc, const void* packed, const void* x,
                                             cql_dtype x_dt, void* y, cql_dtype y_dt, int32_t batch,
                                             cql_stream_t stream) {
  uint64_t need = 0;
  cql_status st = cql_workspace_size(desc, batch, &need);
  if (st != CQL_OK) return st;
  if (need > kNoallocScratchBytes) return CQL_ERR_SIZE;   // layer or batch too large for the fixed scratch
  void* ws = scratch_for_current_device(&st);
  if (ws == nullptr) return st;
  // The array keeps the last call's contents, laid out for that call's layer
  // and batch; the forward expects its accumulators zero, so clear the part
  // this call uses (a memset, not an allocation).
  if (cudaMemsetAsync(ws, 0, need, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return CQL_ERR_CUDA;
  return compressed_linear_forward(desc, packed, x, x_dt, y, y_dt, batch, ws, kNoallocScratchBytes, stream);
}

}  // extern "C"
