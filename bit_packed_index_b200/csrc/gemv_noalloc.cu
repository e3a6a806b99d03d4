// gemv_noalloc.cu -- vq_gemv_noalloc: the decode GEMV without a caller-provided
// workspace.
//
// Who needs this: code that cannot allocate device memory at the point where
// it runs the layer -- for example a serving loop inside a pre-reserved
// memory pool, a plug-in called from another framework's allocator-controlled
// context, or a caller with no CUDA allocation API at hand.  vq_gemv may need
// scratch for its split-K partial sums (vq_gemv_workspace_size() > 0 for
// narrow layers and larger batches); this entry point takes that scratch from
// a fixed array compiled into the library instead.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds kScratchBytes of it until the process exits, and every call
// on a device shares it.  Host code cannot use the variable's name as a device
// address: the library looks the address up with cudaGetSymbolAddress on the
// first call made on each device (with that device current) and caches it.
// Plans that can shrink their scratch (the tiled lookup-table kernel runs on
// fewer blocks) are sized to the array.  The split-K kernels write every
// partial sum before the finalize pass reads it, so nothing in the array has to start at zero and leftover contents from
// an earlier call are harmless.  Two calls whose kernels overlap on the GPU
// (different streams, same device) race on the array.
#include <mutex>
#include <vector>

#include "vq_internal.cuh"

namespace vqk {
namespace {

constexpr size_t kScratchBytes = VQ_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_gemv_scratch[kScratchBytes];

// Device address of g_gemv_scratch on the current device, looked up once per
// device.  Returns nullptr (and records the CUDA error) if the lookup fails.
void* scratch_for_current_device(cudaError_t* err) {
  static std::mutex mu;
  static std::vector<void*> addr;
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(addr.size()) <= dev) addr.resize(dev + 1, nullptr);
  if (!addr[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_gemv_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace vqk

using namespace vqk;

extern "C" vq_status vq_gemv_noalloc(const vq_layer_desc* layer, const void* x, vq_dtype x_dtype,
                                     int32_t batch, int64_t ldx, void* y, vq_dtype y_dtype,
                                     int64_t ldy, void* stream) {
  // The scratch array and the plan belong to the current device: a stream of
  // another device is rejected.
  if (stream) {
    int cur = 0, sdev = 0;
    if (cudaGetDevice(&cur) == cudaSuccess &&
        cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &sdev) == cudaSuccess && sdev != cur)
      return VQ_ERR_INVALID_ARG;
  }
  size_t need = 0;
  vq_status st = gemv_workspace_bytes(layer, batch, kScratchBytes, &need);
  if (st != VQ_OK) return st;
  if (need > kScratchBytes) return VQ_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    cudaError_t e = cudaSuccess;
    ws = scratch_for_current_device(&e);
    if (!ws) return cuda_status(e);
  }
  return gemv_run(layer, x, x_dtype, batch, ldx, y, y_dtype, ldy, ws, need, kScratchBytes,
                  static_cast<cudaStream_t>(stream));
}
