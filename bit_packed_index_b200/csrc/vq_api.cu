// vq_api.cu -- the extern "C" entry points of libvq (declared in include/vq.h):
// argument validation on the host, then one launcher per call.  Nothing is
// launched when an argument is rejected.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "vq_internal.cuh"

static_assert(sizeof(vq_layer_desc) == 104, "vq_layer_desc layout is part of the ABI");

namespace vqk {
namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<uint64_t> g_launches{0};

struct DeviceAttrs {
  int sms = 0;
  int smem_optin = 0;
};

DeviceAttrs& attrs_for_current_device() {
  static std::mutex mu;
  static std::vector<DeviceAttrs> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1);
  DeviceAttrs& a = cache[dev];
  if (a.sms == 0) {
    cudaDeviceGetAttribute(&a.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&a.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (a.sms <= 0) a.sms = 148;
    if (a.smem_optin <= 0) a.smem_optin = 227 * 1024;
  }
  return a;
}

bool dtype_ok_in(vq_dtype t) { return t == VQ_BF16 || t == VQ_FP16; }
bool dtype_ok_out(vq_dtype t) { return t == VQ_BF16 || t == VQ_FP16 || t == VQ_FP32; }
size_t dtype_size(vq_dtype t) { return t == VQ_FP32 ? 4 : 2; }

}  // namespace

vq_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return VQ_OK;
  g_last_cuda_error = static_cast<int>(e);
  return VQ_ERR_CUDA;
}

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

int device_sm_count() { return attrs_for_current_device().sms; }

cudaError_t set_func_attr(const void* func, cudaFuncAttribute attr, int value) {
  struct Entry {
    int dev;
    const void* func;
    cudaFuncAttribute attr;
    int value;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : done)
      if (e.dev == dev && e.func == func && e.attr == attr &&
          (e.value == value || (attr == cudaFuncAttributeMaxDynamicSharedMemorySize && e.value >= value)))
        return cudaSuccess;
  }
  const cudaError_t err = cudaFuncSetAttribute(func, attr, value);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(mu);
  for (Entry& e : done)
    if (e.dev == dev && e.func == func && e.attr == attr) {
      if (attr != cudaFuncAttributeMaxDynamicSharedMemorySize || value > e.value) e.value = value;
      return cudaSuccess;
    }
  done.push_back({dev, func, attr, value});
  return cudaSuccess;
}
int device_smem_optin() { return attrs_for_current_device().smem_optin; }

int resident_blocks_per_sm(const void* func, int threads, size_t smem) {
  struct Entry {
    int dev;
    const void* func;
    int threads;
    size_t smem;
    int blocks;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : done)
      if (e.dev == dev && e.func == func && e.threads == threads && e.smem == smem) return e.blocks;
  }
  int blocks = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, func, threads, smem) != cudaSuccess) {
    cudaGetLastError();   // leave no sticky error for the launch to report
    blocks = 1;
  }
  blocks = std::max(1, blocks);
  std::lock_guard<std::mutex> lock(mu);
  done.push_back({dev, func, threads, smem, blocks});
  return blocks;
}

vq_status check_layer(const vq_layer_desc* desc, Layer* out) {
  if (!desc || !out) return VQ_ERR_INVALID_ARG;
  const vq_layer_desc& D = *desc;
  if (D.out_features < 0 || D.in_features < 0) return VQ_ERR_INVALID_ARG;
  if (D.vec_dim < 1 || D.vec_dim > kMaxVecDim) return VQ_ERR_INVALID_ARG;
  if (D.n_books < 1 || D.n_books > 2) return VQ_ERR_INVALID_ARG;
  if ((D.idx_layout != VQ_IDX_ROWS && D.idx_layout != VQ_IDX_TILE4) || D.reserved != 0)
    return VQ_ERR_INVALID_ARG;
  Layer L{};
  L.layout = D.idx_layout;
  L.n = D.out_features;
  L.kin = D.in_features;
  L.d = D.vec_dim;
  L.nb = D.n_books;
  L.nvec = static_cast<int>((static_cast<int64_t>(D.in_features) + D.vec_dim - 1) / D.vec_dim);
  for (int m = 0; m < L.nb; ++m) {
    const int b = D.log2k[m];
    if (b < 1 || b > 16) return VQ_ERR_INVALID_ARG;
    const int64_t need = L.layout == VQ_IDX_ROWS
                             ? (static_cast<int64_t>(L.nvec) * b + 127) / 128 * 4
                             : (static_cast<int64_t>(L.n) * 4 * b + 127) / 128 * 4;
    const int64_t rw = D.idx_row_words[m];
    if (rw < need || rw % 4 != 0) return VQ_ERR_INVALID_ARG;
    if (L.n > 0 && L.nvec > 0) {
      if (!D.idx[m] || !D.codebook[m]) return VQ_ERR_INVALID_ARG;
      if (!aligned(D.idx[m], 16) || !aligned(D.codebook[m], 16)) return VQ_ERR_ALIGNMENT;
    }
    L.b[m] = b;
    L.rw[m] = rw;
    L.idx[m] = D.idx[m];
    L.book[m] = D.codebook[m];
  }
  if (L.nb == 1) {      // unused book-2 slots mirror book 1 so kernels never see nulls
    L.b[1] = L.b[0];
    L.rw[1] = L.rw[0];
    L.idx[1] = L.idx[0];
    L.book[1] = L.book[0];
  }
  if ((D.scale && !aligned(D.scale, 2)) || (D.bias && !aligned(D.bias, 2)) ||
      (D.out_bias && !aligned(D.out_bias, 2)))
    return VQ_ERR_ALIGNMENT;
  L.scale = D.scale;
  L.bias = D.bias;
  L.ob = D.out_bias;
  *out = L;
  return VQ_OK;
}

vq_status gemv_workspace_bytes(const vq_layer_desc* layer, int32_t batch, size_t cap,
                               size_t* bytes) {
  if (!bytes) return VQ_ERR_INVALID_ARG;
  Layer L;
  vq_status st = check_layer(layer, &L);
  if (st != VQ_OK) return st;
  if (batch < 0) return VQ_ERR_INVALID_ARG;
  if (batch > kMaxBatch) return VQ_ERR_UNSUPPORTED;
  *bytes = 0;
  if (batch == 0 || L.n == 0) return VQ_OK;
  GemvPlan p;
  st = plan_gemv(L, batch, &p, cap);
  if (st != VQ_OK) return st;
  *bytes = p.ws_bytes;
  return VQ_OK;
}

vq_status gemv_run(const vq_layer_desc* layer, const void* x, vq_dtype x_dtype, int32_t batch,
                   int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy, void* workspace,
                   size_t workspace_bytes, size_t cap, cudaStream_t stream) {
  Layer L;
  vq_status st = check_layer(layer, &L);
  if (st != VQ_OK) return st;
  if (batch < 0 || !dtype_ok_in(x_dtype) || !dtype_ok_out(y_dtype)) return VQ_ERR_INVALID_ARG;
  if (batch > kMaxBatch) return VQ_ERR_UNSUPPORTED;
  if (ldx < L.kin || ldy < L.n) return VQ_ERR_INVALID_ARG;
  if (batch == 0 || L.n == 0) return VQ_OK;
  if (!y || (!x && L.kin > 0)) return VQ_ERR_INVALID_ARG;
  if (!aligned(x, 2) || !aligned(y, dtype_size(y_dtype))) return VQ_ERR_ALIGNMENT;
  GemvPlan p;
  st = plan_gemv(L, batch, &p, cap);
  if (st != VQ_OK) return st;
  if (p.ws_bytes > 0) {
    if (!workspace || workspace_bytes < p.ws_bytes) return VQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return VQ_ERR_ALIGNMENT;
  }
  return launch_gemv(L, p, x, x_dtype == VQ_FP16, batch, ldx, y, y_dtype, ldy,
                     static_cast<float*>(workspace), stream);
}

// Layers sharing x: validated descriptions, the common checks of both entry points.
constexpr int kMaxMultiLayers = 16;

vq_status multi_check(const vq_layer_desc* const* layers, int32_t n_layers, int32_t batch, Layer* L) {
  if (!layers || n_layers < 1 || n_layers > kMaxMultiLayers || batch < 0) return VQ_ERR_INVALID_ARG;
  if (batch > kMaxBatch) return VQ_ERR_UNSUPPORTED;
  for (int l = 0; l < n_layers; ++l) {
    vq_status st = check_layer(layers[l], &L[l]);
    if (st != VQ_OK) return st;
    if (L[l].kin != L[0].kin) return VQ_ERR_INVALID_ARG;
  }
  return VQ_OK;
}

// Workspace of the fused launch when the layers qualify, else the largest
// single-layer need (the layers then run one after another on the stream).
vq_status multi_workspace(const Layer* L, const vq_layer_desc* const* layers, int n_layers, int32_t batch,
                          bool* fused, LutMultiPlan* mp, size_t* bytes) {
  *fused = batch == 1 && plan_gemv_lut_multi(L, n_layers, batch, ~static_cast<size_t>(0), mp);
  if (*fused) {
    *bytes = mp->ws_bytes;
    return VQ_OK;
  }
  size_t need = 0;
  for (int l = 0; l < n_layers; ++l) {
    size_t b = 0;
    vq_status st = gemv_workspace_bytes(layers[l], batch, ~static_cast<size_t>(0), &b);
    if (st != VQ_OK) return st;
    need = std::max(need, b);
  }
  *bytes = need;
  return VQ_OK;
}

}  // namespace vqk

using namespace vqk;

extern "C" {

vq_status vq_hessian_workspace_size(int32_t n_tokens, int32_t d_in, size_t* bytes) {
  if (!bytes || n_tokens < 0 || d_in < 0) return VQ_ERR_INVALID_ARG;
  *bytes = hessian_workspace_bytes(n_tokens, d_in);
  return VQ_OK;
}

vq_status vq_hessian(const void* x, vq_dtype x_dtype, int32_t n_tokens, int32_t d_in, int64_t ldx, float* h,
                     int64_t ldh, void* workspace, size_t workspace_bytes, void* stream) {
  if (n_tokens < 1 || d_in < 0 || ldx < d_in || ldh < d_in || !dtype_ok_in(x_dtype)) return VQ_ERR_INVALID_ARG;
  if (d_in == 0) return VQ_OK;
  if (!x || !h) return VQ_ERR_INVALID_ARG;
  if (!aligned(x, 2) || !aligned(h, 4)) return VQ_ERR_ALIGNMENT;
  const size_t need = hessian_workspace_bytes(n_tokens, d_in);
  if (!workspace || workspace_bytes < need) return VQ_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return VQ_ERR_ALIGNMENT;
  return launch_hessian(x, x_dtype == VQ_FP16, n_tokens, d_in, ldx, h, ldh, workspace, workspace_bytes,
                        static_cast<cudaStream_t>(stream));
}

vq_status vq_gemv_multi_workspace_size(const vq_layer_desc* const* layers, int32_t n_layers, int32_t batch,
                                       size_t* bytes) {
  if (!bytes) return VQ_ERR_INVALID_ARG;
  Layer L[kMaxMultiLayers];
  vq_status st = multi_check(layers, n_layers, batch, L);
  if (st != VQ_OK) return st;
  bool fused;
  LutMultiPlan mp;
  return multi_workspace(L, layers, n_layers, batch, &fused, &mp, bytes);
}

vq_status vq_gemv_multi(const vq_layer_desc* const* layers, int32_t n_layers, const void* x, vq_dtype x_dtype,
                        int32_t batch, int64_t ldx, void* const* y, vq_dtype y_dtype, const int64_t* ldy,
                        void* workspace, size_t workspace_bytes, void* stream) {
  Layer L[kMaxMultiLayers];
  vq_status st = multi_check(layers, n_layers, batch, L);
  if (st != VQ_OK) return st;
  if (!dtype_ok_in(x_dtype) || !dtype_ok_out(y_dtype)) return VQ_ERR_INVALID_ARG;
  if (batch == 0) return VQ_OK;
  if (!y || !ldy) return VQ_ERR_INVALID_ARG;
  if (ldx < L[0].kin) return VQ_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (ldy[l] < L[l].n) return VQ_ERR_INVALID_ARG;
  bool fused;
  LutMultiPlan mp;
  size_t need = 0;
  st = multi_workspace(L, layers, n_layers, batch, &fused, &mp, &need);
  if (st != VQ_OK) return st;
  if (!fused) {
    for (int l = 0; l < n_layers; ++l) {
      st = gemv_run(layers[l], x, x_dtype, batch, ldx, y[l], y_dtype, ldy[l], workspace, workspace_bytes,
                    ~static_cast<size_t>(0), static_cast<cudaStream_t>(stream));
      if (st != VQ_OK) return st;
    }
    return VQ_OK;
  }
  if (!x) return VQ_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    if (!y[l]) return VQ_ERR_INVALID_ARG;
    if (!aligned(y[l], dtype_size(y_dtype))) return VQ_ERR_ALIGNMENT;
  }
  if (!aligned(x, 2)) return VQ_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < need) return VQ_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return VQ_ERR_ALIGNMENT;
  return cuda_status(launch_gemv_lut_multi(L, n_layers, mp, x, x_dtype == VQ_FP16, y, y_dtype,
                                           static_cast<float*>(workspace), static_cast<cudaStream_t>(stream)));
}

vq_status vq_dequant(const vq_layer_desc* layer, uint16_t* w_hat, int64_t ldw, void* stream) {
  Layer L;
  vq_status st = check_layer(layer, &L);
  if (st != VQ_OK) return st;
  if (ldw < L.kin) return VQ_ERR_INVALID_ARG;
  if (L.n == 0 || L.kin == 0) return VQ_OK;
  if (!w_hat) return VQ_ERR_INVALID_ARG;
  if (!aligned(w_hat, 2)) return VQ_ERR_ALIGNMENT;
  return launch_dequant(L, w_hat, ldw, static_cast<cudaStream_t>(stream));
}

vq_status vq_repack_tile4(const vq_layer_desc* src, uint32_t* const dst[2],
                          const int64_t dst_tile_words[2], void* stream) {
  Layer L;
  vq_status st = check_layer(src, &L);
  if (st != VQ_OK) return st;
  if (L.layout != VQ_IDX_ROWS || !dst || !dst_tile_words) return VQ_ERR_INVALID_ARG;
  for (int m = 0; m < L.nb; ++m) {
    const int64_t need = (static_cast<int64_t>(L.n) * 4 * L.b[m] + 127) / 128 * 4;
    if (dst_tile_words[m] < need || dst_tile_words[m] % 4 != 0) return VQ_ERR_INVALID_ARG;
    if (L.n > 0 && L.nvec > 0) {
      if (!dst[m]) return VQ_ERR_INVALID_ARG;
      if (!aligned(dst[m], 16)) return VQ_ERR_ALIGNMENT;
    }
  }
  if (L.n == 0 || L.nvec == 0) return VQ_OK;
  return launch_repack_tile4(L, dst, dst_tile_words, static_cast<cudaStream_t>(stream));
}

vq_status vq_gemv_workspace_size(const vq_layer_desc* layer, int32_t batch, size_t* bytes) {
  return gemv_workspace_bytes(layer, batch, ~static_cast<size_t>(0), bytes);
}

vq_status vq_gemv(const vq_layer_desc* layer, const void* x, vq_dtype x_dtype, int32_t batch,
                  int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy, void* workspace,
                  size_t workspace_bytes, void* stream) {
  return gemv_run(layer, x, x_dtype, batch, ldx, y, y_dtype, ldy, workspace, workspace_bytes,
                  ~static_cast<size_t>(0), static_cast<cudaStream_t>(stream));
}

vq_status vq_gemm_workspace_size(const vq_layer_desc* layer, int32_t m, vq_dtype x_dtype,
                                 size_t* bytes) {
  if (!bytes) return VQ_ERR_INVALID_ARG;
  Layer L;
  vq_status st = check_layer(layer, &L);
  if (st != VQ_OK) return st;
  if (m < 0 || !dtype_ok_in(x_dtype)) return VQ_ERR_INVALID_ARG;
  if (L.d > 8) return VQ_ERR_UNSUPPORTED;
  *bytes = (m == 0 || L.n == 0) ? 0 : gemm_workspace_bytes(L, m, x_dtype == VQ_FP16);
  return VQ_OK;
}

vq_status vq_gemm(const vq_layer_desc* layer, const void* x, vq_dtype x_dtype, int32_t m,
                  int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy, void* workspace,
                  size_t workspace_bytes, void* stream) {
  Layer L;
  vq_status st = check_layer(layer, &L);
  if (st != VQ_OK) return st;
  if (m < 0 || !dtype_ok_in(x_dtype) || !dtype_ok_out(y_dtype)) return VQ_ERR_INVALID_ARG;
  if (L.d > 8 || m > (1 << 30)) return VQ_ERR_UNSUPPORTED;
  if (ldx < L.kin || ldy < L.n) return VQ_ERR_INVALID_ARG;
  if (m == 0 || L.n == 0) return VQ_OK;
  if (!y || (!x && L.kin > 0)) return VQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || ldx % 8 != 0 || !aligned(y, dtype_size(y_dtype))) return VQ_ERR_ALIGNMENT;
  const size_t need = gemm_workspace_bytes(L, m, x_dtype == VQ_FP16);
  if (need > 0) {
    if (!workspace || workspace_bytes < need) return VQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return VQ_ERR_ALIGNMENT;
  }
  return launch_gemm(L, x, x_dtype == VQ_FP16, m, ldx, y, y_dtype, ldy, workspace,
                     workspace_bytes, static_cast<cudaStream_t>(stream));
}

const char* vq_status_string(vq_status status) {
  switch (status) {
    case VQ_OK: return "ok";
    case VQ_ERR_INVALID_ARG: return "invalid argument";
    case VQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case VQ_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case VQ_ERR_WORKSPACE: return "workspace missing or too small";
    case VQ_ERR_CUDA: return "CUDA error";
    case VQ_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int vq_last_cuda_error(void) { return g_last_cuda_error; }

int vq_abi_version(void) { return VQ_ABI_VERSION; }

uint64_t vq_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
