// dlrm_sparse_interact_host_static: the host-buffer stage with its device
// staging in a fixed array that the library owns, for callers that cannot
// allocate device memory themselves.
//
// The staging lives in one file-scope __device__ array, so every GPU that
// loads this library holds DLRM_STATIC_SCRATCH_BYTES of it until the process
// exits. Host code cannot use the array's name as a device address (on the
// host it names a stand-in object), so the address is looked up once per
// device with cudaGetSymbolAddress, with that device current, and cached.
#include <atomic>
#include <cstdint>

#include "dlrm_sparse.h"
#include "launch.h"

namespace {

static __device__ __align__(256) unsigned char g_host_staging[DLRM_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_staging_addr[kMaxDevices];

// Device address of g_host_staging on the current device (looked up on the
// first call for that device). Two threads racing on the first call store the
// same address.
int staging_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return dlrm::cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return DLRM_ERR_ARG;
  void* p = g_staging_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_host_staging);
    if (e != cudaSuccess) return dlrm::cuda_fail(e);
    g_staging_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return DLRM_OK;
}

constexpr size_t round_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

}  // namespace

extern "C" int dlrm_sparse_interact_host_static(const float* const* weights,
                                                const int32_t* indices_host,
                                                const int32_t* offsets_host,
                                                const float* dense_host, int B, int F, int L,
                                                int D, int concat_dense, float* pooled_host,
                                                float* inter_host, dlrm_stream_t stream) {
  if (F < 1 || F > DLRM_MAX_TABLES) return DLRM_ERR_TOO_MANY_TABLES;
  if (B < 1 || L < 0 || D < 1) return DLRM_ERR_SHAPE;
  if (static_cast<int64_t>(B) * L > INT32_MAX) return DLRM_ERR_SHAPE;
  if (offsets_host == nullptr || dense_host == nullptr || inter_host == nullptr)
    return DLRM_ERR_NULL;
  if (L > 0 && indices_host == nullptr) return DLRM_ERR_NULL;
  // Region sizes: [indices | offsets | dense] back to back (so a packed host
  // batch crosses in one copy), then the interaction rows and the pooled
  // vectors, each on a 256-byte boundary (16-byte aligned vector paths).
  const size_t P = static_cast<size_t>(F + 1) * F / 2;
  const size_t n_idx = static_cast<size_t>(F) * B * L * sizeof(int32_t);
  const size_t n_off = static_cast<size_t>(F) * B * sizeof(int32_t);
  const size_t n_dense = static_cast<size_t>(B) * D * sizeof(float);
  const size_t n_inter = static_cast<size_t>(B) * (concat_dense ? D + P : P) * sizeof(float);
  const size_t n_pooled = pooled_host ? static_cast<size_t>(B) * F * D * sizeof(float) : 0;
  const size_t at_inter = round_up(n_idx + n_off + n_dense, 256);
  const size_t at_pooled = round_up(at_inter + n_inter, 256);
  if (at_pooled + n_pooled > DLRM_STATIC_SCRATCH_BYTES) return DLRM_ERR_SCRATCH;
  void* base = nullptr;
  const int rc = staging_address(&base);
  if (rc != DLRM_OK) return rc;
  auto* s = static_cast<unsigned char*>(base);
  // Every byte of the array that this call reads is written earlier in the
  // same call (the three input copies, then the kernel), so nothing has to
  // be cleared first.
  return dlrm_sparse_interact_host(
      weights, indices_host, offsets_host, dense_host, B, F, L, D, concat_dense,
      reinterpret_cast<int32_t*>(s), reinterpret_cast<int32_t*>(s + n_idx),
      reinterpret_cast<float*>(s + n_idx + n_off),
      pooled_host ? reinterpret_cast<float*>(s + at_pooled) : nullptr,
      reinterpret_cast<float*>(s + at_inter), pooled_host, inter_host, stream);
}
