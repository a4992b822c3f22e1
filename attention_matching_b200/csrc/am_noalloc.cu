// am_compact_heads_noalloc: the full compaction with its scratch memory in a
// fixed device array owned by this library, for callers that cannot allocate
// device memory (see include/am_b200.h for who they are and the rules).
#include "am_internal.cuh"

#include <mutex>

namespace am {
namespace {

// The scratch area.  In host code this name is only a stand-in for the
// symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[AM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch area on the current device, looked up once
// per device with that device current.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

// Status words are stored most-severe-wins as 1000·severity + code; report
// the plain code.
__global__ void k_status_codes(const int32_t* words, int32_t* out, int H) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) out[h] = words[h] % 1000;
}

}  // namespace
}  // namespace am

extern "C" am_status_t am_compact_heads_noalloc(const void* Q, const void* K, const void* V, int32_t n,
                                                int32_t T, int32_t d, int32_t H, const int32_t* budgets,
                                                const am_opts_t* opts, const int64_t* out_offsets, void* C_k,
                                                float* beta, float* C_v, int32_t* indices, int32_t* status_out,
                                                void* stream) {
  size_t need = 0;
  am_status_t st = am_workspace_size(n, T, d, H, budgets, opts, &need);
  if (st != AM_OK) return st;
  if (need > AM_NOALLOC_SCRATCH_BYTES) return AM_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (am::scratch_address(&scratch) != cudaSuccess) return AM_ERR_CUDA;
  // one stream: this entry creates no stream or event either
  st = am::compact_heads_impl(Q, K, V, n, T, d, H, budgets, opts, scratch, AM_NOALLOC_SCRATCH_BYTES, out_offsets,
                              C_k, beta, C_v, indices, stream, 1);
  if (st != AM_OK) return st;
  if (status_out) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int32_t* words =
        reinterpret_cast<const int32_t*>(reinterpret_cast<const char*>(scratch) + am::kWsHeaderBytes);
    am::k_status_codes<<<(H + 127) / 128, 128, 0, s>>>(words, status_out, H);
    if (cudaGetLastError() != cudaSuccess) return AM_ERR_CUDA;
  }
  return AM_OK;
}
