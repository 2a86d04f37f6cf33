// static_scratch.cu -- sfn_sparse_ffn_forward_static: the bf16 forward with its
// scratch in a fixed device array, for callers that cannot allocate.
//
// Some callers cannot allocate device memory at the point where they run the
// layer: a plugin interface that hands the layer only its input and output
// pointers, a serving process whose allocator has already claimed the GPU's
// memory, or a latency-critical loop that must not risk the implicit
// synchronisation of cudaMalloc.  This entry point gives them the same
// forward with no allocation at all: its scratch is the file-scope array
// below, which the CUDA runtime places in device memory when this library's
// module is loaded on a GPU and keeps there until the process exits.
//
// It runs exactly the kernels of sfn_sparse_ffn_forward_ws, pointed at that
// array.  It calls no cudaMalloc, cudaFree or other allocating routine.
#include <mutex>

#include "sfn_internal.cuh"

namespace {

// The scratch.  Host code must never hand `g_static_scratch` itself to a
// kernel: in host code the name is only a host-side stand-in for the device
// symbol.  Its device address comes from cudaGetSymbolAddress, below.
static __device__ __align__(256) unsigned char g_static_scratch[SFN_STATIC_SCRATCH_BYTES];

std::mutex g_mu;
void *g_scratch_addr[64];  // device address of g_static_scratch, per device

// Device address of the scratch on the current device.  The first call on a
// device looks it up, with that device current, and caches it.
cudaError_t scratch_address(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" sfn_status sfn_sparse_ffn_forward_static(const void *x, const void *A,
                                                    const void *B, const void *Wg,
                                                    const void *Wu, const void *Wd, void *y,
                                                    uint64_t *mask, int64_t T, int d, int d_i,
                                                    int r, int bank, int k,
                                                    sfn_stream_t stream) {
  const size_t need = sfn_workspace_bytes(T, d, d_i, r, bank, k, SFN_DTYPE_BF16);
  if (need == 0)  // T == 0 or invalid arguments: report them, enqueue nothing
    return sfn_sparse_ffn_forward_ws(x, A, B, Wg, Wu, Wd, y, mask, T, d, d_i, r, bank, k,
                                     nullptr, 0, stream);
  if (need > (size_t)SFN_STATIC_SCRATCH_BYTES) return SFN_ERR_WORKSPACE;
  void *ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) {
    cudaGetLastError();
    return SFN_ERR_CUDA;
  }
  // Every scratch byte the kernels read is written earlier in the same call,
  // so the array's leftover contents from a previous call need no clearing.
  return sfn_sparse_ffn_forward_ws(x, A, B, Wg, Wu, Wd, y, mask, T, d, d_i, r, bank, k, ws,
                                   (size_t)SFN_STATIC_SCRATCH_BYTES, stream);
}
