// nsa_noalloc.cu -- nsa_forward_noalloc: the whole path without a caller
// workspace, for callers that cannot allocate device memory.
//
// Some hosts of this library may not call cudaMalloc (or any allocator) on
// the path where they run attention: a serving process whose device memory
// is owned by another framework's pool allocator, a plugin that is handed
// only the tensors it computes on, or a latency-critical loop that bans
// cudaMalloc because it can synchronise the device and stall other streams.
// They still own and pass the inputs and outputs; the scratch the path
// needs (pooled vectors, per-row kept lists, the plan flag) comes from a
// fixed array in device memory that the library itself declares.
//
// The array is a file-scope __device__ object of NSA_NOALLOC_SCRATCH_BYTES;
// every GPU on which the library's kernels are loaded holds it until the
// process exits. Host code cannot use the array's name as a device address,
// so the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and caches it. Under lazy
// module loading (the CUDA default) that lookup may load the library's
// device code on the device, reserving the array then, and may synchronise:
// callers should make one warm-up call per device at initialisation (or run
// with CUDA_MODULE_LOADING=EAGER), and in any case before any stream capture. Every call shares the one
// array: two calls whose work overlaps on the GPU (e.g. on two streams) race
// and give wrong results. Nothing in the array needs to start at zero: the
// pooling kernel clears the plan flag and every other scratch byte a call
// reads is written earlier in the same call.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/nsa.h"
#include "nsa_kernels.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[NSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
void *g_scratch_ptr[kMaxDev] = {};
std::mutex g_scratch_mu;

}  // namespace

extern "C" nsa_status nsa_forward_noalloc(const void *q, const void *k, const void *v, int B, int Hq, int Hkv,
                                          int Sq, int Skv, int D, const nsa_spec *spec, const int8_t *pins,
                                          const int64_t *pin_strides, const int8_t *drops,
                                          const int64_t *drop_strides, float scale, void *out, float *lse,
                                          int8_t *keep_out, nsa_stream_t stream) {
  // size check first (host only), so an oversized call fails before any CUDA call
  const size_t need = nsa_workspace_bytes(B, Hq, Hkv, Sq, Skv, D, spec);
  if (need == 0)  // invalid sizes or spec: let nsa_forward report the exact reason
    return nsa_forward(q, k, v, B, Hq, Hkv, Sq, Skv, D, spec, pins, pin_strides, drops, drop_strides, scale, out,
                       lse, keep_out, nullptr, 0, stream);
  if (need > (size_t)NSA_NOALLOC_SCRATCH_BYTES) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "nsa_forward_noalloc: these sizes need %zu scratch bytes, above the fixed %zu-byte array; "
             "use nsa_forward with a caller workspace",
             need, (size_t)NSA_NOALLOC_SCRATCH_BYTES);
    nsa::set_last_error(msg);
    return NSA_ERR_INVALID_ARG;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    nsa::set_last_error("nsa_forward_noalloc: no usable current CUDA device");
    return NSA_ERR_CUDA;
  }
  void *ptr = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || p == nullptr) {
        char msg[200];
        snprintf(msg, sizeof(msg), "nsa_forward_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        nsa::set_last_error(msg);
        return NSA_ERR_CUDA;
      }
      g_scratch_ptr[dev] = p;
    }
    ptr = g_scratch_ptr[dev];
  }
  return nsa_forward(q, k, v, B, Hq, Hkv, Sq, Skv, D, spec, pins, pin_strides, drops, drop_strides, scale, out, lse,
                     keep_out, ptr, (size_t)NSA_NOALLOC_SCRATCH_BYTES, stream);
}
