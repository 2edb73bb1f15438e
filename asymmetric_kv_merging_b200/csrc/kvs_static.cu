// kvs_decode_attn_static: the decode step with its scratch memory built into the
// library, for callers that cannot allocate device memory when they call us.
//
// Such callers exist: a runtime whose device-memory plan is fixed before it starts
// serving (every byte belongs to its own pool), a host framework that gives a plugin
// nothing but a stream to enqueue work on, or code that must not call cudaMalloc
// because allocation would synchronise the device in the middle of its step. They
// cannot provide the workspace kvs_decode_attn needs, so this entry point uses a
// fixed buffer that lives in the library's own device memory instead.
//
// The buffer is a file-scope __device__ array of kvs_static_scratch_bytes() bytes;
// every GPU that loads the library holds it until the process exits. In host code the
// array's name is only a host-side stand-in, never a device address, so its device
// address is looked up once per device (cudaGetSymbolAddress, with that device
// current) and that address is what the kernels receive.
#include <cuda_runtime.h>

#include <mutex>

#include "kvs.h"
#include "kvs_common.cuh"
#include "kvs_kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = 4u << 20;   // 4 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the built-in scratch on the current device (looked up once).
kvs_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVS_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KVS_OK;
}

}  // namespace

extern "C" {

size_t kvs_static_scratch_bytes(void) { return kStaticScratchBytes; }

kvs_status kvs_decode_attn_static(const kvs_cache_desc* desc, const void* q, void* K, void* V,
                                  float* logn, int32_t* len, const void* k_new,
                                  const void* v_new, void* out, kvs_stream_t stream) {
  const size_t need = kvs_workspace_size(desc, 0, KVS_OP_DECODE);
  if (need == 0) return desc ? KVS_ERR_UNSUPPORTED : KVS_ERR_INVALID_ARG;
  if (need > kStaticScratchBytes) return KVS_ERR_WORKSPACE;   // shape too large for the buffer
  void* scratch = nullptr;
  kvs_status s = scratch_on_current_device(&scratch);
  if (s != KVS_OK) return s;
  // The buffer keeps whatever the previous call left. The arrival counters must start at
  // zero (a call whose pipeline wait gave up can leave them set), so that block is
  // cleared on the stream first; the flag word before it is left alone, so that flags
  // accumulate until kvs_static_device_flags reads and clears them.
  const size_t counters = kvs::decode_layout(*desc).counters;
  const size_t head_region = kvs::persistent_bytes(*desc);
  if (cudaMemsetAsync(static_cast<char*>(scratch) + counters, 0, head_region - counters,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KVS_ERR_CUDA;
  return kvs_decode_attn(desc, q, K, V, logn, len, k_new, v_new, out, scratch,
                         kStaticScratchBytes, stream);
}

kvs_status kvs_static_device_flags(int32_t* flags, int32_t clear, kvs_stream_t stream) {
  if (!flags) return KVS_ERR_INVALID_ARG;
  void* scratch = nullptr;
  kvs_status s = scratch_on_current_device(&scratch);
  if (s != KVS_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, scratch, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return KVS_ERR_CUDA;
  if (clear && cudaMemsetAsync(scratch, 0, sizeof(int32_t), st) != cudaSuccess) return KVS_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return KVS_ERR_CUDA;
  *flags = h;
  return KVS_OK;
}

}  // extern "C"
