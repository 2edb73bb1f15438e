// Measurement helper, not part of the method: the device-memory read ceiling of the
// decode step's access pattern. One thread per CTA streams consecutive 128-row boxes of
// a [rows, d] bf16 array through a shared-memory ring with 2D TMA loads (128-byte
// swizzle, L2 evict-first), as the decode kernel feeds its K and V rows, with as many
// bytes in flight as the decode's ring holds (six 32 KB stages = its three stages of K and
// V), and a consumer warp only waits for each stage and releases it. Timing it over as many bytes
// as one decode step reads, on as many SMs as the decode launch uses, gives the time the
// decode kernel would take if its MMAs, softmax and combine were free.
#include <cudaTypedefs.h>

#include "kvs_common.cuh"
#include "kvs_kernels.h"
#include "ptx.cuh"

namespace kvs {

constexpr int kProbeRows = 128;
constexpr int kProbeStages = 6;

template <int D>
__global__ void __launch_bounds__(64, 1)
stream_probe_kernel(const __grid_constant__ CUtensorMap tm, long long rows,
                    int32_t* __restrict__ flags) {
  constexpr int kBoxes = D / 64;
  constexpr int kStage = kBoxes * kProbeRows * 128;
  extern __shared__ unsigned char dsm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(dsm) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kProbeStages * kStage);
  uint64_t* empty = full + kProbeStages;
  const long long tiles = (rows + kProbeRows - 1) / kProbeRows;
  const long long t0 = tiles * blockIdx.x / gridDim.x, t1 = tiles * (blockIdx.x + 1) / gridDim.x;
  const int n = (int)(t1 - t0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kProbeStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm);
      const uint64_t once = policy_evict_first();
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int s = i % kProbeStages;
        if (i >= kProbeStages && !mbar_wait(&empty[s], ((i / kProbeStages) - 1) & 1)) {
          set_flag(flags, KVS_FLAG_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&full[s], kStage);
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx)
          tma_load_2d_hint(base + s * kStage + bx * kProbeRows * 128, &tm, bx * 64,
                           (int)((t0 + i) * kProbeRows), &full[s], once);
        issued = i + 1;
      }
      for (int i = issued > kProbeStages ? issued - kProbeStages : 0; i < issued; ++i)
        if (!mbar_wait(&full[i % kProbeStages], (i / kProbeStages) & 1))
          set_flag(flags, KVS_FLAG_TIMEOUT);
    }
    __syncwarp();
  } else {
    for (int i = 0; i < n; ++i) {
      const int s = i % kProbeStages;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (i / kProbeStages) & 1));
      if (!ok) {
        if (lane == 0) set_flag(flags, KVS_FLAG_TIMEOUT);
        break;
      }
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
  __syncthreads();
}

cudaError_t launch_stream_probe(const void* buf, long long rows, int d, int ctas, char* ws,
                                cudaStream_t st) {
  if (rows <= 0 || rows >= (1ll << 31) || ctas <= 0 || (d != 64 && d != 128))
    return cudaErrorInvalidValue;
  CUtensorMap m;
  if (!encode_rows_map(&m, buf, (unsigned long long)rows, d, kProbeRows)) return cudaErrorInvalidValue;
  // the ring, then the full / empty barriers (2 x kProbeStages x 8 bytes), 1024-byte alignment
  const size_t smem = (size_t)kProbeStages * (d / 64) * kProbeRows * 128 + 256 + 1024;
  const void* fn = d == 128 ? (const void*)stream_probe_kernel<128> : (const void*)stream_probe_kernel<64>;
  if (!ensure_smem_attr(fn, smem)) return cudaErrorInvalidValue;
  if (d == 128)
    stream_probe_kernel<128><<<ctas, 64, smem, st>>>(m, rows, reinterpret_cast<int32_t*>(ws));
  else
    stream_probe_kernel<64><<<ctas, 64, smem, st>>>(m, rows, reinterpret_cast<int32_t*>(ws));
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace kvs
