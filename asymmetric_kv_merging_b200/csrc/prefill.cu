// Chunked streaming prefill compression: append a prompt chunk, then merge back to the
// budget in place.
//
// The serving loop of the KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的
// 数学与工程", §实验设置: compression context budget 2048, chunk size 512, 32 preserved
// initial tokens): the prompt enters the cache one chunk at a time and every chunk is
// followed by as many merge rounds as bring each head back to the budget. The rounds are
// the hot path's own kernels (window statistics, pair scores, selection, in-place merge);
// this file adds the row append and the host-side round plan.
#include <cuda_runtime.h>

#include "kvs_common.cuh"
#include "kvs_kernels.h"

namespace kvs {

constexpr int kAppendThreads = 256;
constexpr int kAppendRowsPerBlock = 64;

// grid (ceil(n / kAppendRowsPerBlock), B*H_kv). Every block reads len[head] before it
// arrives on the head's counter; the last block to arrive advances len, so no block
// reads len after it changed.
template <typename T, int D>
__global__ void __launch_bounds__(kAppendThreads)
append_rows_kernel(T* __restrict__ K, T* __restrict__ V, float* __restrict__ logn,
                   int32_t* __restrict__ len, int L, const T* __restrict__ k_rows,
                   const T* __restrict__ v_rows, int n, int T_cap, int32_t* __restrict__ counters,
                   int32_t* __restrict__ flags) {
  constexpr int VN = Vec16<T>::n;
  constexpr int VPR = D / VN;                       // 16-byte vectors per row
  __shared__ int s_ok, s_last;
  const int head = blockIdx.y;
  const int r0 = blockIdx.x * kAppendRowsPerBlock;
  const int r1 = min(n, r0 + kAppendRowsPerBlock);
  // this thread's vectors of the new rows are loaded together with the length check (the
  // loads do not depend on it), so the block waits one round trip, not one per vector
  constexpr int kPer = (kAppendRowsPerBlock * VPR + kAppendThreads - 1) / kAppendThreads;
  const uint4* ks = reinterpret_cast<const uint4*>(k_rows + ((size_t)head * n + r0) * D);
  const uint4* vs = reinterpret_cast<const uint4*>(v_rows + ((size_t)head * n + r0) * D);
  const int nv = (r1 - r0) * VPR;
  uint4 kv[kPer], vv[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = threadIdx.x + j * kAppendThreads;
    if (i < nv) {
      kv[j] = __ldcs(ks + i);
      vv[j] = __ldcs(vs + i);
    }
  }
  if (threadIdx.x == 0) {
    s_ok = (len[head] == L);
    if (!s_ok && blockIdx.x == 0) set_flag(flags, KVS_FLAG_BAD_LENGTH);
  }
  __syncthreads();
  if (!s_ok) return;                                // the whole head is left as it is
  uint4* kd = reinterpret_cast<uint4*>(K + ((size_t)head * T_cap + L + r0) * D);
  uint4* vd = reinterpret_cast<uint4*>(V + ((size_t)head * T_cap + L + r0) * D);
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = threadIdx.x + j * kAppendThreads;
    if (i < nv) {
      kd[i] = kv[j];
      vd[i] = vv[j];
    }
  }
  if (logn)
    for (int r = r0 + threadIdx.x; r < r1; r += kAppendThreads)
      logn[(size_t)head * T_cap + L + r] = 0.f;     // appended rows have count 1
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&counters[head], 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (s_last && threadIdx.x == 0) {
    len[head] = L + n;
    counters[head] = 0;
  }
}

__global__ void fill2_kernel(int32_t* a, int32_t va, int32_t* b, int32_t vb, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    a[i] = va;
    b[i] = vb;
  }
}

template <typename T, int D>
static cudaError_t launch_append_t(const kvs_cache_desc& d, void* K, void* V, float* logn,
                                   int32_t* len, int L, const void* k_rows, const void* v_rows,
                                   int n, char* ws, cudaStream_t st) {
  dim3 grid((n + kAppendRowsPerBlock - 1) / kAppendRowsPerBlock, d.B * d.H_kv);
  append_rows_kernel<T, D><<<grid, kAppendThreads, 0, st>>>(
      (T*)K, (T*)V, logn, len, L, (const T*)k_rows, (const T*)v_rows, n, d.T_cap,
      reinterpret_cast<int32_t*>(ws + kWsAlign), reinterpret_cast<int32_t*>(ws));
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_append_rows(const kvs_cache_desc& d, void* K, void* V, float* logn,
                               int32_t* len, int L, const void* k_rows, const void* v_rows, int n,
                               char* ws, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  if (d.dtype == KVS_BF16)
    return d.d == 128 ? launch_append_t<bf16, 128>(d, K, V, logn, len, L, k_rows, v_rows, n, ws, st)
                      : launch_append_t<bf16, 64>(d, K, V, logn, len, L, k_rows, v_rows, n, ws, st);
  return d.d == 128 ? launch_append_t<float, 128>(d, K, V, logn, len, L, k_rows, v_rows, n, ws, st)
                    : launch_append_t<float, 64>(d, K, V, logn, len, L, k_rows, v_rows, n, ws, st);
}

cudaError_t launch_fill2(int32_t* a, int32_t va, int32_t* b, int32_t vb, int n, cudaStream_t st) {
  fill2_kernel<<<(n + 255) / 256, 256, 0, st>>>(a, va, b, vb, n);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace kvs
