// Epilogue shared by the decode kernels: merge the CTA's per-warp softmax partials,
// publish the split's partial, and let the last CTA of a head combine all splits,
// attend and append the new row, and reset the head's arrival counter.
//
// Softmax partials are (m, l, acc) in the log2 domain: m the running maximum of
// s = log2(e) (q.k / sqrt(d) + logn), l = sum 2^(s - m), acc = sum 2^(s - m) v.
#pragma once

#include "kvs_common.cuh"

namespace kvs {

template <typename T>
__device__ __forceinline__ void store_out(T* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<bf16>(bf16* p, float v) { *p = __float2bfloat16_rn(v); }

// All `nthreads` threads of the CTA call this after __syncthreads(); the warp partials
// sm[NW][G], sl[NW][G], sacc[NW][G][D] live in shared memory. qs[G][D] holds the
// scaled queries (fp32, log2 domain). Query head g of KV head `head` (= b*H_kv + h)
// is head*G + g. Returns after the CTA's part is done.
template <typename T, int D, int G, int NW>
__device__ __forceinline__ void decode_epilogue(
    const float (*sm)[G], const float (*sl)[G], const float (*sacc)[G][D], const float (*qs)[D],
    float* s_new, int* s_last, int tid, int nthreads, int head, int split, int nsplit, int L,
    bool bad, int T_cap, T* K, T* V, float* logn, int32_t* len, const T* k_new,
    const T* v_new, T* out, int32_t* counters, float* part_ml, float* part_acc,
    int32_t* flags) {
  const int lane = tid & 31, warp = tid >> 5;
  float* pml = part_ml + ((size_t)(head)*G) * nsplit * 2;
  float* pacc = part_acc + ((size_t)(head)*G) * nsplit * D;
  for (int i = tid; i < G * D; i += nthreads) {
    const int g = i / D, c = i - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sm[w][g]);
    float Ls = 0.f, A = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float f = exp2f(sm[w][g] - M);
        Ls = fmaf(sl[w][g], f, Ls);
        A = fmaf(sacc[w][g][c], f, A);
      }
    }
    pacc[((size_t)g * nsplit + split) * D + c] = A;
    if (c == 0) {
      pml[((size_t)g * nsplit + split) * 2 + 0] = M;
      pml[((size_t)g * nsplit + split) * 2 + 1] = Ls;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) *s_last = (atomicAdd(&counters[head], 1) == nsplit - 1);
  __syncthreads();
  if (!*s_last) return;
  __threadfence();

  const bool append = (k_new != nullptr) && (v_new != nullptr) && !bad;
  const bool fits = L < T_cap;
  const T* kn = append ? k_new + (size_t)head * D : nullptr;
  const T* vn = append ? v_new + (size_t)head * D : nullptr;
  if (append && fits) {
    for (int g = warp; g < G; g += nthreads / 32) {
      float sp = 0.f;
      for (int c = lane; c < D; c += 32) sp = fmaf(qs[g][c], to_f32(kn[c]), sp);
      sp = warp_sum(sp);
      if (lane == 0) s_new[g] = sp;   // appended rows have count 1: no bias
    }
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += nthreads) {
    const int g = i / D, c = i - g * D;
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) {
      const float ls = __ldcg(pml + ((size_t)g * nsplit + s) * 2 + 1);
      if (ls > 0.f) M = fmaxf(M, __ldcg(pml + ((size_t)g * nsplit + s) * 2));
    }
    if (append && fits) M = fmaxf(M, s_new[g]);
    float Ls = 0.f, A = 0.f;
    if (M > -INFINITY) {
      for (int s = 0; s < nsplit; ++s) {
        const float ls = __ldcg(pml + ((size_t)g * nsplit + s) * 2 + 1);
        if (ls > 0.f) {
          const float f = exp2f(__ldcg(pml + ((size_t)g * nsplit + s) * 2) - M);
          Ls = fmaf(ls, f, Ls);
          A = fmaf(__ldcg(pacc + ((size_t)g * nsplit + s) * D + c), f, A);
        }
      }
      if (append && fits) {
        const float f = exp2f(s_new[g] - M);
        Ls += f;
        A = fmaf(to_f32(vn[c]), f, A);
      }
    }
    store_out<T>(out + ((size_t)head * G + g) * D + c, Ls > 0.f ? A / Ls : 0.f);
  }
  if (append) {
    if (fits) {
      for (int c = tid; c < D; c += nthreads) {
        K[((size_t)head * T_cap + L) * D + c] = kn[c];
        V[((size_t)head * T_cap + L) * D + c] = vn[c];
      }
      if (tid == 0 && logn) logn[(size_t)head * T_cap + L] = 0.f;
    } else if (tid == 0) {
      set_flag(flags, KVS_FLAG_OUT_CAPACITY);
    }
  }
  __syncthreads();
  if (tid == 0) {
    if (append && fits) len[head] = L + 1;
    counters[head] = 0;
  }
}

}  // namespace kvs
