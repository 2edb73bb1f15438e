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
// is head*G + g. `scratch` is shared memory for 2*G*nsplit + 2*G floats that may
// overlap sacc (sacc is consumed before scratch is written). Returns after the CTA's
// part is done.
template <typename T, int D, int G, int NW>
__device__ __forceinline__ void decode_epilogue(
    const float (*sm)[G], const float (*sl)[G], const float (*sacc)[G][D], const float (*qs)[D],
    float* s_new, int* s_last, float* scratch, int tid, int nthreads, int head, int split,
    int nsplit, int L,
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
  // The combine must not wait on one L2 round trip per split: stage every split's
  // (m, l) in shared memory with one parallel pass, turn them into scale factors,
  // then reduce the accumulators four columns per thread with independent loads.
  float* f_m = scratch;                    // [G * nsplit]   split maxima, then scale factors
  float* f_l = scratch + G * nsplit;       // [G * nsplit]   split sums
  float* g_stat = f_l + G * nsplit;        // [G][2]         combined (M, 1/L)
  for (int i = tid; i < G * nsplit; i += nthreads) {
    const float2 ml = __ldcg(reinterpret_cast<const float2*>(pml) + i);
    f_m[i] = ml.x;
    f_l[i] = ml.y;
  }
  __syncthreads();
  for (int g = tid; g < G; g += nthreads) {
    float M = (append && fits) ? s_new[g] : -INFINITY;
    for (int s = 0; s < nsplit; ++s)
      if (f_l[g * nsplit + s] > 0.f) M = fmaxf(M, f_m[g * nsplit + s]);
    float Ls = (append && fits && M > -INFINITY) ? exp2f(s_new[g] - M) : 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const float ls = f_l[g * nsplit + s];
      const float f = (ls > 0.f && M > -INFINITY) ? exp2f(f_m[g * nsplit + s] - M) : 0.f;
      f_m[g * nsplit + s] = f;               // now the scale factor of split s
      Ls = fmaf(ls, f, Ls);
    }
    g_stat[2 * g] = M;
    g_stat[2 * g + 1] = Ls > 0.f ? 1.f / Ls : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < G * (D / 4); e += nthreads) {
    const int g = e / (D / 4), c = (e - g * (D / 4)) * 4;
    // every split wrote its accumulator (zeros when it saw no rows), so the loads need
    // no guard and sixteen of them can be in flight at once
    float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* src = reinterpret_cast<const float4*>(pacc + (size_t)g * nsplit * D + c);
#pragma unroll 16
    for (int s = 0; s < nsplit; ++s) {
      const float f = f_m[g * nsplit + s];
      const float4 v = __ldcg(src + (size_t)s * (D / 4));
      A.x = fmaf(v.x, f, A.x); A.y = fmaf(v.y, f, A.y);
      A.z = fmaf(v.z, f, A.z); A.w = fmaf(v.w, f, A.w);
    }
    if (append && fits) {
      const float f = exp2f(s_new[g] - g_stat[2 * g]);
      A.x = fmaf(to_f32(vn[c]), f, A.x); A.y = fmaf(to_f32(vn[c + 1]), f, A.y);
      A.z = fmaf(to_f32(vn[c + 2]), f, A.z); A.w = fmaf(to_f32(vn[c + 3]), f, A.w);
    }
    const float inv = g_stat[2 * g + 1];
    T* o = out + ((size_t)head * G + g) * D + c;
    store_out<T>(o, A.x * inv); store_out<T>(o + 1, A.y * inv);
    store_out<T>(o + 2, A.z * inv); store_out<T>(o + 3, A.w * inv);
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
