// Split-K GQA decode attention over the merged cache, with the split combine and
// the optional append fused in.
//
// Attention of the KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程",
// §数学主线三) with the log-count logit bias of merged rows; this is the decoder
// stage the pages time (Figure 5).
//
// Grid (nsplit, B*H_kv). The G query heads of a KV head share every K/V row read.
// A CTA's warps take 32-row tiles of its split: lane t computes the G logits of
// row t from a register copy of its key row; the warp updates the online softmax;
// then every lane accumulates its D/32 output columns over the tile's rows.
// The CTA writes (m, l, acc) for its split, bumps the head's arrival counter, and
// the last CTA to arrive combines all splits (no CTA ever waits on another),
// attends the appended row, appends it, and resets the counter.
#include "decode_common.cuh"
#include "kvs_common.cuh"
#include "kvs_kernels.h"

namespace kvs {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;

template <typename T> struct ColVec;      // D/32 columns per lane, as one load
template <> struct ColVec<bf16> {
  template <int CPL>
  __device__ static __forceinline__ void load(const bf16* p, float* f) {
    if constexpr (CPL == 4) {
      uint2 u = __ldcs(reinterpret_cast<const uint2*>(p));
      f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
    } else {
      uint32_t u = __ldcs(reinterpret_cast<const unsigned int*>(p));
      f[0] = bf16_lo(u); f[1] = bf16_hi(u);
    }
  }
};
template <> struct ColVec<float> {
  template <int CPL>
  __device__ static __forceinline__ void load(const float* p, float* f) {
    if constexpr (CPL == 4) {
      float4 v = __ldcs(reinterpret_cast<const float4*>(p));
      f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    } else {
      float2 v = __ldcs(reinterpret_cast<const float2*>(p));
      f[0] = v.x; f[1] = v.y;
    }
  }
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(const T* __restrict__ q, T* K, T* V, float* logn, int32_t* len,
              const T* __restrict__ k_new,
              const T* __restrict__ v_new, T* __restrict__ out, int H_kv, int T_cap, int nsplit,
              int32_t* __restrict__ counters, float* __restrict__ part,
              int32_t* __restrict__ flags) {
  constexpr int VN = Vec16<T>::n;
  constexpr int VPR = D / VN;              // 16-byte vectors per row
  constexpr int CPL = D / 32;              // output columns per lane
  __shared__ __align__(16) float qs[G][D];
  __shared__ float s_m[kDecWarps][G], s_l[kDecWarps][G];
  __shared__ __align__(16) float s_acc[kDecWarps][G][D];
  __shared__ float s_new[G];
  __shared__ float s_fac[G][kMaxDecodeSplits];
  __shared__ float s_gstat[G][2];
  __shared__ int s_last;

  const int head = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int L = len[head];
  const bool bad = L < 0 || L > T_cap;
  if (bad) {
    if (split == 0 && tid == 0) set_flag(flags, KVS_FLAG_BAD_LENGTH);
    L = 0;
  }
  const float qscale = kLog2e / sqrtf((float)D);
  for (int i = tid; i < G * D; i += kDecThreads) {
    const int g = i / D, c = i - g * D;
    qs[g][c] = to_f32(q[((size_t)head * G + g) * D + c]) * qscale;
  }
  __syncthreads();

  int chunk = (L + nsplit - 1) / nsplit;
  chunk = (chunk + 31) & ~31;
  const int t0 = split * chunk, t1 = min(L, t0 + chunk);
  const T* Kh = K + (size_t)head * T_cap * D;
  const T* Vh = V + (size_t)head * T_cap * D;
  const float* lnh = logn ? logn + (size_t)head * T_cap : nullptr;

  float m[G], l[G], acc[G][CPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int k = 0; k < CPL; ++k) acc[g][k] = 0.f;
  }

  for (int tb = t0 + warp * 32; tb < t1; tb += kDecWarps * 32) {
    const int t = tb + lane;
    const bool valid = t < t1;
    float s[G];
#pragma unroll
    for (int g = 0; g < G; ++g) s[g] = 0.f;
    if (valid) {
      const T* kr = Kh + (size_t)t * D;
#pragma unroll 4
      for (int cv = 0; cv < VPR; ++cv) {
        float f[VN];
        load_vec_cs(kr + cv * VN, f);
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
          for (int e = 0; e < VN; e += 4) {
            const float4 qv = *reinterpret_cast<const float4*>(&qs[g][cv * VN + e]);
            s[g] = fmaf(qv.x, f[e], s[g]);
            s[g] = fmaf(qv.y, f[e + 1], s[g]);
            s[g] = fmaf(qv.z, f[e + 2], s[g]);
            s[g] = fmaf(qv.w, f[e + 3], s[g]);
          }
        }
      }
      const float lb = lnh ? __ldcs(lnh + t) * kLog2e : 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) s[g] += lb;
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) s[g] = -INFINITY;
    }
    float p[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float m_new = fmaxf(m[g], warp_max(s[g]));
      const float corr = exp2f(m[g] - m_new);
      p[g] = exp2f(s[g] - m_new);
      l[g] = l[g] * corr + warp_sum(p[g]);
#pragma unroll
      for (int k = 0; k < CPL; ++k) acc[g][k] *= corr;
      m[g] = m_new;
    }
    const int nv = min(32, t1 - tb);
    const T* vr = Vh + (size_t)tb * D + lane * CPL;
#pragma unroll 4
    for (int i = 0; i < nv; ++i) {
      float v[CPL];
      ColVec<T>::template load<CPL>(vr + (size_t)i * D, v);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pg = __shfl_sync(0xffffffffu, p[g], i);
#pragma unroll
        for (int k = 0; k < CPL; ++k) acc[g][k] = fmaf(pg, v[k], acc[g][k]);
      }
    }
  }

  // combine the warps of this CTA, publish the split, finish if last
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) { s_m[warp][g] = m[g]; s_l[warp][g] = l[g]; }
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int k = 0; k < CPL; ++k) s_acc[warp][g][lane * CPL + k] = acc[g][k];
  __syncthreads();
  // the (m, l) staging of the last CTA overlays s_acc, which is consumed by then
  static_assert(kDecWarps * G * D >= 2 * G * kMaxDecodeSplits, "(m, l) staging fits s_acc");
  const DecodeSmem<D, G, kDecWarps> S{s_m, s_l, s_acc, qs, s_new, s_fac, s_gstat, &s_last};
  const DecodeArgs<T> a{head, split, nsplit, L, T_cap, bad, K, V, logn, len, k_new, v_new,
                        out, counters, part, flags};
  decode_epilogue<T, D, G, kDecWarps>(S, &s_acc[0][0][0], a, tid, kDecThreads);
}

template <typename T, int D>
static cudaError_t launch_decode_t(const kvs_cache_desc& d, const void* q, void* K, void* V,
                                   float* logn, int32_t* len, const void* k_new,
                                   const void* v_new, void* out, const DecodeLayout& Ly,
                                   char* ws, cudaStream_t st) {
  const int G = d.H_q / d.H_kv;
  dim3 grid(Ly.nsplit, d.B * d.H_kv);
  int32_t* flags = reinterpret_cast<int32_t*>(ws);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + Ly.counters);
  float* part = reinterpret_cast<float*>(ws + Ly.part);
#define KVS_DEC(GG)                                                                         \
  decode_kernel<T, D, GG><<<grid, kDecThreads, 0, st>>>(                                   \
      (const T*)q, (T*)K, (T*)V, logn, len, (const T*)k_new, (const T*)v_new, (T*)out,      \
      d.H_kv, d.T_cap, Ly.nsplit, counters, part, flags)
  switch (G) {
    case 1: KVS_DEC(1); break;
    case 2: KVS_DEC(2); break;
    case 4: KVS_DEC(4); break;
    case 8: KVS_DEC(8); break;
    default: return cudaErrorInvalidValue;
  }
#undef KVS_DEC
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_decode(const kvs_cache_desc& d, const void* q, void* K, void* V, float* logn,
                          int32_t* len, const void* k_new, const void* v_new, void* out,
                          const DecodeLayout& Ly, char* ws, cudaStream_t st) {
  // bf16 caches take the TMA + tensor-core kernel; fp32 caches (and caches too large
  // for 32-bit TMA row coordinates) the CUDA-core kernel below
  if (decode_tc_supported(d))
    return launch_decode_tc(d, q, K, V, logn, len, k_new, v_new, out, Ly, ws, st);
  if (d.dtype == KVS_BF16) {
    if (d.d == 128) return launch_decode_t<bf16, 128>(d, q, K, V, logn, len, k_new, v_new, out, Ly, ws, st);
    return launch_decode_t<bf16, 64>(d, q, K, V, logn, len, k_new, v_new, out, Ly, ws, st);
  }
  if (d.d == 128) return launch_decode_t<float, 128>(d, q, K, V, logn, len, k_new, v_new, out, Ly, ws, st);
  return launch_decode_t<float, 64>(d, q, K, V, logn, len, k_new, v_new, out, Ly, ws, st);
}

}  // namespace kvs
