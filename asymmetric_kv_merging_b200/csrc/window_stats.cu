// Window statistics of one scoring pass (CUDA-core path, any dtype / head dim).
//
// Attention forward of the KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称
// KV 合并的数学与工程", §数学主线三): e = q k^T / sqrt(d) (+ log count), alpha =
// softmax(e), o = sum alpha v, for every window query; the window mean of alpha
// and of o feed the pair norms of §数学主线四.
//
//   window_partial_kernel : per (KV head, key split): online softmax of the G*W
//                           window queries over the split's keys -> (m, l, o) partials
//   window_combine_kernel : per (KV head, block of queries): merge the splits ->
//                           per-query (m, l), and sums of o_q over the block
//   obar_kernel           : per KV head: o_bar = mean_q o_q from the block sums
//   alpha_bar_kernel      : per (KV head, 64 keys): alpha_bar_t = mean_q 2^(s_qt - m_q) / l_q
//
// Logits are kept in the log2 domain: s = (q log2(e)/sqrt(d)) . k + log2(e) logn.
#include "kvs_common.cuh"
#include "kvs_kernels.h"

namespace kvs {

constexpr int kWinThreads = 128;
constexpr int kWinTile = 16;
constexpr int kAlphaTokens = 64;
constexpr int kAlphaThreads = 256;

template <typename T, int D>
__device__ __forceinline__ void load_queries_scaled(const T* __restrict__ Qw, float* Qs, int DP,
                                                    int b, int h, int H_q, int G, int W,
                                                    int tid, int nthreads) {
  const float qscale = kLog2e / sqrtf((float)D);
  const int Qn = G * W;
  for (int idx = tid; idx < Qn * D; idx += nthreads) {
    int q = idx / D, c = idx - q * D;
    int g = q / W, j = q - g * W;
    size_t src = (((size_t)b * H_q + (size_t)h * G + g) * W + j) * D + c;
    Qs[q * DP + c] = to_f32(Qw[src]) * qscale;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kWinThreads)
window_partial_kernel(const T* __restrict__ K, const T* __restrict__ V,
                      const float* __restrict__ logn, const int32_t* __restrict__ len,
                      const T* __restrict__ Qw, int H_kv, int H_q, int T_cap, int W, int nsplit,
                      float* __restrict__ part_ml, float* __restrict__ part_o,
                      int32_t* __restrict__ flags) {
  extern __shared__ __align__(16) float smem[];
  constexpr int DP = D + 4;
  constexpr int VN = Vec16<T>::n;
  constexpr int VPR = D / VN;
  const int G = H_q / H_kv;
  const int Qn = G * W;
  float* Qs = smem;                    // [Qn][DP]
  float* Os = Qs + Qn * DP;            // [Qn][DP]
  float* Ks = Os + Qn * DP;            // [kWinTile][DP]
  float* Vs = Ks + kWinTile * DP;      // [kWinTile][DP]
  float* Ls = Vs + kWinTile * DP;      // [kWinTile]

  const int unit = blockIdx.y, split = blockIdx.x;
  const int b = unit / H_kv, h = unit - b * H_kv;
  const int tid = threadIdx.x;
  int L = len[unit];
  if (L < 0 || L > T_cap) {
    if (split == 0 && tid == 0) set_flag(flags, KVS_FLAG_BAD_LENGTH);
    L = 0;
  }
  const int chunk = (L + nsplit - 1) / nsplit;
  const int t0 = split * chunk;
  const int t1 = min(L, t0 + chunk);

  load_queries_scaled<T, D>(Qw, Qs, DP, b, h, H_q, G, W, tid, kWinThreads);
  for (int idx = tid; idx < Qn * DP; idx += kWinThreads) Os[idx] = 0.f;

  const int q = tid;
  const bool active = q < Qn;
  const int pos = active ? L - W + (q % W) : -1;   // last position this query sees
  float m = -INFINITY, l = 0.f;
  const T* Kh = K + (size_t)unit * T_cap * D;
  const T* Vh = V + (size_t)unit * T_cap * D;
  const float* lnh = logn ? logn + (size_t)unit * T_cap : nullptr;

  for (int tb = t0; tb < t1; tb += kWinTile) {
    const int nt = min(kWinTile, t1 - tb);
    __syncthreads();
    for (int idx = tid; idx < kWinTile * VPR; idx += kWinThreads) {
      int r = idx / VPR, cv = idx - r * VPR;
      float fk[VN], fv[VN];
      if (r < nt) {
        load_vec(Kh + (size_t)(tb + r) * D + cv * VN, fk);
        load_vec(Vh + (size_t)(tb + r) * D + cv * VN, fv);
      } else {
#pragma unroll
        for (int e = 0; e < VN; ++e) { fk[e] = 0.f; fv[e] = 0.f; }
      }
#pragma unroll
      for (int e = 0; e < VN; ++e) {
        Ks[r * DP + cv * VN + e] = fk[e];
        Vs[r * DP + cv * VN + e] = fv[e];
      }
    }
    if (tid < kWinTile) Ls[tid] = (tid < nt && lnh) ? lnh[tb + tid] * kLog2e : 0.f;
    __syncthreads();
    if (active && pos >= tb) {
      float s[kWinTile];
#pragma unroll
      for (int i = 0; i < kWinTile; ++i) s[i] = 0.f;
      for (int c = 0; c < D; c += 4) {
        float4 qv = *reinterpret_cast<const float4*>(&Qs[q * DP + c]);
#pragma unroll
        for (int i = 0; i < kWinTile; ++i) {
          float4 kv = *reinterpret_cast<const float4*>(&Ks[i * DP + c]);
          s[i] = fmaf(qv.x, kv.x, s[i]);
          s[i] = fmaf(qv.y, kv.y, s[i]);
          s[i] = fmaf(qv.z, kv.z, s[i]);
          s[i] = fmaf(qv.w, kv.w, s[i]);
        }
      }
      float tmax = -INFINITY;
#pragma unroll
      for (int i = 0; i < kWinTile; ++i) {
        bool vis = (i < nt) && (tb + i <= pos);
        s[i] = vis ? s[i] + Ls[i] : -INFINITY;
        tmax = fmaxf(tmax, s[i]);
      }
      const float m_new = fmaxf(m, tmax);
      const float corr = exp2f(m - m_new);
      float psum = 0.f;
#pragma unroll
      for (int i = 0; i < kWinTile; ++i) {
        s[i] = exp2f(s[i] - m_new);
        psum += s[i];
      }
      l = l * corr + psum;
      for (int c = 0; c < D; c += 4) {
        float4 o = *reinterpret_cast<float4*>(&Os[q * DP + c]);
        o.x *= corr; o.y *= corr; o.z *= corr; o.w *= corr;
#pragma unroll
        for (int i = 0; i < kWinTile; ++i) {
          float4 vv = *reinterpret_cast<const float4*>(&Vs[i * DP + c]);
          o.x = fmaf(s[i], vv.x, o.x);
          o.y = fmaf(s[i], vv.y, o.y);
          o.z = fmaf(s[i], vv.z, o.z);
          o.w = fmaf(s[i], vv.w, o.w);
        }
        *reinterpret_cast<float4*>(&Os[q * DP + c]) = o;
      }
      m = m_new;
    }
  }
  __syncthreads();
  const size_t part = (size_t)unit * nsplit + split;
  if (active) {
    part_ml[(part * Qn + q) * 2 + 0] = m;
    part_ml[(part * Qn + q) * 2 + 1] = l;
  }
  float* po = part_o + part * Qn * D;
  for (int idx = tid; idx < Qn * D; idx += kWinThreads) {
    int qq = idx / D, c = idx - qq * D;
    po[idx] = Os[qq * DP + c];
  }
}

// Combine, with many CTAs (one CTA per head walking every partial of every query was
// latency-bound). window_combine_kernel: one CTA per block of kCombQ queries of a head;
// each warp takes queries in turn for (M, L), then every thread (one column) sums its
// column of o_q over the block's queries into one row of block sums. obar_kernel: per
// head, o_bar = (sum of the block rows, in order) / number of queries with a finite
// normaliser.
constexpr int kCombQ = 4;

template <int D>
__global__ void __launch_bounds__(D)
window_combine_kernel(const float* __restrict__ part_ml, const float* __restrict__ part_o,
                      int Qn, int nsplit, float* __restrict__ stats, float* __restrict__ osum,
                      int32_t* __restrict__ flags) {
  extern __shared__ __align__(16) float fac[];   // [kCombQ][nsplit]
  const int unit = blockIdx.y, qb = blockIdx.x, c = threadIdx.x;
  const int lane = c & 31, warp = c >> 5;
  const int q0 = qb * kCombQ, nq = min(kCombQ, Qn - q0);
  const float* ml = part_ml + (size_t)unit * nsplit * Qn * 2;
  for (int j = warp; j < nq; j += D / 32) {
    const int q = q0 + j;
    float M = -INFINITY;
    for (int s = lane; s < nsplit; s += 32) {
      const float ls = ml[((size_t)s * Qn + q) * 2 + 1];
      if (ls > 0.f) M = fmaxf(M, ml[((size_t)s * Qn + q) * 2]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Lsum = 0.f;
    if (M > -INFINITY)
      for (int s = lane; s < nsplit; s += 32) {
        const float ls = ml[((size_t)s * Qn + q) * 2 + 1];
        if (ls > 0.f) Lsum += ls * exp2f(ml[((size_t)s * Qn + q) * 2] - M);
      }
    Lsum = warp_sum(Lsum);
    const bool ok = Lsum > 0.f && isfinite(Lsum) && isfinite(M);
    const float inv = ok ? 1.f / Lsum : 0.f;
    for (int s = lane; s < nsplit; s += 32) {
      const float ls = ml[((size_t)s * Qn + q) * 2 + 1];
      fac[j * nsplit + s] = (ok && ls > 0.f) ? exp2f(ml[((size_t)s * Qn + q) * 2] - M) * inv : 0.f;
    }
    if (lane == 0) {
      stats[((size_t)unit * Qn + q) * 2 + 0] = M;
      stats[((size_t)unit * Qn + q) * 2 + 1] = ok ? Lsum : 0.f;
      if (!ok && M > -INFINITY) set_flag(flags, KVS_FLAG_NONFINITE_STATS);
    }
  }
  __syncthreads();
  float acc = 0.f;
  for (int j = 0; j < nq; ++j) {
    const float* po = part_o + ((size_t)unit * nsplit * Qn + q0 + j) * D + c;
    const float* f = fac + j * nsplit;
    float a4[4] = {0.f, 0.f, 0.f, 0.f};
    int s = 0;
    for (; s + 4 <= nsplit; s += 4) {
#pragma unroll
      for (int k = 0; k < 4; ++k) a4[k] = fmaf(f[s + k], po[(size_t)(s + k) * Qn * D], a4[k]);
    }
    for (; s < nsplit; ++s) a4[0] = fmaf(f[s], po[(size_t)s * Qn * D], a4[0]);
    acc += (a4[0] + a4[1]) + (a4[2] + a4[3]);
  }
  osum[((size_t)unit * 128 + qb) * D + c] = acc;
}

template <int D>
__global__ void __launch_bounds__(D)
obar_kernel(const float* __restrict__ stats, const float* __restrict__ osum, int Qn,
            float* __restrict__ obar) {
  __shared__ int s_valid;
  const int unit = blockIdx.x, c = threadIdx.x;
  if (c == 0) s_valid = 0;
  __syncthreads();
  int nv = 0;
  for (int q = c; q < Qn; q += D) nv += stats[((size_t)unit * Qn + q) * 2 + 1] > 0.f;
  if (nv) atomicAdd(&s_valid, nv);
  const int nb = (Qn + kCombQ - 1) / kCombQ;
  const float* col = osum + (size_t)unit * 128 * D + c;
  float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int b = 0;
  for (; b + 8 <= nb; b += 8) {
#pragma unroll
    for (int k = 0; k < 8; ++k) a8[k] += col[(size_t)(b + k) * D];
  }
  for (; b < nb; ++b) a8[b & 7] += col[(size_t)b * D];
  __syncthreads();
  const float t = ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
  obar[(size_t)unit * D + c] = s_valid > 0 ? t / (float)s_valid : 0.f;
}

template <typename T, int D>
__global__ void __launch_bounds__(kAlphaThreads)
alpha_bar_kernel(const T* __restrict__ K, const float* __restrict__ logn,
                 const int32_t* __restrict__ len, const T* __restrict__ Qw, int H_kv, int H_q,
                 int T_cap, int W, const float* __restrict__ stats, float* __restrict__ alpha) {
  extern __shared__ __align__(16) float asm_[];
  constexpr int DP = D + 4;
  constexpr int VN = Vec16<T>::n;
  constexpr int VPR = D / VN;
  constexpr int NG = kAlphaThreads / kAlphaTokens;   // query groups
  const int G = H_q / H_kv;
  const int Qn = G * W;
  float* Qs = asm_;                         // [Qn][DP]
  float* Ks = Qs + Qn * DP;                 // [kAlphaTokens][DP]
  float* Mq = Ks + kAlphaTokens * DP;       // [Qn]
  float* Il = Mq + Qn;                      // [Qn]
  float* Ls = Il + Qn;                      // [kAlphaTokens]
  float* red = Ls + kAlphaTokens;           // [kAlphaThreads]
  __shared__ int s_valid;

  const int unit = blockIdx.y;
  const int b = unit / H_kv, h = unit - b * H_kv;
  const int tid = threadIdx.x;
  const int L = len[unit];
  const int tb = blockIdx.x * kAlphaTokens;
  if (L < 0 || L > T_cap || tb >= L) return;
  if (tid == 0) s_valid = 0;
  load_queries_scaled<T, D>(Qw, Qs, DP, b, h, H_q, G, W, tid, kAlphaThreads);
  const T* Kh = K + (size_t)unit * T_cap * D;
  const int nt = min(kAlphaTokens, L - tb);
  for (int idx = tid; idx < kAlphaTokens * VPR; idx += kAlphaThreads) {
    int r = idx / VPR, cv = idx - r * VPR;
    float fk[VN];
    if (r < nt) {
      load_vec(Kh + (size_t)(tb + r) * D + cv * VN, fk);
    } else {
#pragma unroll
      for (int e = 0; e < VN; ++e) fk[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < VN; ++e) Ks[r * DP + cv * VN + e] = fk[e];
  }
  if (tid < kAlphaTokens)
    Ls[tid] = (tid < nt && logn) ? logn[(size_t)unit * T_cap + tb + tid] * kLog2e : 0.f;
  __syncthreads();
  for (int q = tid; q < Qn; q += kAlphaThreads) {
    float M = stats[((size_t)unit * Qn + q) * 2 + 0];
    float Ln = stats[((size_t)unit * Qn + q) * 2 + 1];
    bool ok = Ln > 0.f && isfinite(Ln) && isfinite(M);
    Mq[q] = ok ? M : 0.f;
    Il[q] = ok ? 1.f / Ln : 0.f;
    if (ok) atomicAdd(&s_valid, 1);
  }
  __syncthreads();
  const int tl = tid % kAlphaTokens, grp = tid / kAlphaTokens;
  const int t = tb + tl;
  float acc = 0.f;
  for (int q = grp; q < Qn; q += NG) {
    const float il = Il[q];
    if (il == 0.f) continue;
    const int pos = L - W + (q % W);
    if (t > pos) continue;
    float s = 0.f;
    for (int c = 0; c < D; c += 4) {
      float4 qv = *reinterpret_cast<const float4*>(&Qs[q * DP + c]);
      float4 kv = *reinterpret_cast<const float4*>(&Ks[tl * DP + c]);
      s = fmaf(qv.x, kv.x, s);
      s = fmaf(qv.y, kv.y, s);
      s = fmaf(qv.z, kv.z, s);
      s = fmaf(qv.w, kv.w, s);
    }
    acc = fmaf(exp2f(s + Ls[tl] - Mq[q]), il, acc);
  }
  red[tid] = acc;
  __syncthreads();
  if (grp == 0 && tl < nt) {
    float tot = 0.f;
#pragma unroll
    for (int g2 = 0; g2 < NG; ++g2) tot += red[g2 * kAlphaTokens + tl];
    alpha[(size_t)unit * T_cap + t] = s_valid > 0 ? tot / (float)s_valid : 0.f;
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------

template <typename T, int D>
static cudaError_t launch_window_stats_t(const kvs_cache_desc& d, const void* K, const void* V,
                                         const float* logn, const int32_t* len, const void* Qw,
                                         int W, const ScoreLayout& Ly, char* ws,
                                         cudaStream_t st) {
  const int units = d.B * d.H_kv;
  const int Qn = Ly.Qn;
  int32_t* flags = reinterpret_cast<int32_t*>(ws);
  float* part_ml = reinterpret_cast<float*>(ws + Ly.part_ml);
  float* part_o = reinterpret_cast<float*>(ws + Ly.part_o);
  float* stats = reinterpret_cast<float*>(ws + Ly.stats);
  float* obar = reinterpret_cast<float*>(ws + Ly.obar);
  float* alpha = reinterpret_cast<float*>(ws + Ly.alpha);
  constexpr int DP = D + 4;

  size_t sm1 = (size_t)(2 * Qn * DP + 2 * kWinTile * DP + kWinTile) * sizeof(float);
  auto k1 = window_partial_kernel<T, D>;
  if (!ensure_smem_attr((const void*)k1, sm1)) return cudaErrorInvalidValue;
  k1<<<dim3(Ly.nsplit, units), kWinThreads, sm1, st>>>(
      (const T*)K, (const T*)V, logn, len, (const T*)Qw, d.H_kv, d.H_q, d.T_cap, W, Ly.nsplit,
      part_ml, part_o, flags);

  // block sums of o_q in the fp32 window-output rows (ceil(Qn / kCombQ) <= 128 rows a head)
  float* osum = reinterpret_cast<float*>(ws + Ly.oq);
  size_t sm2 = (size_t)kCombQ * Ly.nsplit * sizeof(float);
  auto k2 = window_combine_kernel<D>;
  if (!ensure_smem_attr((const void*)k2, sm2)) return cudaErrorInvalidValue;
  k2<<<dim3((Qn + kCombQ - 1) / kCombQ, units), D, sm2, st>>>(part_ml, part_o, Qn, Ly.nsplit,
                                                               stats, osum, flags);
  obar_kernel<D><<<units, D, 0, st>>>(stats, osum, Qn, obar);

  size_t sm3 = (size_t)(Qn * DP + kAlphaTokens * DP + 2 * Qn + kAlphaTokens + kAlphaThreads) *
               sizeof(float);
  auto k3 = alpha_bar_kernel<T, D>;
  if (!ensure_smem_attr((const void*)k3, sm3)) return cudaErrorInvalidValue;
  dim3 g3((d.T_cap + kAlphaTokens - 1) / kAlphaTokens, units);
  k3<<<g3, kAlphaThreads, sm3, st>>>((const T*)K, logn, len, (const T*)Qw, d.H_kv, d.H_q,
                                     d.T_cap, W, stats, alpha);
  count_launches(4);
  return cudaGetLastError();
}

cudaError_t launch_window_stats(const kvs_cache_desc& d, const void* K, const void* V,
                                const float* logn, const int32_t* len, const void* Qw, int W,
                                const ScoreLayout& Ly, char* ws, cudaStream_t st) {
  if (d.dtype == KVS_BF16) {
    if (d.d == 128) return launch_window_stats_t<bf16, 128>(d, K, V, logn, len, Qw, W, Ly, ws, st);
    return launch_window_stats_t<bf16, 64>(d, K, V, logn, len, Qw, W, Ly, ws, st);
  }
  if (d.d == 128) return launch_window_stats_t<float, 128>(d, K, V, logn, len, Qw, W, Ly, ws, st);
  return launch_window_stats_t<float, 64>(d, K, V, logn, len, Qw, W, Ly, ws, st);
}

}  // namespace kvs
