// Pair norms, merge weight and score for every candidate pair of every KV head.
//
// KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程"),
// §数学主线四: c11 = a_m (1 - 2 a_m)(v_m - o), c22 likewise, c12 = -a_m a_m1 (v_m + v_m1 - 2o);
// the forward-only merged key k* = [(|c11| - |c12|) k_m + (|c22| - |c12|) k_m1] /
// (|c11| - 2|c12| + |c22|). §数学主线二: the objective whose minimum value ranks
// the pairs; the diagonal form (ablation) drops its coupling term, |c12| = 0. Window-mean attention a and o_bar come from the window-statistics pass.
//
// One pair is handled by LPR lanes (LPR = 16-byte vectors per row); each lane holds
// a 16-byte slice of k_a, k_b, v_a, v_b and the matching slice of o_bar; the four
// squared norms are reduced with xor shuffles inside the lane group.
#include "kvs_common.cuh"
#include "kvs_kernels.h"

namespace kvs {

constexpr int kScoreThreads = 256;
constexpr int kScoreIters = 4;

template <typename T, int D>
__global__ void __launch_bounds__(kScoreThreads)
pair_score_kernel(const T* __restrict__ K, const T* __restrict__ V,
                  const float* __restrict__ alpha, const float* __restrict__ obar,
                  const int32_t* __restrict__ len, const int32_t* __restrict__ cand_begin,
                  int n_recent, int T_cap, int form, float* __restrict__ score,
                  float* __restrict__ w_b) {
  constexpr int VN = Vec16<T>::n;
  constexpr int LPR = D / VN;                 // lanes per row: 8, 16 or 32
  constexpr int PPI = 32 / LPR;               // pairs per warp per iteration
  constexpr int WARPS = kScoreThreads / 32;
  constexpr int PAIRS_PER_CTA = WARPS * PPI * kScoreIters;

  const int unit = blockIdx.y;
  const int L = len[unit];
  const int c0 = cand_begin[unit];
  if (L < 0 || L > T_cap || c0 < 0) return;
  const int span = L - n_recent - c0;
  const int P = span > 0 ? span / 2 : 0;
  const int p_cta = blockIdx.x * PAIRS_PER_CTA;
  if (p_cta >= P) return;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int li = lane % LPR, gi = lane / LPR;
  float ob[VN];
#pragma unroll
  for (int e = 0; e < VN; ++e) ob[e] = obar[(size_t)unit * D + li * VN + e];

  const T* Kh = K + (size_t)unit * T_cap * D;
  const T* Vh = V + (size_t)unit * T_cap * D;
  const float* ah = alpha + (size_t)unit * T_cap;
  const size_t pbase = (size_t)unit * (T_cap / 2);

#pragma unroll 1
  for (int it = 0; it < kScoreIters; ++it) {
    const int p = p_cta + (it * WARPS + warp) * PPI + gi;
    const bool valid = p < P;
    const int a = c0 + 2 * p;
    float ka[VN], kb[VN], va[VN], vb[VN];
    if (valid) {
      load_vec_cs(Kh + (size_t)a * D + li * VN, ka);
      load_vec_cs(Kh + (size_t)(a + 1) * D + li * VN, kb);
      load_vec_cs(Vh + (size_t)a * D + li * VN, va);
      load_vec_cs(Vh + (size_t)(a + 1) * D + li * VN, vb);
    } else {
#pragma unroll
      for (int e = 0; e < VN; ++e) { ka[e] = kb[e] = va[e] = vb[e] = 0.f; }
    }
    float dd = 0.f, ea = 0.f, eb = 0.f, ec = 0.f;
#pragma unroll
    for (int e = 0; e < VN; ++e) {
      const float dk = kb[e] - ka[e];
      const float ra = va[e] - ob[e];
      const float rb = vb[e] - ob[e];
      const float rc = ra + rb;
      dd = fmaf(dk, dk, dd);
      ea = fmaf(ra, ra, ea);
      eb = fmaf(rb, rb, eb);
      ec = fmaf(rc, rc, ec);
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) {
      dd += __shfl_xor_sync(0xffffffffu, dd, o);
      ea += __shfl_xor_sync(0xffffffffu, ea, o);
      eb += __shfl_xor_sync(0xffffffffu, eb, o);
      ec += __shfl_xor_sync(0xffffffffu, ec, o);
    }
    if (valid && li == 0) {
      const float aa = ah[a], ab = ah[a + 1];
      const float n11 = fabsf(aa * (1.f - 2.f * aa)) * sqrtf(ea);
      const float n22 = fabsf(ab * (1.f - 2.f * ab)) * sqrtf(eb);
      // the diagonal form drops the coupling term (ablation): N12 = 0
      const float n12 = form == KVS_FORM_DIAGONAL ? 0.f : aa * ab * sqrtf(ec);
      const float den = n11 - 2.f * n12 + n22;
      const bool ok = isfinite(n11) && isfinite(n12) && isfinite(n22) && isfinite(den) &&
                      den > 1e-6f * (n11 + n22);
      float w, s;
      if (ok) {
        w = (n22 - n12) / den;
        s = dd * (n11 * n22 - n12 * n12) / den;
      } else {
        w = 0.5f;
        s = dd * (n11 + 2.f * n12 + n22) * 0.25f;
      }
      score[pbase + p] = s;
      w_b[pbase + p] = w;
    }
  }
}

template <typename T, int D>
static cudaError_t launch_pair_score_t(const kvs_cache_desc& d, const void* K, const void* V,
                                       const int32_t* len, const int32_t* cand_begin,
                                       int n_recent, int form, const ScoreLayout& Ly, char* ws,
                                       float* score, float* w_b, cudaStream_t st) {
  constexpr int VN = Vec16<T>::n;
  constexpr int LPR = D / VN;
  constexpr int PAIRS_PER_CTA = (kScoreThreads / 32) * (32 / LPR) * kScoreIters;
  const int units = d.B * d.H_kv;
  const int pmax = d.T_cap / 2;
  dim3 grid((pmax + PAIRS_PER_CTA - 1) / PAIRS_PER_CTA, units);
  pair_score_kernel<T, D><<<grid, kScoreThreads, 0, st>>>(
      (const T*)K, (const T*)V, reinterpret_cast<const float*>(ws + Ly.alpha),
      reinterpret_cast<const float*>(ws + Ly.obar), len, cand_begin, n_recent, d.T_cap, form,
      score, w_b);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_pair_score(const kvs_cache_desc& d, const void* K, const void* V,
                              const int32_t* len, const int32_t* cand_begin, int n_recent,
                              int form, const ScoreLayout& Ly, char* ws, float* score,
                              float* w_b, cudaStream_t st) {
  if (d.dtype == KVS_BF16) {
    if (d.d == 128)
      return launch_pair_score_t<bf16, 128>(d, K, V, len, cand_begin, n_recent, form, Ly, ws, score, w_b, st);
    return launch_pair_score_t<bf16, 64>(d, K, V, len, cand_begin, n_recent, form, Ly, ws, score, w_b, st);
  }
  if (d.d == 128)
    return launch_pair_score_t<float, 128>(d, K, V, len, cand_begin, n_recent, form, Ly, ws, score, w_b, st);
  return launch_pair_score_t<float, 64>(d, K, V, len, cand_begin, n_recent, form, Ly, ws, score, w_b, st);
}

}  // namespace kvs
