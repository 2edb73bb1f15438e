// Pair selection to the budget, merge and compaction of one round.
//
// Merge rule: KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程"),
// §数学主线四 forward-only merged Key, k* = k_a + w_b (k_b - k_a). Values are kept
// (核心判断: merge homogeneous Keys, preserve heterogeneous Values): a merged row stores
// the count-weighted mean value and log(count) as a logit bias, which is exactly
// attention over the original rows sharing k*.
//
// select_kernel (one CTA per selection unit):
//   R = min(P, max(0, len - target)); the threshold key is the R-th smallest
//   (score_key, index), found by a radix select (a 12-bit histogram pass over the
//   scores, then the threshold bin's keys resolved in shared memory); then per block of
//   kMergePairsPerBlock pairs the counts of keys below / equal to the threshold,
//   exclusive-scanned in unit order (h, p), give every merge CTA its offsets.
// merge_kernel (out-of-place): one CTA per (head, pair block) plus copy CTAs for
//   the protected prefix and suffix; a block-level ballot scan gives each pair's
//   output row; rows move as 16-byte vectors, merged rows are computed in fp32.
// merge_inplace_kernel: one CTA per head walks the span in order, staging each
//   chunk in shared memory (a ring of stages, the next chunk's copies in flight)
//   before writing it to lower (or equal) rows.
#include "kvs_common.cuh"
#include "kvs_kernels.h"
#include "ptx.cuh"

namespace kvs {

constexpr int kSelThreads = 1024;
constexpr int kSelCand = 6144;   // threshold-bin keys resolved in shared memory
constexpr int kMergeThreads = 256;
constexpr int kCopyRows = 256;
// Pairs staged per in-place step: 32 for rows up to 256 bytes, 16 for 512-byte rows
// (one warp plans a step; two 32 KB stages of K and V rows).
template <typename T, int D>
constexpr int inplace_chunk() { return D * (int)sizeof(T) <= 256 ? 32 : 16; }

__device__ __forceinline__ int head_pairs(int L, int c0, int n_recent) {
  int s = L - n_recent - c0;
  return s > 0 ? s / 2 : 0;
}

// Block-wide exclusive scan of one int per thread (blockDim = kSelThreads).
__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_tot[lane] = wi - w;          // exclusive warp offsets
    if (lane == 31) warp_tot[32] = wi;
  }
  __syncthreads();
  int r = warp_tot[warp] + incl - v;
  total = warp_tot[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kSelThreads, 1)
select_kernel(const float* __restrict__ score, const int32_t* __restrict__ len,
              const int32_t* __restrict__ cand_begin, int n_recent,
              const int32_t* __restrict__ target, int scope, int H_kv, int T_cap, int nblk,
              SelUnit* __restrict__ sel, HeadInfo* __restrict__ hinfo, int2* __restrict__ blk,
              int32_t* __restrict__ flags) {
  // launched with programmatic stream serialisation: wait for the preceding grid (and its
  // memory) before any access, then let the next grid be scheduled
  griddep_wait();
  griddep_launch_dependents();
  __shared__ int hist[4096];
  __shared__ uint32_t cand[kSelCand];
  __shared__ int warp_tot[33];
  __shared__ int s_digit, s_before, s_R, s_P, s_bad, s_ncand;
  const int u = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int nh = scope == KVS_SCOPE_POOLED ? H_kv : 1;
  const int h_first = scope == KVS_SCOPE_POOLED ? u * H_kv : u;
  const int pstride = T_cap / 2;

  if (tid == 0) {
    long long tot_len = 0, tot_P = 0, min_len = 0;
    int bad = 0;
    for (int i = 0; i < nh; ++i) {
      const int hh = h_first + i;
      const int L = len[hh], c0 = cand_begin[hh];
      if (L < 0 || L > T_cap || c0 < 0) bad = 1;
      const int P = bad ? 0 : head_pairs(L, c0, n_recent);
      hinfo[hh].len_in = L;
      hinfo[hh].P = P;
      hinfo[hh].c0 = c0;
      tot_len += L;
      tot_P += P;
      // repeated rounds shrink a span of S candidate rows to one row (S >= 1), so the
      // shortest length this head can reach is L - S + min(S, 1)
      const long long S = bad ? 0 : max(0, L - n_recent - c0);
      min_len += L - S + (S > 0 ? 1 : 0);
    }
    if (!bad && (long long)target[u] < min_len) set_flag(flags, KVS_FLAG_BUDGET);
    long long want = tot_len - (long long)target[u];
    if (want < 0) want = 0;
    if (want > tot_P) want = tot_P;
    s_R = bad ? 0 : (int)want;
    s_P = (int)tot_P;
    s_bad = bad;
    if (bad) {
      set_flag(flags, KVS_FLAG_BAD_LENGTH);
      for (int i = 0; i < nh; ++i) hinfo[h_first + i].len_in = -1;
    }
  }
  __syncthreads();
  if (s_bad) return;
  const int R = s_R, Ptot = s_P;

  uint32_t thr;
  int need_eq;
  if (R == 0) {
    thr = 0u;
    need_eq = 0;
  } else if (R == Ptot) {
    thr = 0xffffffffu;
    need_eq = 0;
  } else {
    // Radix select of the R-th smallest key: a 12-bit histogram of every key, then the
    // keys of the threshold's bin are gathered into shared memory (when they fit) and
    // their remaining 20 bits are resolved there in two 10-bit passes; otherwise the
    // remaining bits take three more passes over the scores (8, 8 and 4 bits).
    uint32_t prefix = 0u, pmask = 0u;
    int rank = R;   // 1-based rank of the threshold among the unit's keys
    auto global_pass = [&](int shift, int bits) {
      const int nb = 1 << bits;
      for (int i = tid; i < nb; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int i = 0; i < nh; ++i) {
        const int hh = h_first + i;
        const int P = hinfo[hh].P;
        const float* sc = score + (size_t)hh * pstride;
        // eight independent loads per thread are in flight before any is used
        constexpr int kBatch = 8;
        for (int p0 = 0; p0 < P; p0 += kSelThreads * kBatch) {
          float v[kBatch];
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            const int p = p0 + k * kSelThreads + tid;
            v[k] = p < P ? sc[p] : 0.f;
          }
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            const int p = p0 + k * kSelThreads + tid;
            const bool in = p < P;
            const uint32_t key = in ? score_key(v[k]) : 0u;
            const bool match = in && ((key & pmask) == prefix);
            const unsigned dg = (key >> shift) & (unsigned)(nb - 1);
            // aggregate equal digits inside the warp before the shared atomic
            const unsigned peers = __match_any_sync(0xffffffffu, match ? dg : 0x10000u + lane);
            if (match && (__ffs(peers) - 1) == lane) atomicAdd(&hist[dg], __popc(peers));
          }
        }
      }
      __syncthreads();
    };
    // the digit whose bin holds rank `rank` among nb bins; updates prefix, pmask, rank
    auto pick = [&](int shift, int bits) {
      const int nb = 1 << bits;
      const int per = nb > kSelThreads ? nb / kSelThreads : 1;
      int sum = 0;
      if (tid * per < nb)
        for (int k = 0; k < per; ++k) sum += hist[tid * per + k];
      int total;
      const int excl = block_excl_scan(sum, warp_tot, total);
      if (tid * per < nb && excl < rank && rank <= excl + sum) {
        int acc = excl;
        for (int k = 0; k < per; ++k) {
          const int c = hist[tid * per + k];
          if (rank <= acc + c) { s_digit = tid * per + k; s_before = acc; break; }
          acc += c;
        }
      }
      __syncthreads();
      prefix |= (uint32_t)s_digit << shift;
      pmask |= (uint32_t)(nb - 1) << shift;
      rank -= s_before;
      const int in_bin = hist[s_digit];
      __syncthreads();
      return in_bin;
    };
    global_pass(20, 12);
    const int in_bin = pick(20, 12);
    if (in_bin <= kSelCand) {
      // gather the bin's keys
      if (tid == 0) s_ncand = 0;
      __syncthreads();
      for (int i = 0; i < nh; ++i) {
        const int hh = h_first + i;
        const int P = hinfo[hh].P;
        const float* sc = score + (size_t)hh * pstride;
        // eight independent loads per thread in flight, as in the histogram pass
        constexpr int kBatch = 8;
        for (int p0 = 0; p0 < P; p0 += kSelThreads * kBatch) {
          float v[kBatch];
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            const int p = p0 + k * kSelThreads + tid;
            v[k] = p < P ? sc[p] : 0.f;
          }
#pragma unroll
          for (int k = 0; k < kBatch; ++k) {
            const int p = p0 + k * kSelThreads + tid;
            const uint32_t key = p < P ? score_key(v[k]) : 0u;
            const bool match = p < P && (key & pmask) == prefix;
            const unsigned ball = __ballot_sync(0xffffffffu, match);
            int base = 0;
            if (lane == 0 && ball) base = atomicAdd(&s_ncand, __popc(ball));
            base = __shfl_sync(0xffffffffu, base, 0);
            if (match) cand[base + __popc(ball & ((1u << lane) - 1u))] = key;
          }
        }
      }
      __syncthreads();
      const int nc = s_ncand;
      for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
        for (int i = tid; i < 1024; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < nc; i += kSelThreads) {
          const uint32_t key = cand[i];
          if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 1023u], 1);
        }
        __syncthreads();
        pick(shift, 10);
      }
    } else {
      global_pass(12, 8);
      pick(12, 8);
      global_pass(4, 8);
      pick(4, 8);
      global_pass(0, 4);
      pick(0, 4);
    }
    thr = prefix;
    need_eq = rank;
  }

  // Per block counts of keys below / equal to the threshold, (h, block) order.
  const int nent = nh * nblk;
  if (R == 0 || R == Ptot) {
    // nothing or everything is merged: every count follows from P alone, no score is read
    for (int e = tid; e < nent; e += kSelThreads) {
      const int i = e / nblk, j = e - i * nblk;
      const int hh = h_first + i;
      const int P = hinfo[hh].P;
      const int in_blk = max(0, min(kMergePairsPerBlock, P - j * kMergePairsPerBlock));
      blk[(size_t)hh * nblk + j] = make_int2(R == 0 ? 0 : in_blk, 0);
    }
    __syncthreads();
  } else {
    for (int e0 = 0; e0 < nent; e0 += kSelThreads / 32) {
      const int e = e0 + warp;
      if (e < nent) {
        const int i = e / nblk, j = e - i * nblk;
        const int hh = h_first + i;
        const int P = hinfo[hh].P;
        const float* sc = score + (size_t)hh * pstride;
        int lt = 0, eq = 0;
        float v[kMergePairsPerBlock / 32];
#pragma unroll
        for (int k = 0; k < kMergePairsPerBlock / 32; ++k) {
          const int p = j * kMergePairsPerBlock + k * 32 + lane;
          v[k] = p < P ? sc[p] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < kMergePairsPerBlock / 32; ++k) {
          const int p = j * kMergePairsPerBlock + k * 32 + lane;
          const bool in = p < P;
          const uint32_t key = in ? score_key(v[k]) : 0u;
          lt += __popc(__ballot_sync(0xffffffffu, in && key < thr));
          eq += __popc(__ballot_sync(0xffffffffu, in && key == thr));
        }
        if (lane == 0) blk[(size_t)hh * nblk + j] = make_int2(lt, eq);
      }
    }
    __syncthreads();
  }
  // Unit-wide exclusive scans of both counts.
  int carry_lt = 0, carry_eq = 0;
  for (int e0 = 0; e0 < nent; e0 += kSelThreads) {
    const int e = e0 + tid;
    const int i = e / nblk, j = e - i * nblk;
    int2 v = make_int2(0, 0);
    if (e < nent) v = blk[(size_t)(h_first + i) * nblk + j];
    int tl, te;
    const int xl = block_excl_scan(v.x, warp_tot, tl);
    const int xe = block_excl_scan(v.y, warp_tot, te);
    if (e < nent) blk[(size_t)(h_first + i) * nblk + j] = make_int2(carry_lt + xl, carry_eq + xe);
    carry_lt += tl;
    carry_eq += te;
  }
  __syncthreads();
  // Per head: scan values at its first block and its merged-pair count.
  if (tid < nh) {
    const int hh = h_first + tid;
    const int2 first = blk[(size_t)hh * nblk];
    const int2 next = (tid + 1 < nh) ? blk[(size_t)(hh + 1) * nblk] : make_int2(carry_lt, carry_eq);
    const int lt_h = next.x - first.x;
    const int eq_sel = min(need_eq, next.y) - min(need_eq, first.y);
    hinfo[hh].lt0 = first.x;
    hinfo[hh].eq0 = first.y;
    hinfo[hh].R = lt_h + eq_sel;
  }
  if (tid == 0) {
    sel[u].thr_key = thr;
    sel[u].need_eq = need_eq;
    sel[u].R = R;
    sel[u].P = Ptot;
  }
}

// Copy `rows` consecutive rows of K, V (and logn) from row `src` to row `dst`.
template <typename T, int D>
__device__ __forceinline__ void copy_rows(const T* __restrict__ Kh, const T* __restrict__ Vh,
                                          const float* __restrict__ lnh, T* __restrict__ Ko,
                                          T* __restrict__ Vo, float* __restrict__ lno, int src,
                                          int dst, int rows) {
  constexpr int VPR = D * (int)sizeof(T) / 16;
  const int nvec = rows * VPR;
  for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
    const int r = i / VPR, c = i - r * VPR;
    const size_t so = ((size_t)(src + r) * D) * sizeof(T) + (size_t)c * 16;
    const size_t dof = ((size_t)(dst + r) * D) * sizeof(T) + (size_t)c * 16;
    store_raw(reinterpret_cast<char*>(Ko) + dof, load_raw(reinterpret_cast<const char*>(Kh) + so));
    store_raw(reinterpret_cast<char*>(Vo) + dof, load_raw(reinterpret_cast<const char*>(Vh) + so));
  }
  for (int r = threadIdx.x; r < rows; r += blockDim.x) lno[dst + r] = lnh ? lnh[src + r] : 0.f;
}

// Selection flags and output rows of up to 128 consecutive pairs (threads < 128).
struct PairPlan {
  int off;
  bool sel;
};

__device__ __forceinline__ PairPlan plan_pair(int t, int pbase, int P, const float* sc,
                                              const SelUnit& su, int lt_before, int eq_unit,
                                              const HeadInfo& hi, int* s_cnt) {
  // s_cnt: 8 ints of shared scratch (4 warps x {lt, eq}); all 128 threads call this.
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int p = pbase + t;
  const bool in = p < P;
  const uint32_t key = in ? score_key(sc[p]) : 0xffffffffu;
  const bool lt = in && key < su.thr_key;
  const bool eq = in && key == su.thr_key;
  const unsigned blt = __ballot_sync(0xffffffffu, lt);
  const unsigned beq = __ballot_sync(0xffffffffu, eq);
  if (lane == 0) { s_cnt[warp * 2] = __popc(blt); s_cnt[warp * 2 + 1] = __popc(beq); }
  asm volatile("bar.sync 1, 128;");
  int wl = 0, we = 0;
  for (int w = 0; w < warp; ++w) { wl += s_cnt[w * 2]; we += s_cnt[w * 2 + 1]; }
  const unsigned lower = (1u << lane) - 1u;
  const int lt_rank = wl + __popc(blt & lower);
  const int eq_rank = we + __popc(beq & lower);
  const int eqg = eq_unit + eq_rank;
  PairPlan pp;
  pp.sel = lt || (eq && eqg < su.need_eq);
  const int sel_before = lt_before + lt_rank + min(su.need_eq, eqg) - min(su.need_eq, hi.eq0);
  pp.off = hi.c0 + 2 * p - sel_before;
  asm volatile("bar.sync 1, 128;");
  return pp;
}

template <typename T, int D>
__global__ void __launch_bounds__(kMergeThreads)
merge_kernel(const T* __restrict__ K, const T* __restrict__ V, const float* __restrict__ logn,
             const float* __restrict__ score, const float* __restrict__ w_b, int scope, int H_kv,
             int T_cap, int T_cap_out, int nblk, const SelUnit* __restrict__ sel,
             const HeadInfo* __restrict__ hinfo, const int2* __restrict__ blk,
             T* __restrict__ K_out, T* __restrict__ V_out, float* __restrict__ logn_out,
             int32_t* __restrict__ len_out, uint8_t* __restrict__ dbg_sel,
             int32_t* __restrict__ dbg_off, float* __restrict__ dbg_km,
             int32_t* __restrict__ flags) {
  // launched with programmatic stream serialisation: wait for the preceding grid (and its
  // memory) before any access, then let the next grid be scheduled
  griddep_wait();
  griddep_launch_dependents();
  constexpr int MB = kMergePairsPerBlock;
  constexpr int VN = Vec16<T>::n;
  constexpr int LPR = D / VN;
  __shared__ int s_off[MB];
  __shared__ unsigned char s_sel[MB];
  __shared__ float s_w[MB];
  __shared__ int s_cnt[8];

  const int head = blockIdx.y;
  const HeadInfo hi = hinfo[head];
  if (hi.len_in < 0) return;
  const int u = scope == KVS_SCOPE_POOLED ? head / H_kv : head;
  const SelUnit su = sel[u];
  const int L = hi.len_in, P = hi.P, R = hi.R, c0 = hi.c0;
  const int L_out = L - R;
  if (L_out > T_cap_out) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_flag(flags, KVS_FLAG_OUT_CAPACITY);
    return;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) len_out[head] = L_out;

  const T* Kh = K + (size_t)head * T_cap * D;
  const T* Vh = V + (size_t)head * T_cap * D;
  const float* lnh = logn ? logn + (size_t)head * T_cap : nullptr;
  T* Ko = K_out + (size_t)head * T_cap_out * D;
  T* Vo = V_out + (size_t)head * T_cap_out * D;
  float* lno = logn_out + (size_t)head * T_cap_out;
  const int x = blockIdx.x;

  if (x >= nblk) {   // protected rows: prefix [0, c0) in place, suffix shifted down by R
    const int ct = x - nblk;
    const int r0 = ct * kCopyRows;
    const int pre = min(c0, L);     // a span start past the end leaves only [0, L)
    if (r0 < pre) copy_rows<T, D>(Kh, Vh, lnh, Ko, Vo, lno, r0, r0, min(kCopyRows, pre - r0));
    const int s0 = c0 + 2 * P + r0;
    if (s0 < L) copy_rows<T, D>(Kh, Vh, lnh, Ko, Vo, lno, s0, s0 - R, min(kCopyRows, L - s0));
    return;
  }

  const int pbase = x * MB;
  if (pbase >= P) return;
  const float* sc = score + (size_t)head * (T_cap / 2);
  const float* wb = w_b + (size_t)head * (T_cap / 2);
  if (threadIdx.x < MB) {
    const int2 bs = blk[(size_t)head * nblk + x];
    const int t = threadIdx.x;
    const PairPlan pp = plan_pair(t, pbase, P, sc, su, bs.x - hi.lt0, bs.y, hi, s_cnt);
    s_off[t] = pp.off;
    s_sel[t] = pp.sel ? 1 : 0;
    const int p = pbase + t;
    s_w[t] = (p < P) ? wb[p] : 0.f;
    if (p < P) {
      if (dbg_sel) dbg_sel[(size_t)head * (T_cap / 2) + p] = pp.sel ? 1 : 0;
      if (dbg_off) dbg_off[(size_t)head * (T_cap / 2) + p] = pp.off;
    }
  }
  __syncthreads();

  const int nvalid = min(MB, P - pbase);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int WARPS = kMergeThreads / 32;
  if constexpr (LPR <= 16) {
    // LPR lanes per pair, each holding the same 16-byte slice of both rows of its pair (no
    // exchange between lanes; every lane of a merged pair computes its slice)
    constexpr int PPI = 32 / LPR;                   // pairs per warp iteration
    const int slot = lane / LPR, c = lane % LPR;
    // U warp iterations per batch: every load of the batch is issued before the first is
    // used, so that a warp keeps several rows' bytes in flight
    constexpr int U = 2;
    auto pair_rows = [&](int t, const uint4& ka_r, const uint4& kb_r, const uint4& va_r,
                         const uint4& vb_r, float la, float lb) {
      if (t >= nvalid) return;
      const int p = pbase + t;
      const int off = s_off[t];
      if (s_sel[t]) {
        float ka[VN], kb[VN], va[VN], vb[VN], ko[VN], vo[VN];
        load_vec(reinterpret_cast<const T*>(&ka_r), ka);
        load_vec(reinterpret_cast<const T*>(&kb_r), kb);
        load_vec(reinterpret_cast<const T*>(&va_r), va);
        load_vec(reinterpret_cast<const T*>(&vb_r), vb);
        const float w = s_w[t];
        const float na = expf(la), nb = expf(lb);
        const float inv = 1.f / (na + nb);
#pragma unroll
        for (int e = 0; e < VN; ++e) {
          ko[e] = fmaf(w, kb[e] - ka[e], ka[e]);
          vo[e] = (na * va[e] + nb * vb[e]) * inv;
        }
        store_vec(Ko + (size_t)off * D + c * VN, ko);
        store_vec(Vo + (size_t)off * D + c * VN, vo);
        if (c == 0) lno[off] = logf(na + nb);
        if (dbg_km) {
          float* dk = dbg_km + ((size_t)head * (T_cap / 2) + p) * D + c * VN;
#pragma unroll
          for (int e = 0; e < VN; e += 4) *reinterpret_cast<float4*>(dk + e) = make_float4(ko[e], ko[e + 1], ko[e + 2], ko[e + 3]);
        }
      } else {
        store_raw(Ko + (size_t)off * D + c * VN, ka_r);
        store_raw(Ko + (size_t)(off + 1) * D + c * VN, kb_r);
        store_raw(Vo + (size_t)off * D + c * VN, va_r);
        store_raw(Vo + (size_t)(off + 1) * D + c * VN, vb_r);
        if (c == 0) {
          lno[off] = la;
          lno[off + 1] = lb;
        }
      }
    };
    for (int base0 = warp * PPI; base0 < nvalid; base0 += WARPS * PPI * U) {
      uint4 kas[U], kbs[U], vas[U], vbs[U];
      float las[U], lbs[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = base0 + u * WARPS * PPI + slot;
        kas[u] = kbs[u] = vas[u] = vbs[u] = make_uint4(0, 0, 0, 0);
        las[u] = lbs[u] = 0.f;
        if (t < nvalid) {
          const int row = c0 + 2 * (pbase + t);
          kas[u] = load_raw(Kh + (size_t)row * D + c * VN);
          kbs[u] = load_raw(Kh + (size_t)(row + 1) * D + c * VN);
          vas[u] = load_raw(Vh + (size_t)row * D + c * VN);
          vbs[u] = load_raw(Vh + (size_t)(row + 1) * D + c * VN);
          if (lnh) {
            las[u] = lnh[row];
            lbs[u] = lnh[row + 1];
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        pair_rows(base0 + u * WARPS * PPI + slot, kas[u], kbs[u], vas[u], vbs[u], las[u], lbs[u]);
    }
  } else {
    // LPR == 32: one lane holds the same 16-byte slice of both rows.
    for (int t = warp; t < nvalid; t += WARPS) {
      const int p = pbase + t;
      const int a = c0 + 2 * p;
      const uint4 ka_r = load_raw(Kh + (size_t)a * D + lane * VN);
      const uint4 kb_r = load_raw(Kh + (size_t)(a + 1) * D + lane * VN);
      const uint4 va_r = load_raw(Vh + (size_t)a * D + lane * VN);
      const uint4 vb_r = load_raw(Vh + (size_t)(a + 1) * D + lane * VN);
      const float la = lnh ? lnh[a] : 0.f, lb = lnh ? lnh[a + 1] : 0.f;
      const int off = s_off[t];
      if (s_sel[t]) {
        float ka[VN], kb[VN], va[VN], vb[VN], ko[VN], vo[VN];
        load_vec(reinterpret_cast<const T*>(&ka_r), ka);
        load_vec(reinterpret_cast<const T*>(&kb_r), kb);
        load_vec(reinterpret_cast<const T*>(&va_r), va);
        load_vec(reinterpret_cast<const T*>(&vb_r), vb);
        const float w = s_w[t];
        const float na = expf(la), nb = expf(lb);
        const float inv = 1.f / (na + nb);
#pragma unroll
        for (int e = 0; e < VN; ++e) {
          ko[e] = fmaf(w, kb[e] - ka[e], ka[e]);
          vo[e] = (na * va[e] + nb * vb[e]) * inv;
        }
        store_vec(Ko + (size_t)off * D + lane * VN, ko);
        store_vec(Vo + (size_t)off * D + lane * VN, vo);
        if (lane == 0) lno[off] = logf(na + nb);
        if (dbg_km) {
          float* dk = dbg_km + ((size_t)head * (T_cap / 2) + p) * D + lane * VN;
#pragma unroll
          for (int e = 0; e < VN; e += 4) *reinterpret_cast<float4*>(dk + e) = make_float4(ko[e], ko[e + 1], ko[e + 2], ko[e + 3]);
        }
      } else {
        store_raw(Ko + (size_t)off * D + lane * VN, ka_r);
        store_raw(Ko + (size_t)(off + 1) * D + lane * VN, kb_r);
        store_raw(Vo + (size_t)off * D + lane * VN, va_r);
        store_raw(Vo + (size_t)(off + 1) * D + lane * VN, vb_r);
        if (lane == 0) { lno[off] = la; lno[off + 1] = lb; }
      }
    }
  }
}

// In-place variant: one CTA per head; each chunk is read completely into shared
// memory before any of its rows is written, and rows only move to lower indices,
// so no unread row is ever overwritten.
// 16- and 4-byte asynchronous global -> shared copies (cp.async), completed per thread
// by commit / wait groups.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Shared-memory stages of the in-place merge's walk: items k + 1 .. k + ST - 1 are copied
// in while item k is processed. Two stages: three measured the same on the 32-layer
// prefill (the walk is not bound by its copies' latency there) with half again the
// shared memory per CTA.
constexpr int kInplaceStages = 2;
// Wait until at most kInplaceStages - 1 of this thread's copy groups are pending: with
// one group committed per item (and kInplaceStages - 1 before the walk), item k's landed.
__device__ __forceinline__ void cp_async_wait_stages() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kInplaceStages - 1) : "memory");
}

// In-place merge of one head per CTA. Items are the pair chunks of the span (CH pairs,
// 2 CH rows), then the suffix chunks (2 CH rows). Every output row lies at or below its
// input row, so no item writes a row that a later item still has to read: the rows of
// the next items are being copied into the other shared-memory stages while item k is
// written back (reading ahead never conflicts: rows only move down), and the planning
// warp loads the scores of chunk k + 1 while it plans chunk k.
template <typename T, int D>
__global__ void __launch_bounds__(kMergeThreads)
merge_inplace_kernel(T* __restrict__ K, T* __restrict__ V, float* __restrict__ logn,
                     const float* __restrict__ score, const float* __restrict__ w_b, int scope,
                     int H_kv, int T_cap, const SelUnit* __restrict__ sel,
                     const HeadInfo* __restrict__ hinfo, int32_t* __restrict__ len,
                     uint8_t* __restrict__ dbg_sel, int32_t* __restrict__ dbg_off,
                     float* __restrict__ dbg_km, int32_t* __restrict__ flags) {
  constexpr int CH = inplace_chunk<T, D>();
  constexpr int SROWS = 2 * CH;                                // rows per stage
  constexpr int VPR = D * (int)sizeof(T) / 16;
  constexpr int VN = Vec16<T>::n;
  extern __shared__ __align__(16) unsigned char ism[];
  uint4* sK = reinterpret_cast<uint4*>(ism);                             // [ST][SROWS][VPR]
  uint4* sV = sK + kInplaceStages * SROWS * VPR;                         // [ST][SROWS][VPR]
  float* sL = reinterpret_cast<float*>(sV + kInplaceStages * SROWS * VPR);  // [ST][SROWS]
  __shared__ int s_off[32];
  __shared__ unsigned char s_sel[32];
  __shared__ float s_w[32];
  __shared__ int s_lt, s_eq;

  const int head = blockIdx.x;
  const HeadInfo hi = hinfo[head];
  if (hi.len_in < 0) return;
  const int L = hi.len_in, P = hi.P, R = hi.R, c0 = hi.c0;
  if (L - c0 > kInplaceMaxSpan) {
    if (threadIdx.x == 0) set_flag(flags, KVS_FLAG_INPLACE_SPAN);
    return;
  }
  const int u = scope == KVS_SCOPE_POOLED ? head / H_kv : head;
  const SelUnit su = sel[u];
  T* Kh = K + (size_t)head * T_cap * D;
  T* Vh = V + (size_t)head * T_cap * D;
  float* lnh = logn + (size_t)head * T_cap;
  const float* sc = score + (size_t)head * (T_cap / 2);
  const float* wb = w_b + (size_t)head * (T_cap / 2);
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid == 0) { s_lt = 0; s_eq = hi.eq0; }

  if (R > 0) {
    const int n_pc = (P + CH - 1) / CH;                        // pair chunks
    const int s_begin = c0 + 2 * P;                            // suffix rows move down by R
    const int n_sc = (L - s_begin + SROWS - 1) / SROWS;
    const int n_items = n_pc + n_sc;
    auto item_row0 = [&](int k) { return k < n_pc ? c0 + 2 * CH * k : s_begin + SROWS * (k - n_pc); };
    auto item_rows = [&](int k) {
      return k < n_pc ? 2 * min(CH, P - CH * k) : min(SROWS, L - (s_begin + SROWS * (k - n_pc)));
    };
    auto load_stage = [&](int b, int k) {
      const int r0 = item_row0(k), nr = item_rows(k);
      uint4* dk = sK + b * SROWS * VPR;
      uint4* dv = sV + b * SROWS * VPR;
      float* dl = sL + b * SROWS;
      for (int i = tid; i < nr * VPR; i += blockDim.x) {
        const int r = i / VPR, c = i - r * VPR;
        cp_async16(dk + i, Kh + (size_t)(r0 + r) * D + c * VN);
        cp_async16(dv + i, Vh + (size_t)(r0 + r) * D + c * VN);
      }
      for (int r = tid; r < nr; r += blockDim.x) cp_async4(dl + r, lnh + r0 + r);
    };
    // the first kInplaceStages - 1 items in flight before the walk starts
    for (int k = 0; k < kInplaceStages - 1; ++k) {
      if (k < n_items) load_stage(k, k);
      cp_async_commit();                                       // (possibly empty)
    }
    // the planning warp's scores and weights of the current pair chunk
    float sc_cur = 0.f, w_cur = 0.f;
    if (tid < 32 && lane < min(CH, P)) {
      sc_cur = sc[lane];
      w_cur = wb[lane];
    }
    __syncthreads();                                           // s_lt / s_eq initialised
    for (int k = 0; k < n_items; ++k) {
      const int b = k % kInplaceStages;
      // the stage freed by item k - 1 takes item k + ST - 1
      if (k + kInplaceStages - 1 < n_items)
        load_stage((k + kInplaceStages - 1) % kInplaceStages, k + kInplaceStages - 1);
      cp_async_commit();                                       // (empty near the end)
      if (k < n_pc && tid < 32) {                              // one warp plans the chunk
        const int pb = CH * k, np = min(CH, P - pb);
        float sc_next = 0.f, w_next = 0.f;
        if (k + 1 < n_pc && lane < min(CH, P - pb - CH)) {
          sc_next = sc[pb + CH + lane];
          w_next = wb[pb + CH + lane];
        }
        const int p = pb + lane;
        const bool in = lane < np;
        const uint32_t key = in ? score_key(sc_cur) : 0xffffffffu;
        const bool lt = in && key < su.thr_key;
        const bool eq = in && key == su.thr_key;
        const unsigned blt = __ballot_sync(0xffffffffu, lt);
        const unsigned beq = __ballot_sync(0xffffffffu, eq);
        const unsigned lower = (1u << lane) - 1u;
        const int eqg = s_eq + __popc(beq & lower);
        const bool sl = lt || (eq && eqg < su.need_eq);
        const int sel_before = s_lt + __popc(blt & lower) + min(su.need_eq, eqg) -
                               min(su.need_eq, hi.eq0);
        const int off = c0 + 2 * p - sel_before;
        s_off[lane] = off;
        s_sel[lane] = sl ? 1 : 0;
        s_w[lane] = in ? w_cur : 0.f;
        if (in) {
          if (dbg_sel) dbg_sel[(size_t)head * (T_cap / 2) + p] = sl ? 1 : 0;
          if (dbg_off) dbg_off[(size_t)head * (T_cap / 2) + p] = off;
        }
        __syncwarp();
        if (lane == 0) { s_lt += __popc(blt); s_eq += __popc(beq); }
        sc_cur = sc_next;
        w_cur = w_next;
      }
      cp_async_wait_stages();                                  // this thread's copies of item k landed
      __syncthreads();                                         // everyone's, and the plan
      const uint4* cK = sK + b * SROWS * VPR;
      const uint4* cV = sV + b * SROWS * VPR;
      const float* cL = sL + b * SROWS;
      if (k < n_pc) {
        const int pb = CH * k, np = min(CH, P - pb);
        for (int i = tid; i < np * VPR; i += blockDim.x) {
          const int t = i / VPR, c = i - t * VPR;
          const int off = s_off[t];
          const uint4 ka_r = cK[(2 * t) * VPR + c], kb_r = cK[(2 * t + 1) * VPR + c];
          const uint4 va_r = cV[(2 * t) * VPR + c], vb_r = cV[(2 * t + 1) * VPR + c];
          if (s_sel[t]) {
            float ka[VN], kb[VN], va[VN], vb[VN], ko[VN], vo[VN];
            load_vec(reinterpret_cast<const T*>(&ka_r), ka);
            load_vec(reinterpret_cast<const T*>(&kb_r), kb);
            load_vec(reinterpret_cast<const T*>(&va_r), va);
            load_vec(reinterpret_cast<const T*>(&vb_r), vb);
            const float w = s_w[t];
            const float na = expf(cL[2 * t]), nb = expf(cL[2 * t + 1]);
            const float inv = 1.f / (na + nb);
#pragma unroll
            for (int e = 0; e < VN; ++e) {
              ko[e] = fmaf(w, kb[e] - ka[e], ka[e]);
              vo[e] = (na * va[e] + nb * vb[e]) * inv;
            }
            store_vec(Kh + (size_t)off * D + c * VN, ko);
            store_vec(Vh + (size_t)off * D + c * VN, vo);
            if (c == 0) lnh[off] = logf(na + nb);
            if (dbg_km) {
              float* dk = dbg_km + ((size_t)head * (T_cap / 2) + pb + t) * D + c * VN;
#pragma unroll
              for (int e = 0; e < VN; e += 4) *reinterpret_cast<float4*>(dk + e) = make_float4(ko[e], ko[e + 1], ko[e + 2], ko[e + 3]);
            }
          } else {
            *reinterpret_cast<uint4*>(Kh + (size_t)off * D + c * VN) = ka_r;
            *reinterpret_cast<uint4*>(Kh + (size_t)(off + 1) * D + c * VN) = kb_r;
            *reinterpret_cast<uint4*>(Vh + (size_t)off * D + c * VN) = va_r;
            *reinterpret_cast<uint4*>(Vh + (size_t)(off + 1) * D + c * VN) = vb_r;
            if (c == 0) { lnh[off] = cL[2 * t]; lnh[off + 1] = cL[2 * t + 1]; }
          }
        }
      } else {
        const int s0 = item_row0(k), nr = item_rows(k);
        for (int i = tid; i < nr * VPR; i += blockDim.x) {
          const int r = i / VPR, c = i - r * VPR;
          *reinterpret_cast<uint4*>(Kh + (size_t)(s0 + r - R) * D + c * VN) = cK[i];
          *reinterpret_cast<uint4*>(Vh + (size_t)(s0 + r - R) * D + c * VN) = cV[i];
        }
        for (int r = tid; r < nr; r += blockDim.x) lnh[s0 + r - R] = cL[r];
      }
      __syncthreads();                                         // stage b and the plan are free
    }
  } else if (dbg_sel || dbg_off) {
    for (int p = tid; p < P; p += blockDim.x) {
      if (dbg_sel) dbg_sel[(size_t)head * (T_cap / 2) + p] = 0;
      if (dbg_off) dbg_off[(size_t)head * (T_cap / 2) + p] = c0 + 2 * p;
    }
  }
  __syncthreads();
  if (tid == 0) len[head] = L - R;
}

cudaError_t launch_select(const kvs_cache_desc& d, const float* score, const int32_t* len,
                          const int32_t* cand_begin, int n_recent, const int32_t* target,
                          int scope, const MergeLayout& Ly, char* ws, cudaStream_t st) {
  const int units = scope == KVS_SCOPE_POOLED ? d.B : d.B * d.H_kv;
  const cudaError_t e = launch_pdl(
      select_kernel, dim3(units), dim3(kSelThreads), 0, st, score, len, cand_begin, n_recent,
      target, scope, d.H_kv, d.T_cap, Ly.nblk, reinterpret_cast<SelUnit*>(ws + Ly.sel),
      reinterpret_cast<HeadInfo*>(ws + Ly.head), reinterpret_cast<int2*>(ws + Ly.blk),
      reinterpret_cast<int32_t*>(ws));
  count_launches(1);
  return e;
}

template <typename T, int D>
static cudaError_t launch_merge_t(const kvs_cache_desc& d, const void* K, const void* V,
                                  const float* logn, const float* score, const float* w_b,
                                  int scope, int T_cap_out, bool inplace, void* K_out,
                                  void* V_out, float* logn_out, int32_t* len_out,
                                  uint8_t* dbg_sel, int32_t* dbg_off, float* dbg_km,
                                  const MergeLayout& Ly, char* ws, cudaStream_t st) {
  const int heads = d.B * d.H_kv;
  const SelUnit* sel = reinterpret_cast<const SelUnit*>(ws + Ly.sel);
  const HeadInfo* hinfo = reinterpret_cast<const HeadInfo*>(ws + Ly.head);
  const int2* blk = reinterpret_cast<const int2*>(ws + Ly.blk);
  int32_t* flags = reinterpret_cast<int32_t*>(ws);
  if (inplace) {
    constexpr int VPR = D * (int)sizeof(T) / 16;
    constexpr int CH = inplace_chunk<T, D>();
    // kInplaceStages stages of K, V (2 CH rows each) and log-counts
    constexpr size_t smem = (size_t)kInplaceStages * 2 * (2 * CH * VPR) * 16 +
                            (size_t)kInplaceStages * 2 * CH * sizeof(float);
    static_assert(smem <= 100 * 1024, "in-place staging");
    auto kfn = merge_inplace_kernel<T, D>;
    if (!ensure_smem_attr((const void*)kfn, smem)) return cudaErrorInvalidValue;
    kfn<<<heads, kMergeThreads, smem, st>>>((T*)K_out, (T*)V_out, logn_out, score, w_b, scope,
                                            d.H_kv, d.T_cap, sel, hinfo, len_out, dbg_sel,
                                            dbg_off, dbg_km, flags);
    count_launches(1);
    return cudaGetLastError();
  }
  const int ncopy = (d.T_cap + kCopyRows - 1) / kCopyRows;
  dim3 grid(Ly.nblk + ncopy, heads);
  const cudaError_t e = launch_pdl(
      merge_kernel<T, D>, grid, dim3(kMergeThreads), 0, st, (const T*)K, (const T*)V, logn, score,
      w_b, scope, d.H_kv, d.T_cap, T_cap_out, Ly.nblk, sel, hinfo, blk, (T*)K_out, (T*)V_out,
      logn_out, len_out, dbg_sel, dbg_off, dbg_km, flags);
  count_launches(1);
  return e;
}

cudaError_t launch_merge(const kvs_cache_desc& d, const void* K, const void* V, const float* logn,
                         const float* score, const float* w_b, int scope, int T_cap_out,
                         bool inplace, void* K_out, void* V_out, float* logn_out,
                         int32_t* len_out, uint8_t* dbg_sel, int32_t* dbg_off, float* dbg_km,
                         const MergeLayout& Ly, char* ws, cudaStream_t st) {
#define KVS_MERGE_ARGS K, V, logn, score, w_b, scope, T_cap_out, inplace, K_out, V_out, logn_out, \
                       len_out, dbg_sel, dbg_off, dbg_km, Ly, ws, st
  if (d.dtype == KVS_BF16) {
    if (d.d == 128) return launch_merge_t<bf16, 128>(d, KVS_MERGE_ARGS);
    return launch_merge_t<bf16, 64>(d, KVS_MERGE_ARGS);
  }
  if (d.d == 128) return launch_merge_t<float, 128>(d, KVS_MERGE_ARGS);
  return launch_merge_t<float, 64>(d, KVS_MERGE_ARGS);
#undef KVS_MERGE_ARGS
}

}  // namespace kvs
