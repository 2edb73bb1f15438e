// Window statistics for bf16 caches on the 5th-generation tensor cores.
//
// Attention forward of the KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程",
// §数学主线三) for the G*W window queries of a KV head, reduced to what the pair norms
// of §数学主线四 need: alpha_bar_t = mean_q softmax_t and o_bar = mean_q o_q.
// Because o_bar = sum_t alpha_bar_t v_t, no P.V contraction is needed: the only dense
// contraction is S = Q K^T (M = 128 padded window queries, N = 128 keys, K = d), done
// twice:
//   pass A (MASS = false): per (KV head, key split) the online row maximum and row sum
//          of 2^s, s = log2(e) (q.k / sqrt(d) + logn)  -> per-split (m, l);
//   pass B (MASS = true):  with the combined (m, l), P = 2^(s - m) / l, its column sums
//          over the window queries give alpha_bar for the split's keys, and the CUDA
//          cores form o_bar's split partial sum_t alpha_bar_t v_t from the V tile.
// Warp roles: warp 0 issues TMA tile loads (128-byte swizzle, no multicast) of Q once
// and of K (and V) per 128-key tile into mbarrier-guarded rings; warp 1 owns the
// tensor memory (two 128-column fp32 S buffers) and one thread issues tcgen05.mma
// with smem descriptors, committing to mbarriers; warps 2-9 read S rows from tensor
// memory (one row, half of the keys, per thread) and do the softmax arithmetic.
// Every wait is bounded.
#include <cudaTypedefs.h>

#include "kvs_common.cuh"
#include "kvs_kernels.h"
#include "ptx.cuh"

namespace kvs {

constexpr int kWtKeys = 128;            // keys per tile: MMA N
constexpr int kWtRows = 128;            // window-query rows, padded: MMA M
constexpr int kWtSoft = 8;              // softmax warps (two per TMEM lane quarter)
constexpr int kWtThreads = (2 + kWtSoft) * 32;
constexpr uint32_t kWtTmemCols = 256;   // two S buffers of 128 fp32 columns

template <int D, bool MASS>
struct WtShape {
  static constexpr int kBoxes = D / 64;                 // 64-element boxes per row
  static constexpr int kBox = 128 * 128;                // one box: 128 rows x 128 bytes
  static constexpr int kTile = kBoxes * kBox;           // a Q, K or V tile
  static constexpr int kKStages = MASS ? 2 : 3;
  static constexpr int kVStages = MASS ? 2 : 0;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kTile;
  static constexpr int kVOff = kKOff + kKStages * kTile;
  static constexpr int kBarOff = kVOff + kVStages * kTile;
  static constexpr int kSmem = kBarOff + 256 + 1024;    // barriers + 1024-byte alignment slack
};

template <int D, bool MASS>
__global__ void __launch_bounds__(kWtThreads, 1)
window_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const float* __restrict__ logn,
                 const int32_t* __restrict__ len, int H_kv, int H_q, int W, int T_cap,
                 int nsplit, const float* __restrict__ stats, float* __restrict__ part_ml,
                 float* __restrict__ alpha, float* __restrict__ opart,
                 int32_t* __restrict__ flags) {
  using S = WtShape<D, MASS>;
  constexpr int KS = S::kKStages, VS = S::kVStages;
  extern __shared__ unsigned char dsm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(dsm) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::kBarOff);
  uint64_t* q_full = bars;                       // 1
  uint64_t* k_full = bars + 1;                   // KS
  uint64_t* k_empty = k_full + KS;               // KS
  uint64_t* s_full = k_empty + KS;               // 2
  uint64_t* s_empty = s_full + 2;                // 2
  uint64_t* v_full = s_empty + 2;                // VS
  uint64_t* v_empty = v_full + VS;               // VS
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;               // set when any wait gives up
  __shared__ float red[4][kWtKeys];              // column sums per lane quarter (pass B)
  __shared__ float abar[kWtKeys];                // alpha_bar of the tile's keys (pass B)
  __shared__ float ored[2 * kWtSoft * 32];       // row-group partials of o_bar (pass B)

  const int unit = blockIdx.y, split = blockIdx.x;
  const int b = unit / H_kv, h = unit - b * H_kv;
  const int G = H_q / H_kv, Qn = G * W;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int L = len[unit];
  if (L < 0 || L > T_cap) {
    if (split == 0 && tid == 0) set_flag(flags, KVS_FLAG_BAD_LENGTH);
    L = 0;
  }
  int chunk = (L + nsplit - 1) / nsplit;
  chunk = (chunk + kWtKeys - 1) / kWtKeys * kWtKeys;
  const int t0 = split * chunk, t1 = min(L, t0 + chunk);
  const int ntiles = t1 > t0 ? (t1 - t0 + kWtKeys - 1) / kWtKeys : 0;
  const int q_row0 = (b * H_q + h * G) * W;      // first window-query row of this KV head
  const int k_row0 = unit * T_cap + t0;          // first cache row of this split

  if (tid == 0) {
    s_abort = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < KS; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&s_full[s], 1); mbar_init(&s_empty[s], kWtSoft); }
    for (int s = 0; s < VS; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], kWtSoft); }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&s_tmem, kWtTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      if (MASS) prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(q_full, S::kTile);
#pragma unroll
      for (int bx = 0; bx < S::kBoxes; ++bx)
        tma_load_2d(base + S::kQOff + bx * S::kBox, &tmQ, bx * 64, q_row0, q_full);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % KS;
        if (i >= KS && !mbar_wait_ab(&k_empty[s], ((i / KS) - 1) & 1, &s_abort)) {
          set_flag(flags, KVS_FLAG_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&k_full[s], S::kTile);
#pragma unroll
        for (int bx = 0; bx < S::kBoxes; ++bx)
          tma_load_2d(base + S::kKOff + s * S::kTile + bx * S::kBox, &tmK, bx * 64,
                      k_row0 + i * kWtKeys, &k_full[s]);
        if constexpr (MASS) {
          const int v = i % VS;
          if (i >= VS && !mbar_wait_ab(&v_empty[v], ((i / VS) - 1) & 1, &s_abort)) {
            set_flag(flags, KVS_FLAG_TIMEOUT);
            issued = i + 1;   // the K tile above was issued
            break;
          }
          mbar_arrive_expect_tx(&v_full[v], S::kTile);
#pragma unroll
          for (int bx = 0; bx < S::kBoxes; ++bx)
            tma_load_2d(base + S::kVOff + v * S::kTile + bx * S::kBox, &tmV, bx * 64,
                        k_row0 + i * kWtKeys, &v_full[v]);
        }
        issued = i + 1;
      }
      // loads still in flight must land before the CTA ends
      // (bounded by the plain limit even after an abort: these are our own copies)
      if (!mbar_wait(q_full, 0)) set_flag(flags, KVS_FLAG_TIMEOUT);
      for (int i = issued > KS ? issued - KS : 0; i < issued; ++i)
        if (!mbar_wait(&k_full[i % KS], (i / KS) & 1)) set_flag(flags, KVS_FLAG_TIMEOUT);
      if constexpr (MASS)
        for (int i = issued > VS ? issued - VS : 0; i < issued; ++i)
          if (!mbar_wait(&v_full[i % VS], (i / VS) & 1)) set_flag(flags, KVS_FLAG_TIMEOUT);
    }
    __syncwarp();   // reconverge before the CTA-wide barrier below
  } else if (warp == 1) {
    // ---------------- MMA issuer: S[buf] = Q K^T ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(kWtRows, kWtKeys);
      const uint32_t q_addr = smem_u32(base + S::kQOff);
      bool ok = mbar_wait_ab(q_full, 0, &s_abort);
      int done = 0;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % KS, buf = i & 1;
        if (!mbar_wait_ab(&k_full[s], (i / KS) & 1, &s_abort) ||
            (i >= 2 && !mbar_wait_ab(&s_empty[buf], ((i / 2) - 1) & 1, &s_abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(base + S::kKOff + s * S::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (uint32_t)((ks >> 2) * S::kBox + (ks & 3) * 32);
          umma_bf16_ss(tmem + buf * kWtKeys, umma_desc_k_sw128(q_addr + off),
                       umma_desc_k_sw128(k_addr + off), idesc, ks > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[buf]);
        umma_commit(&k_empty[s]);
        done = i + 1;
      }
      if (!ok) set_flag(flags, KVS_FLAG_TIMEOUT);
      // the last MMAs must finish before the tensor memory is released
      if (done > 0 && !mbar_wait(&s_full[(done - 1) & 1], ((done - 1) / 2) & 1))
        set_flag(flags, KVS_FLAG_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps: two per TMEM lane quarter ----------------
    // warp 2 + sw (sw = 0..7) reads lane quarter (warp & 3), i.e. window-query rows
    // 32 * quarter + lane, and the key columns [NC * half, NC * half + NC) of each tile
    constexpr int NC = kWtKeys / (kWtSoft / 4);   // 64 key columns per softmax warp
    constexpr int NST = kWtSoft * 32;             // 256 softmax threads
    const int sw = warp - 2;
    const int quarter = warp & 3;
    const int half = sw >> 2;
    const int c0w = half * NC;
    const int r = quarter * 32 + lane;            // window-query row of the KV head
    const int st = tid - 64;                      // index among the softmax threads
    const int pos = L - W + (r % W);              // last cache position row r attends
    const bool row_ok = r < Qn && pos >= 0;
    const int Qv = G * min(W, L);                 // window queries with a position >= 0
    const float qscale = kLog2e / sqrtf((float)D);
    const float* lnh = logn ? logn + (size_t)unit * T_cap : nullptr;
    __shared__ __align__(16) float lns[2][kWtKeys];   // log2(e) * logn of the tile's keys
    __shared__ float rowstat[kWtRows][2];         // pass A: second half's (m, l) per row
    float m = -INFINITY, l = 0.f;                 // pass A: running statistics of the half-row
    float Mr = 0.f, invL = 0.f;                   // pass B: final row statistics
    if (MASS && row_ok) {
      const float M0 = stats[((size_t)unit * Qn + r) * 2], L0 = stats[((size_t)unit * Qn + r) * 2 + 1];
      if (L0 > 0.f && isfinite(L0) && isfinite(M0)) { Mr = M0; invL = 1.f / L0; }
    }
    float oacc2[2] = {0.f, 0.f};                  // pass B: o_bar partials of a column pair
    // each tile's log-counts are fetched one tile ahead (threads st < 128, one key each)
    float ln_next = (lnh && st < kWtKeys && t0 + st < t1) ? lnh[t0 + st] : 0.f;
    for (int i = 0; i < ntiles; ++i) {
      const int buf = i & 1;
      const int tb = t0 + i * kWtKeys;
      const float ln_cur = ln_next;
      if (lnh && st < kWtKeys) ln_next = (tb + kWtKeys + st < t1) ? lnh[tb + kWtKeys + st] : 0.f;
      bool live = mbar_wait_ab(&s_full[buf], (i / 2) & 1, &s_abort);
      live = __all_sync(0xffffffffu, live);       // tcgen05.ld is warp-collective
      float sv[NC];
      if (live) {
        tc_fence_after();
        const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * kWtKeys + c0w);
#pragma unroll
        for (int c = 0; c < NC / 32; ++c) {
          float part[32];
          tmem_ld32(ta + c * 32, part);
#pragma unroll
          for (int j = 0; j < 32; ++j) sv[c * 32 + j] = part[j];
        }
      } else {
        set_flag(flags, KVS_FLAG_TIMEOUT);
#pragma unroll
        for (int j = 0; j < NC; ++j) sv[j] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[buf]);  // this warp is done with the S buffer
      if (lnh) {
        if (st < kWtKeys) lns[buf][st] = ln_cur * kLog2e;
        named_bar(1, NST);
      }
      // logits in the log2 domain. Only the split's last tile and the last W cache
      // positions need masks (split end, causal window); interior tiles skip them.
      const bool interior = tb + kWtKeys <= t1 && tb + kWtKeys - 1 <= L - W;
      if (interior && live && row_ok) {
        if (lnh) {
#pragma unroll
          for (int j = 0; j < NC; j += 4) {
            const float4 lv = *reinterpret_cast<const float4*>(&lns[buf][c0w + j]);
            sv[j] = fmaf(sv[j], qscale, lv.x);
            sv[j + 1] = fmaf(sv[j + 1], qscale, lv.y);
            sv[j + 2] = fmaf(sv[j + 2], qscale, lv.z);
            sv[j + 3] = fmaf(sv[j + 3], qscale, lv.w);
          }
        } else {
#pragma unroll
          for (int j = 0; j < NC; ++j) sv[j] *= qscale;
        }
      } else {
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          const int t = tb + c0w + j;
          const bool vis = live && row_ok && t < t1 && t <= pos;
          sv[j] = vis ? fmaf(sv[j], qscale, lnh ? lns[buf][c0w + j] : 0.f) : -INFINITY;
        }
      }
      if constexpr (!MASS) {
        // eight independent chains instead of one long dependency chain
        float tm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) tm[k] = sv[k];
#pragma unroll
        for (int j = 8; j < NC; ++j) tm[j & 7] = fmaxf(tm[j & 7], sv[j]);
        const float tmax = fmaxf(fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3])),
                                 fmaxf(fmaxf(tm[4], tm[5]), fmaxf(tm[6], tm[7])));
        const float m_new = fmaxf(m, tmax);
        if (m_new > -INFINITY) {
          float ps[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) ps[k] = 0.f;
#pragma unroll
          for (int j = 0; j < NC; ++j) ps[j & 7] += exp2f(sv[j] - m_new);
          const float psum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
          l = l * exp2f(m - m_new) + psum;
          m = m_new;
        }
      } else {
        // normalised probabilities; column sums over this warp's 32 rows by a
        // transpose-reduce: after it, lane j holds the sum of column j of each 32-column block
#pragma unroll
        for (int c = 0; c < NC / 32; ++c) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = exp2f(sv[c * 32 + j] - Mr) * invL;
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) {
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int k = 0; k < o; ++k) {
              const float give = up ? v[k] : v[k + o];
              const float keep = up ? v[k + o] : v[k];
              v[k] = keep + __shfl_xor_sync(0xffffffffu, give, o);
            }
          }
          red[quarter][c0w + c * 32 + lane] = v[0];
        }
        named_bar(1, NST);
        if (st < kWtKeys) {
          const int t = tb + st;
          float a = (red[0][st] + red[1][st] + red[2][st] + red[3][st]) / (float)(Qv > 0 ? Qv : 1);
          a = (t < t1 && Qv > 0) ? a : 0.f;
          if (t < t1) alpha[(size_t)unit * T_cap + t] = a;
          abar[st] = a;
        }
        const int vs = i % VS;
        bool vlive = mbar_wait_ab(&v_full[vs], (i / VS) & 1, &s_abort);
        named_bar(1, NST);
        if (vlive) {
          // o_bar partial: thread st takes the column pair (2 cp, 2 cp + 1), cp = st % (D/2),
          // over rows j = rg, rg + NRG, ... (rg = st / (D/2)); two accumulators per column
          constexpr int NRG = 2 * NST / D;
          const unsigned char* vt = base + S::kVOff + vs * S::kTile;
          const int cp = st % (D / 2), rg = st / (D / 2);
          const int cc = (2 * cp) & 63, bx = (2 * cp) >> 6;
          const int nvalid = min(kWtKeys, t1 - tb);
          float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
          int j = rg;
          for (; j + NRG < nvalid; j += 2 * NRG) {
            const uint32_t x = *reinterpret_cast<const uint32_t*>(
                vt + bx * S::kBox + j * 128 + ((((cc >> 3) ^ (j & 7)) << 4) + (cc & 7) * 2));
            const int j2 = j + NRG;
            const uint32_t y = *reinterpret_cast<const uint32_t*>(
                vt + bx * S::kBox + j2 * 128 + ((((cc >> 3) ^ (j2 & 7)) << 4) + (cc & 7) * 2));
            a0 = fmaf(abar[j], bf16_lo(x), a0);
            a1 = fmaf(abar[j], bf16_hi(x), a1);
            b0 = fmaf(abar[j2], bf16_lo(y), b0);
            b1 = fmaf(abar[j2], bf16_hi(y), b1);
          }
          if (j < nvalid) {
            const uint32_t x = *reinterpret_cast<const uint32_t*>(
                vt + bx * S::kBox + j * 128 + ((((cc >> 3) ^ (j & 7)) << 4) + (cc & 7) * 2));
            a0 = fmaf(abar[j], bf16_lo(x), a0);
            a1 = fmaf(abar[j], bf16_hi(x), a1);
          }
          oacc2[0] += a0 + b0;
          oacc2[1] += a1 + b1;
        } else {
          set_flag(flags, KVS_FLAG_TIMEOUT);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&v_empty[vs]);
      }
    }
    // per-split outputs
    if constexpr (!MASS) {
      // merge the two half-rows of each window query
      if (half == 1) { rowstat[r][0] = m; rowstat[r][1] = l; }
      named_bar(1, NST);
      if (half == 0 && r < Qn) {
        const float m1 = rowstat[r][0], l1 = rowstat[r][1];
        const float M = fmaxf(m, m1);
        const float Ls = M > -INFINITY ? l * exp2f(m - M) + l1 * exp2f(m1 - M) : 0.f;
        part_ml[(((size_t)unit * nsplit + split) * Qn + r) * 2 + 0] = M;
        part_ml[(((size_t)unit * nsplit + split) * Qn + r) * 2 + 1] = Ls;
      }
    } else {
      // combine the row groups of each column pair
      constexpr int NRG = 2 * NST / D;
      const int cp = st % (D / 2), rg = st / (D / 2);
      ored[rg * D + 2 * cp] = oacc2[0];
      ored[rg * D + 2 * cp + 1] = oacc2[1];
      named_bar(1, NST);
      if (st < D) {
        float a = 0.f;
#pragma unroll
        for (int k = 0; k < NRG; ++k) a += ored[k * D + st];
        opart[((size_t)unit * nsplit + split) * D + st] = a;
      }
    }
  }

  // tensor memory is released by the warp that allocated it, after every read
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kWtTmemCols);
  }
}

// Per KV head: merge the split statistics of every window query.
__global__ void __launch_bounds__(128)
wt_combine_stats_kernel(const float* __restrict__ part_ml, int Qn, int nsplit,
                        float* __restrict__ stats) {
  const int unit = blockIdx.x;
  for (int q = threadIdx.x; q < Qn; q += blockDim.x) {
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) {
      const float* e = part_ml + (((size_t)unit * nsplit + s) * Qn + q) * 2;
      if (e[1] > 0.f) M = fmaxf(M, e[0]);
    }
    float Ls = 0.f;
    if (M > -INFINITY) {
      for (int s = 0; s < nsplit; ++s) {
        const float* e = part_ml + (((size_t)unit * nsplit + s) * Qn + q) * 2;
        if (e[1] > 0.f) Ls = fmaf(e[1], exp2f(e[0] - M), Ls);
      }
    }
    stats[((size_t)unit * Qn + q) * 2 + 0] = M;
    stats[((size_t)unit * Qn + q) * 2 + 1] = Ls;
  }
}

// Per KV head: o_bar = sum over splits of sum_t alpha_bar_t v_t.
__global__ void __launch_bounds__(128)
wt_combine_obar_kernel(const float* __restrict__ opart, int nsplit, int D, float* __restrict__ obar) {
  const int unit = blockIdx.x;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < nsplit; ++s) a += opart[((size_t)unit * nsplit + s) * D + c];
    obar[(size_t)unit * D + c] = a;
  }
}

static int window_tc_splits(const kvs_cache_desc& d) {
  const int units = d.B * d.H_kv;
  int s = 148 / units;            // one CTA per SM, one wave
  if (s < 1) s = 1;
  const int cap = window_splits(d);
  return s < cap ? s : cap;
}

bool window_tc_supported(const kvs_cache_desc& d, int W) {
  const unsigned long long rows = (unsigned long long)d.B * d.H_kv * (unsigned long long)d.T_cap;
  const unsigned long long qrows = (unsigned long long)d.B * d.H_q * (unsigned long long)W;
  return d.dtype == KVS_BF16 && (d.d == 64 || d.d == 128) && (d.H_q / d.H_kv) * W <= kWtRows &&
         rows < (1ull << 31) && qrows < (1ull << 31) && tensor_map_encoder() != nullptr;
}

template <int D, bool MASS>
static bool wt_attr() {
  return ensure_smem_attr((const void*)window_tc_kernel<D, MASS>, WtShape<D, MASS>::kSmem);
}

template <int D>
static cudaError_t launch_wt(const kvs_cache_desc& d, const CUtensorMap& mQ, const CUtensorMap& mK,
                             const CUtensorMap& mV, const float* logn, const int32_t* len, int W,
                             const ScoreLayout& Ly, char* ws, cudaStream_t st) {
  if (!wt_attr<D, false>() || !wt_attr<D, true>()) return cudaErrorInvalidValue;
  const int units = d.B * d.H_kv;
  const int nsplit = window_tc_splits(d);
  const int Qn = Ly.Qn;
  int32_t* flags = reinterpret_cast<int32_t*>(ws);
  float* part_ml = reinterpret_cast<float*>(ws + Ly.part_ml);
  float* opart = reinterpret_cast<float*>(ws + Ly.part_o);
  float* stats = reinterpret_cast<float*>(ws + Ly.stats);
  float* obar = reinterpret_cast<float*>(ws + Ly.obar);
  float* alpha = reinterpret_cast<float*>(ws + Ly.alpha);
  const dim3 grid(nsplit, units);
  window_tc_kernel<D, false><<<grid, kWtThreads, WtShape<D, false>::kSmem, st>>>(
      mQ, mK, mV, logn, len, d.H_kv, d.H_q, W, d.T_cap, nsplit, nullptr, part_ml, nullptr,
      nullptr, flags);
  wt_combine_stats_kernel<<<units, 128, 0, st>>>(part_ml, Qn, nsplit, stats);
  window_tc_kernel<D, true><<<grid, kWtThreads, WtShape<D, true>::kSmem, st>>>(
      mQ, mK, mV, logn, len, d.H_kv, d.H_q, W, d.T_cap, nsplit, stats, nullptr, alpha, opart,
      flags);
  wt_combine_obar_kernel<<<units, 128, 0, st>>>(opart, nsplit, D, obar);
  count_launches(4);
  return cudaGetLastError();
}

cudaError_t launch_window_stats_tc(const kvs_cache_desc& d, const void* K, const void* V,
                                   const float* logn, const int32_t* len, const void* Qw, int W,
                                   const ScoreLayout& Ly, char* ws, cudaStream_t st) {
  const unsigned long long rows = (unsigned long long)d.B * d.H_kv * (unsigned long long)d.T_cap;
  const unsigned long long qrows = (unsigned long long)d.B * d.H_q * (unsigned long long)W;
  CUtensorMap mQ, mK, mV;
  if (!encode_rows_map(&mQ, Qw, qrows, d.d, kWtRows) ||
      !encode_rows_map(&mK, K, rows, d.d, kWtKeys) || !encode_rows_map(&mV, V, rows, d.d, kWtKeys))
    return cudaErrorInvalidValue;
  if (d.d == 128) return launch_wt<128>(d, mQ, mK, mV, logn, len, W, Ly, ws, st);
  return launch_wt<64>(d, mQ, mK, mV, logn, len, W, Ly, ws, st);
}

}  // namespace kvs
