// Window statistics and pair scores for bf16 caches, fused into two passes on the
// 5th-generation tensor cores.
//
// The method: the KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程").
// The attention forward of §数学主线三 gives, for each window query q of a KV head,
// alpha_q = softmax(q K^T / sqrt(d) + logn) and o_q = sum_t alpha_qt v_t; the pair norms
// of §数学主线四 need alpha and o at the pair (c11, c22, c12), and the merged key and its
// score follow in closed form (§数学主线二, §数学主线四).
//
//   pass A (window_fa_kernel, per KV head and key split): S = Q K^T and O += P V on the
//     tensor cores, flash-attention style: per window query the running maximum m and
//     sum l of 2^s and the unnormalised output O, so that the window's o_q are known
//     before any pair is scored. P is rounded to bf16 twice (P = P_hi + P_lo, both
//     multiplied by V) so that O keeps close to fp32 accuracy. The reference maximum
//     of a row moves only when a tile exceeds it by 2^8 (the accumulator is then
//     rescaled in tensor memory), so P <= 2^8 between moves.
//   fa_combine_kernel (per KV head): the splits' (m, l, O) -> per query (M, L) and o_q,
//     o_bar = mean_q o_q, and for pass B's per-query form e_q = o_q - o_bar as bf16 hi / lo
//     rows with |e_q|^2 and o_bar . e_q.
//   pass B (window_score_kernel, per KV head and candidate split): S^T = K Q^T with the
//     keys on the tensor-memory lanes, so that a thread owns one key and its row of
//     window probabilities p_qt = 2^(s_qt - M_q) / L_q: alpha_bar_t is a sum over the
//     thread's own columns. A candidate pair is two adjacent rows of the same 128-row
//     tile (tiles start at the candidate span's first row), so the pair norms, weight
//     and score come straight from the K and V rows already in shared memory.
//     Window form "mean" (the plain reading): the one-query norms at (alpha_bar, o_bar).
//     Window form "per query": the one-query norms of every window query, averaged.
//     With e_q = o_q - o_bar, |v - o_q|^2 = |v - o_bar|^2 - 2 (v.e_q - o_bar.e_q) + |e_q|^2
//     and |v_a + v_b - 2 o_q|^2 = |v_a + v_b - 2 o_bar|^2 - 4 (v_a.e_q + v_b.e_q
//     - 2 o_bar.e_q) + 4 |e_q|^2, the row terms taken directly in fp32 as in the mean form
//     and U = V E^T (E as bf16 hi + lo) on the tensor cores: centring on o_bar keeps the
//     product small where v and o_q are close, so the expansion does not cancel.
//
// Warp roles (both passes): warp 0 issues the TMA loads (128-byte swizzle, no
// multicast), warp 1 owns the tensor memory and one of its threads issues tcgen05.mma,
// warps 2-9 do the softmax arithmetic (two per tensor-memory lane quarter). Every wait
// is bounded.
#include <cudaTypedefs.h>

#include "kvs_common.cuh"
#include "kvs_kernels.h"
#include "ptx.cuh"

namespace kvs {

constexpr int kFuKeys = 128;            // keys per tile
constexpr int kFuSoft = 8;              // softmax warps
constexpr int kFuThreads = (2 + kFuSoft) * 32;
constexpr int kFuSoftThreads = kFuSoft * 32;
constexpr float kRescaleSlack = 8.f;    // log2 units
constexpr int kPrefetch = 3;            // tiles prefetched into L2 beyond the ring

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) &
                                          ~static_cast<uintptr_t>(1023));
}

// ---------------------------------------------------------------------------
// Pass A: per-split softmax statistics and unnormalised window outputs
// ---------------------------------------------------------------------------

template <int D>
struct FaShape {
  static constexpr int kBoxes = D / 64;
  static constexpr int kBox = 128 * 128;                 // 128 rows x 128 bytes
  static constexpr int kTile = kBoxes * kBox;            // a Q, K or V tile
  static constexpr int kPBytes = 2 * kBox;               // P: 128 rows x 128 keys, bf16
  static constexpr int kStages = D == 128 ? 2 : 3;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTile;
  static constexpr int kVOff = kKOff + kStages * kTile;
  static constexpr int kPOff = kVOff + kStages * kTile;  // P_hi, then P_lo
  static constexpr int kSmallOff = kPOff + 2 * kPBytes;
  // barriers (256 B), per-row partial maxima / sums [2][128], log-counts [128],
  // tensor-memory address and abort flag
  static constexpr int kBarBytes = 256;
  static constexpr int kSmallBytes = kBarBytes + 2 * 128 * 4 + 128 * 4 + 16;
  static constexpr int kSmem = kSmallOff + kSmallBytes + 1024;
  static_assert(kSmem <= 232448, "shared memory");
};

constexpr uint32_t kFaTmemCols = 512;   // S0 [0,128), S1 [128,256), O [256, 256 + D)

template <int D>
__global__ void __launch_bounds__(kFuThreads, 1)
window_fa_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const float* __restrict__ logn,
                 const int32_t* __restrict__ len, int H_kv, int H_q, int W, int T_cap, int nsplit,
                 float* __restrict__ part_ml, float* __restrict__ part_o,
                 int32_t* __restrict__ flags) {
  using S = FaShape<D>;
  constexpr int ST = S::kStages;
  extern __shared__ unsigned char dsm[];
  unsigned char* base = align1024(dsm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::kSmallOff);
  uint64_t* q_full = bars;              // 1
  uint64_t* k_full = q_full + 1;        // ST
  uint64_t* k_empty = k_full + ST;      // ST: the QK^T MMA of the stage is done
  uint64_t* v_full = k_empty + ST;      // ST
  uint64_t* v_empty = v_full + ST;      // ST: the P V MMA of the stage is done
  uint64_t* s_full = v_empty + ST;      // 2
  uint64_t* s_empty = s_full + 2;       // 2: every softmax warp has read S
  uint64_t* p_full = s_empty + 2;       // 1: every softmax warp has written P
  uint64_t* pv_done = p_full + 1;       // 1: the P V MMAs of a tile are done
  float* xch = reinterpret_cast<float*>(base + S::kSmallOff + S::kBarBytes);   // [2][128]
  float* lns = xch + 256;                                                      // [128]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(lns + 128);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

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
  chunk = (chunk + kFuKeys - 1) / kFuKeys * kFuKeys;
  const int t0 = split * chunk, t1 = min(L, t0 + chunk);
  const int ntiles = t1 > t0 ? (t1 - t0 + kFuKeys - 1) / kFuKeys : 0;
  const int q_row0 = (b * H_q + h * G) * W;
  const int k_row0 = unit * T_cap + t0;

  if (tid == 0) {
    *s_abort = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], kFuSoft);
    }
    mbar_init(p_full, kFuSoft);
    mbar_init(pv_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(s_tmem, kFaTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(q_full, S::kTile);
#pragma unroll
      for (int bx = 0; bx < S::kBoxes; ++bx)
        tma_load_2d(base + S::kQOff + bx * S::kBox, &tmQ, bx * 64, q_row0, q_full);
      // tiles beyond the ring are prefetched into L2, kPrefetch tiles ahead
      auto prefetch = [&](int i) {
        if (i < ntiles)
#pragma unroll
          for (int bx = 0; bx < S::kBoxes; ++bx) {
            tma_prefetch_2d(&tmK, bx * 64, k_row0 + i * kFuKeys);
            tma_prefetch_2d(&tmV, bx * 64, k_row0 + i * kFuKeys);
          }
      };
      for (int i = ST; i < ST + kPrefetch; ++i) prefetch(i);
      int issued_k = 0, issued_v = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % ST;
        const uint32_t ph = ((i / ST) - 1) & 1;
        prefetch(i + ST + kPrefetch);
        if (i >= ST && !mbar_wait_ab(&k_empty[s], ph, s_abort)) break;
        mbar_arrive_expect_tx(&k_full[s], S::kTile);
#pragma unroll
        for (int bx = 0; bx < S::kBoxes; ++bx)
          tma_load_2d(base + S::kKOff + s * S::kTile + bx * S::kBox, &tmK, bx * 64,
                      k_row0 + i * kFuKeys, &k_full[s]);
        issued_k = i + 1;
        if (i >= ST && !mbar_wait_ab(&v_empty[s], ph, s_abort)) break;
        mbar_arrive_expect_tx(&v_full[s], S::kTile);
#pragma unroll
        for (int bx = 0; bx < S::kBoxes; ++bx)
          tma_load_2d(base + S::kVOff + s * S::kTile + bx * S::kBox, &tmV, bx * 64,
                      k_row0 + i * kFuKeys, &v_full[s]);
        issued_v = i + 1;
      }
      if (issued_v < ntiles) set_flag(flags, KVS_FLAG_TIMEOUT);
      // copies still in flight must land before the CTA ends (the plain bound, even after
      // an abort: these are this CTA's own copies)
      if (!mbar_wait(q_full, 0)) set_flag(flags, KVS_FLAG_TIMEOUT);
      for (int i = issued_k > ST ? issued_k - ST : 0; i < issued_k; ++i)
        if (!mbar_wait(&k_full[i % ST], (i / ST) & 1)) set_flag(flags, KVS_FLAG_TIMEOUT);
      for (int i = issued_v > ST ? issued_v - ST : 0; i < issued_v; ++i)
        if (!mbar_wait(&v_full[i % ST], (i / ST) & 1)) set_flag(flags, KVS_FLAG_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16_f32(128, kFuKeys);
      constexpr uint32_t idesc_pv = umma_idesc_bf16_f32_bmn(128, D);
      const uint32_t q_addr = smem_u32(base + S::kQOff);
      const uint32_t ph_addr = smem_u32(base + S::kPOff);
      const uint32_t pl_addr = ph_addr + S::kPBytes;
      const uint32_t o_tmem = tmem + 256;
      int qk_done = 0, pv_issued = 0;
      // O += P_hi V + P_lo V for tile j (V MN-major: keys are the K dimension)
      auto issue_pv = [&](int j) -> bool {
        const int vs = j % ST;
        if (!mbar_wait_ab(p_full, j & 1, s_abort) ||
            !mbar_wait_ab(&v_full[vs], (j / ST) & 1, s_abort))
          return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(base + S::kVOff + vs * S::kTile);
#pragma unroll
        for (int ks = 0; ks < kFuKeys / 16; ++ks) {
          const uint32_t a_off = (uint32_t)((ks >> 2) * S::kBox + (ks & 3) * 32);
          const uint64_t bdesc = umma_desc_mn_sw128(v_addr + ks * 2048, S::kBox);
          umma_bf16_ss(o_tmem, umma_desc_k_sw128(ph_addr + a_off), bdesc, idesc_pv,
                       (j > 0 || ks > 0) ? 1u : 0u);
          umma_bf16_ss(o_tmem, umma_desc_k_sw128(pl_addr + a_off), bdesc, idesc_pv, 1u);
        }
        umma_commit(pv_done);
        umma_commit(&v_empty[vs]);
        pv_issued = j + 1;
        return true;
      };
      bool ok = mbar_wait_ab(q_full, 0, s_abort);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % ST, buf = i & 1;
        if (!mbar_wait_ab(&k_full[s], (i / ST) & 1, s_abort) ||
            (i >= 2 && !mbar_wait_ab(&s_empty[buf], ((i / 2) - 1) & 1, s_abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(base + S::kKOff + s * S::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (uint32_t)((ks >> 2) * S::kBox + (ks & 3) * 32);
          umma_bf16_ss(tmem + buf * kFuKeys, umma_desc_k_sw128(q_addr + off),
                       umma_desc_k_sw128(k_addr + off), idesc_qk, ks > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[buf]);
        umma_commit(&k_empty[s]);
        qk_done = i + 1;
        if (i >= 1) ok = issue_pv(i - 1);
      }
      if (ok && ntiles > 0) ok = issue_pv(ntiles - 1);
      if (!ok) set_flag(flags, KVS_FLAG_TIMEOUT);
      // the last MMAs must finish before the tensor memory is released
      if (qk_done > 0 && !mbar_wait(&s_full[(qk_done - 1) & 1], ((qk_done - 1) / 2) & 1))
        set_flag(flags, KVS_FLAG_TIMEOUT);
      if (pv_issued > 0 && !mbar_wait(pv_done, (pv_issued - 1) & 1))
        set_flag(flags, KVS_FLAG_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps ----------------
    // warp 2 + sw reads lane quarter (warp & 3): window-query row r = 32 quarter + lane,
    // key columns [64 half, 64 half + 64) of each tile, and O columns
    // [D/2 half, D/2 half + D/2)
    constexpr int NC = kFuKeys / 2;
    constexpr int OC = D / 2;
    const int sw = warp - 2, quarter = warp & 3, half = sw >> 2;
    const int c0w = half * NC;
    const int r = quarter * 32 + lane;
    const int st = tid - 64;
    const int pos = L - W + (r % W);
    const bool row_ok = r < Qn && pos >= 0;
    const float qscale = kLog2e / sqrtf((float)D);
    const float* lnh = logn ? logn + (size_t)unit * T_cap : nullptr;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t o_cols = tmem + lane_base + 256 + half * OC;
    unsigned char* p_hi = base + S::kPOff;
    unsigned char* p_lo = p_hi + S::kPBytes;
    float m_ref = -INFINITY, l = 0.f;
    bool live = true;
    float ln_next = (lnh && st < kFuKeys && t0 + st < t1) ? lnh[t0 + st] : 0.f;
    for (int i = 0; i < ntiles; ++i) {
      const int buf = i & 1;
      const int tb = t0 + i * kFuKeys;
      const float ln_cur = ln_next;
      if (lnh && st < kFuKeys) ln_next = (tb + kFuKeys + st < t1) ? lnh[tb + kFuKeys + st] : 0.f;
      live = live && mbar_wait_ab(&s_full[buf], (i / 2) & 1, s_abort);
      live = __all_sync(0xffffffffu, live);      // tcgen05.ld is warp-collective
      float sv[NC];
      if (live) {
        tc_fence_after();
        const uint32_t ta = tmem + lane_base + (uint32_t)(buf * kFuKeys + c0w);
#pragma unroll
        for (int c = 0; c < NC / 32; ++c) {
          float part[32];
          tmem_ld32(ta + c * 32, part);
#pragma unroll
          for (int j = 0; j < 32; ++j) sv[c * 32 + j] = part[j];
        }
      } else {
#pragma unroll
        for (int j = 0; j < NC; ++j) sv[j] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[buf]);
      if (st < kFuKeys) lns[st] = ln_cur * kLog2e;
      named_bar(1, kFuSoftThreads);                // (a) the tile's log-counts
      // logits in the log2 domain; masks only on the split's last tile and on keys the
      // causal window hides from some queries
      const bool interior = tb + kFuKeys <= t1 && tb + kFuKeys - 1 <= L - W;
      float pm = -INFINITY;
      if (interior && row_ok && live) {
#pragma unroll
        for (int j = 0; j < NC; j += 4) {
          const float4 lv = *reinterpret_cast<const float4*>(&lns[c0w + j]);
          sv[j] = fmaf(sv[j], qscale, lv.x);
          sv[j + 1] = fmaf(sv[j + 1], qscale, lv.y);
          sv[j + 2] = fmaf(sv[j + 2], qscale, lv.z);
          sv[j + 3] = fmaf(sv[j + 3], qscale, lv.w);
        }
      } else {
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          const int t = tb + c0w + j;
          const bool vis = live && row_ok && t < t1 && t <= pos;
          sv[j] = vis ? fmaf(sv[j], qscale, lns[c0w + j]) : -INFINITY;
        }
      }
      {
        float tm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) tm[k] = sv[k];
#pragma unroll
        for (int j = 8; j < NC; ++j) tm[j & 7] = fmaxf(tm[j & 7], sv[j]);
        pm = fmaxf(fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3])),
                   fmaxf(fmaxf(tm[4], tm[5]), fmaxf(tm[6], tm[7])));
      }
      xch[half * 128 + r] = pm;
      named_bar(1, kFuSoftThreads);                // (b) both halves' maxima
      const float mt = fmaxf(pm, xch[(1 - half) * 128 + r]);
      // the reference maximum moves only when the tile exceeds it by 2^8
      const float m_new = (mt > m_ref + kRescaleSlack) ? mt : m_ref;
      const bool resc = m_new != m_ref && m_ref > -INFINITY;
      const float cfac = resc ? ex2_ftz(m_ref - m_new) : 1.f;
      float psum[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) psum[k] = 0.f;
      if (m_new > -INFINITY) {
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          sv[j] = ex2_ftz(sv[j] - m_new);          // -inf -> 0
          psum[j & 7] += sv[j];
        }
      } else {
#pragma unroll
        for (int j = 0; j < NC; ++j) sv[j] = 0.f;
      }
      l = l * cfac + (((psum[0] + psum[1]) + (psum[2] + psum[3])) +
                      ((psum[4] + psum[5]) + (psum[6] + psum[7])));
      // P of this tile replaces the previous one: the previous tile's P V MMAs (which
      // also update O) must be done
      if (i > 0) live = live && mbar_wait_ab(pv_done, (i - 1) & 1, s_abort);
      live = __all_sync(0xffffffffu, live);
      if (live && __any_sync(0xffffffffu, resc)) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < OC / 32; ++c) {
          float ov[32];
          tmem_ld32(o_cols + c * 32, ov);
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] *= cfac;
          tmem_st32(o_cols + c * 32, ov);
        }
        tc_fence_before();
      }
      // P as bf16 hi and lo parts, 128-byte swizzled K-major rows (the MMA's A operand)
#pragma unroll
      for (int k = 0; k < NC / 8; ++k) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = sv[8 * k + 2 * e], c = sv[8 * k + 2 * e + 1];
          hi[e] = pack_bf16x2(a, c);
          lo[e] = pack_bf16x2(a - bf16_lo(hi[e]), c - bf16_hi(hi[e]));
        }
        const uint32_t off = (uint32_t)(half * S::kBox) + swz128(r, k);
        *reinterpret_cast<uint4*>(p_hi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(p_lo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      // value rows past the split's end may hold anything (even non-finite): zero them,
      // since their probability is 0 and 0 x inf is not
      const int nvalid = min(kFuKeys, t1 - tb);
      if (nvalid < kFuKeys) {
        const int vs = i % ST;
        const bool vok = mbar_wait_ab(&v_full[vs], (i / ST) & 1, s_abort);
        if (vok) {
          unsigned char* vt = base + S::kVOff + vs * S::kTile;
          const int nz = (kFuKeys - nvalid) * S::kBoxes * 8;   // 16-byte chunks
          for (int idx = st; idx < nz; idx += kFuSoftThreads) {
            const int rr = nvalid + idx / (S::kBoxes * 8);
            const int rem = idx % (S::kBoxes * 8);
            *reinterpret_cast<uint4*>(vt + (rem >> 3) * S::kBox + rr * 128 + (rem & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
        } else {
          live = false;
        }
      }
      fence_proxy_async_smem();                    // generic writes -> tensor-core reads
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      m_ref = m_new;
    }
    if (!live) set_flag(flags, KVS_FLAG_TIMEOUT);
    // per-split outputs: (m, l) per query row and the unnormalised O row
    float oreg[OC];
#pragma unroll
    for (int j = 0; j < OC; ++j) oreg[j] = 0.f;
    bool got = ntiles > 0 && live && mbar_wait_ab(pv_done, (ntiles - 1) & 1, s_abort);
    got = __all_sync(0xffffffffu, got);
    if (got) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < OC / 32; ++c) {
        float ov[32];
        tmem_ld32(o_cols + c * 32, ov);
#pragma unroll
        for (int j = 0; j < 32; ++j) oreg[c * 32 + j] = ov[j];
      }
    } else if (ntiles > 0) {
      set_flag(flags, KVS_FLAG_TIMEOUT);
    }
    named_bar(1, kFuSoftThreads);                  // every read of xch is done
    xch[half * 128 + r] = l;
    named_bar(1, kFuSoftThreads);
    if (r < Qn) {
      const float ltot = l + xch[(1 - half) * 128 + r];
      const bool any = row_ok && m_ref > -INFINITY && ltot > 0.f && got;
      const size_t prow = ((size_t)unit * nsplit + split) * Qn + r;
      if (half == 0) {
        part_ml[prow * 2 + 0] = any ? m_ref : -INFINITY;
        part_ml[prow * 2 + 1] = any ? ltot : 0.f;
      }
      float* po = part_o + prow * D + half * OC;
#pragma unroll
      for (int j = 0; j < OC; j += 4)
        *reinterpret_cast<float4*>(po + j) = any ? make_float4(oreg[j], oreg[j + 1], oreg[j + 2], oreg[j + 3])
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kFaTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Combine: per KV head, the splits' (m, l, O) -> (M, L) and o_q per window query,
// |o_q|^2, o_q as bf16 hi / lo rows, and o_bar = mean_q o_q
// ---------------------------------------------------------------------------

template <int D>
__global__ void __launch_bounds__(D)
fa_combine_kernel(const float* __restrict__ part_ml, const float* __restrict__ part_o, int Qn,
                  int nsplit, float* __restrict__ stats, float* __restrict__ obar,
                  float* __restrict__ zq_out, float* __restrict__ wq_out, bf16* __restrict__ eq_hi,
                  bf16* __restrict__ eq_lo) {
  extern __shared__ float fac[];                 // [Qn][nsplit] split weights 2^(m - M) / L
  __shared__ float s_z[D / 32][128], s_w[D / 32][128];
  __shared__ int s_valid;
  const int unit = blockIdx.x, c = threadIdx.x, lane = c & 31, wid = c >> 5;
  if (c == 0) s_valid = 0;
  __syncthreads();
  for (int q = c; q < Qn; q += D) {
    const float* e = part_ml + (size_t)unit * nsplit * Qn * 2;
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) {
      const float ls = e[((size_t)s * Qn + q) * 2 + 1];
      if (ls > 0.f) M = fmaxf(M, e[((size_t)s * Qn + q) * 2]);
    }
    float Ls = 0.f;
    if (M > -INFINITY)
      for (int s = 0; s < nsplit; ++s) {
        const float ls = e[((size_t)s * Qn + q) * 2 + 1];
        if (ls > 0.f) Ls = fmaf(ls, exp2f(e[((size_t)s * Qn + q) * 2] - M), Ls);
      }
    const bool valid = Ls > 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const float ls = e[((size_t)s * Qn + q) * 2 + 1];
      fac[q * nsplit + s] = (valid && ls > 0.f) ? exp2f(e[((size_t)s * Qn + q) * 2] - M) / Ls : 0.f;
    }
    stats[((size_t)unit * Qn + q) * 2 + 0] = M;
    stats[((size_t)unit * Qn + q) * 2 + 1] = Ls;
    if (valid) atomicAdd(&s_valid, 1);
  }
  __syncthreads();
  const float* po = part_o + (size_t)unit * nsplit * Qn * D;
  auto o_of = [&](int q) {
    float o = 0.f;
    for (int s = 0; s < nsplit; ++s) o = fmaf(fac[q * nsplit + s], po[((size_t)s * Qn + q) * D + c], o);
    return o;
  };
  float acc = 0.f;
  for (int q = 0; q < Qn; ++q) acc += o_of(q);
  const float ob = s_valid > 0 ? acc / (float)s_valid : 0.f;
  obar[(size_t)unit * D + c] = ob;
  // o_q relative to o_bar, for the per-query window form: e_q = o_q - o_bar as bf16 hi / lo
  // rows (rows past Qn are zero), |e_q|^2 and o_bar . e_q
  for (int q = 0; q < 128; ++q) {
    const float e = q < Qn ? o_of(q) - ob : 0.f;
    const bf16 hi = __float2bfloat16_rn(e);
    const size_t at = ((size_t)unit * 128 + q) * D + c;
    eq_hi[at] = hi;
    eq_lo[at] = __float2bfloat16_rn(e - __bfloat162float(hi));
    const float z = warp_sum(e * e), wv = warp_sum(ob * e);
    if (lane == 0) {
      s_z[wid][q] = z;
      s_w[wid][q] = wv;
    }
  }
  __syncthreads();
  for (int q = c; q < 128; q += D) {
    float z = 0.f, wv = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) {
      z += s_z[w][q];
      wv += s_w[w][q];
    }
    zq_out[(size_t)unit * 128 + q] = z;
    wq_out[(size_t)unit * 128 + q] = wv;
  }
}

// ---------------------------------------------------------------------------
// Pass B: window mass and pair scores over the candidate span
// ---------------------------------------------------------------------------

template <int D, bool PERQ>
struct ScShape {
  static constexpr int kBoxes = D / 64;
  static constexpr int kBox = 128 * 128;
  static constexpr int kTile = kBoxes * kBox;
  static constexpr int kStages = PERQ ? (D == 128 ? 1 : 2) : 2;
  static constexpr int kQOff = 0;
  static constexpr int kOOff = kTile;                        // per query form: O_hi, O_lo
  static constexpr int kStageOff = kOOff + (PERQ ? 2 * kTile : 0);
  static constexpr int kStageBytes = 2 * kTile;              // K tile, then V tile
  static constexpr int kSmallOff = kStageOff + kStages * kStageBytes;
  // barriers (128 B), Z_q = M_q + log2 L_q [128], o_bar [D], |e_q|^2 and o_bar . e_q
  // [2][128] (per query form),
  // per-key partial window mass [2 bufs][2 halves][128], per-pair terms [64][4],
  // per-pair partial norms [2 halves][64][3], tensor-memory address and abort flag
  static constexpr int kBarBytes = 128;
  static constexpr int kZOff = kSmallOff + kBarBytes;         // Z_q [128]
  static constexpr int kObOff = kZOff + 128 * 4;              // o_bar [D <= 128]
  static constexpr int kOn2Off = kObOff + 128 * 4;            // |e_q|^2, o_bar.e_q [2][128]
  static constexpr int kAbarOff = kOn2Off + (PERQ ? 2 * 128 * 4 : 0);
  static constexpr int kTermOff = kAbarOff + (PERQ ? 0 : 4 * 128 * 4);
  static constexpr int kNormOff = kTermOff + (PERQ ? 64 * 4 * 4 : 0);
  static constexpr int kQmodOff = kNormOff + (PERQ ? 2 * 64 * 3 * 4 : 0);   // q mod W [128]
  static constexpr int kMiscOff = kQmodOff + 128 * 4;
  static constexpr int kSmem = kMiscOff + 16 + 1024;
  static_assert(kSmem <= 232448, "shared memory");
};

constexpr uint32_t kScTmemCols = 512;   // S^T0 [0,128), S^T1 [128,256), U [256,384)

// One pair's norms -> (w_b, score), the closed forms of the forward-only objective.
__device__ __forceinline__ void pair_weight_score(float n11, float n12, float n22, float dd,
                                                  int form, float& w, float& s) {
  if (form == KVS_FORM_DIAGONAL) n12 = 0.f;
  const float den = n11 - 2.f * n12 + n22;
  const bool ok = isfinite(n11) && isfinite(n12) && isfinite(n22) && isfinite(den) &&
                  den > 1e-6f * (n11 + n22);
  if (ok) {
    w = (n22 - n12) / den;
    s = dd * (n11 * n22 - n12 * n12) / den;
  } else {
    w = 0.5f;
    s = dd * (n11 + 2.f * n12 + n22) * 0.25f;
  }
}

template <int D, bool PERQ>
__global__ void __launch_bounds__(kFuThreads, 1)
window_score_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmOh,
                    const __grid_constant__ CUtensorMap tmOl, const float* __restrict__ logn,
                    const int32_t* __restrict__ len, const int32_t* __restrict__ cand_begin,
                    int n_recent, int H_kv, int H_q, int W, int T_cap, int nsplit, int form,
                    const float* __restrict__ stats, const float* __restrict__ obar,
                    const float* __restrict__ on2g, const float* __restrict__ wqg,
                    float* __restrict__ score,
                    float* __restrict__ w_b, int32_t* __restrict__ flags) {
  using S = ScShape<D, PERQ>;
  constexpr int ST = S::kStages;
  extern __shared__ unsigned char dsm[];
  unsigned char* base = align1024(dsm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::kSmallOff);
  uint64_t* q_full = bars;              // 1 (Q and, per query, O_hi / O_lo)
  uint64_t* full = q_full + 1;          // ST: K and V tiles of a stage landed
  uint64_t* empty = full + ST;          // ST: every softmax warp is done with the stage
  uint64_t* s_full = empty + ST;        // 2
  uint64_t* s_empty = s_full + 2;       // 2
  uint64_t* u_full = s_empty + 2;       // 1 (per query form)
  uint64_t* u_empty = u_full + 1;       // 1
  float* zq = reinterpret_cast<float*>(base + S::kZOff);
  float* obs = reinterpret_cast<float*>(base + S::kObOff);
  float* on2 = reinterpret_cast<float*>(base + S::kOn2Off);     // |e_q|^2, then o_bar . e_q
  float* abar = reinterpret_cast<float*>(base + S::kAbarOff);     // [2][2][128]
  float* terms = reinterpret_cast<float*>(base + S::kTermOff);    // [64][4]
  float* norms = reinterpret_cast<float*>(base + S::kNormOff);    // [2][64][3]
  int* qmod = reinterpret_cast<int*>(base + S::kQmodOff);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(base + S::kMiscOff);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int unit = blockIdx.y, split = blockIdx.x;
  const int b = unit / H_kv, h = unit - b * H_kv;
  const int G = H_q / H_kv, Qn = G * W;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int L = len[unit];
  const int c0 = cand_begin[unit];
  if (L < 0 || L > T_cap || c0 < 0) L = -1;       // skipped (the window pass flags it)
  const int span = L - n_recent - c0;
  const int P = (L >= 0 && span > 0) ? span / 2 : 0;
  const int ntot = (2 * P + kFuKeys - 1) / kFuKeys;   // candidate tiles of the head
  const int tbeg = (int)((long long)split * ntot / nsplit);
  const int tend = (int)((long long)(split + 1) * ntot / nsplit);
  const int ntiles = tend - tbeg;
  if (ntiles <= 0) return;                           // uniform over the CTA
  const int q_row0 = (b * H_q + h * G) * W;
  const int o_row0 = unit * 128;
  const int k_row0 = unit * T_cap + c0 + tbeg * kFuKeys;

  if (tid == 0) {
    *s_abort = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFuSoft);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], kFuSoft);
    }
    mbar_init(u_full, 1);
    mbar_init(u_empty, kFuSoft);
    fence_mbar_init();
  }
  // per-query constants: Z_q = M_q + log2 L_q (+inf: query without a visible key)
  for (int q = tid; q < 128; q += kFuThreads) {
    float z = INFINITY;
    if (q < Qn) {
      const float M = stats[((size_t)unit * Qn + q) * 2], Ls = stats[((size_t)unit * Qn + q) * 2 + 1];
      if (Ls > 0.f && isfinite(M) && isfinite(Ls)) z = M + __log2f(Ls);
    }
    zq[q] = z;
    qmod[q] = q % W;
    obs[q] = q < D ? obar[(size_t)unit * D + q] : 0.f;
    if (PERQ) {
      on2[q] = on2g[(size_t)unit * 128 + q];
      on2[128 + q] = wqg[(size_t)unit * 128 + q];
    }
  }
  if (warp == 1) tmem_alloc(s_tmem, kScTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  int qv = 0;                                        // window queries with a visible key
  for (int q = 0; q < min(Qn, 128); ++q) qv += zq[q] < INFINITY;
  const float inv_qv = qv > 0 ? 1.f / (float)qv : 0.f;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const uint32_t qbytes = PERQ ? 3 * S::kTile : S::kTile;
      mbar_arrive_expect_tx(q_full, qbytes);
#pragma unroll
      for (int bx = 0; bx < S::kBoxes; ++bx) {
        tma_load_2d(base + S::kQOff + bx * S::kBox, &tmQ, bx * 64, q_row0, q_full);
        if (PERQ) {
          tma_load_2d(base + S::kOOff + bx * S::kBox, &tmOh, bx * 64, o_row0, q_full);
          tma_load_2d(base + S::kOOff + S::kTile + bx * S::kBox, &tmOl, bx * 64, o_row0, q_full);
        }
      }
      // tiles beyond the ring are prefetched into L2, kPrefetch tiles ahead
      auto prefetch = [&](int i) {
        if (i < ntiles)
#pragma unroll
          for (int bx = 0; bx < S::kBoxes; ++bx) {
            tma_prefetch_2d(&tmK, bx * 64, k_row0 + i * kFuKeys);
            tma_prefetch_2d(&tmV, bx * 64, k_row0 + i * kFuKeys);
          }
      };
      for (int i = ST; i < ST + kPrefetch; ++i) prefetch(i);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % ST;
        prefetch(i + ST + kPrefetch);
        if (i >= ST && !mbar_wait_ab(&empty[s], ((i / ST) - 1) & 1, s_abort)) break;
        unsigned char* stg = base + S::kStageOff + s * S::kStageBytes;
        mbar_arrive_expect_tx(&full[s], S::kStageBytes);
#pragma unroll
        for (int bx = 0; bx < S::kBoxes; ++bx) {
          tma_load_2d(stg + bx * S::kBox, &tmK, bx * 64, k_row0 + i * kFuKeys, &full[s]);
          tma_load_2d(stg + S::kTile + bx * S::kBox, &tmV, bx * 64, k_row0 + i * kFuKeys, &full[s]);
        }
        issued = i + 1;
      }
      if (issued < ntiles) set_flag(flags, KVS_FLAG_TIMEOUT);
      if (!mbar_wait(q_full, 0)) set_flag(flags, KVS_FLAG_TIMEOUT);
      for (int i = issued > ST ? issued - ST : 0; i < issued; ++i)
        if (!mbar_wait(&full[i % ST], (i / ST) & 1)) set_flag(flags, KVS_FLAG_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer: S^T = K Q^T (and U = V O^T) ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(kFuKeys, 128);
      const uint32_t q_addr = smem_u32(base + S::kQOff);
      const uint32_t oh_addr = smem_u32(base + S::kOOff);
      const uint32_t ol_addr = oh_addr + S::kTile;
      bool ok = mbar_wait_ab(q_full, 0, s_abort);
      int done = 0;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % ST, buf = i & 1;
        if (!mbar_wait_ab(&full[s], (i / ST) & 1, s_abort) ||
            (i >= 2 && !mbar_wait_ab(&s_empty[buf], ((i / 2) - 1) & 1, s_abort)) ||
            (PERQ && i >= 1 && !mbar_wait_ab(u_empty, (i - 1) & 1, s_abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(base + S::kStageOff + s * S::kStageBytes);
        const uint32_t v_addr = k_addr + S::kTile;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (uint32_t)((ks >> 2) * S::kBox + (ks & 3) * 32);
          umma_bf16_ss(tmem + buf * kFuKeys, umma_desc_k_sw128(k_addr + off),
                       umma_desc_k_sw128(q_addr + off), idesc, ks > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[buf]);
        if (PERQ) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (uint32_t)((ks >> 2) * S::kBox + (ks & 3) * 32);
            umma_bf16_ss(tmem + 256, umma_desc_k_sw128(v_addr + off),
                         umma_desc_k_sw128(oh_addr + off), idesc, ks > 0 ? 1u : 0u);
            umma_bf16_ss(tmem + 256, umma_desc_k_sw128(v_addr + off),
                         umma_desc_k_sw128(ol_addr + off), idesc, 1u);
          }
          umma_commit(u_full);
        }
        done = i + 1;
      }
      if (!ok) set_flag(flags, KVS_FLAG_TIMEOUT);
      if (done > 0 && !mbar_wait(&s_full[(done - 1) & 1], ((done - 1) / 2) & 1))
        set_flag(flags, KVS_FLAG_TIMEOUT);
      if (PERQ && done > 0 && !mbar_wait(u_full, (done - 1) & 1)) set_flag(flags, KVS_FLAG_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps ----------------
    // warp 2 + sw owns lane quarter (warp & 3): key row kr = 32 quarter + lane of each
    // tile, and window-query columns [64 half, 64 half + 64)
    constexpr int NC = 64;
    const int sw = warp - 2, quarter = warp & 3, half = sw >> 2;
    const int kr = quarter * 32 + lane;
    const int st = tid - 64;
    const int qc0 = half * NC;
    const float qscale = kLog2e / sqrtf((float)D);
    const float* lnh = logn ? logn + (size_t)unit * T_cap : nullptr;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    // pair-term threads: pair pp of the tile, quarter part of the head dimension
    const int pp = st >> 2, part = st & 3;
    constexpr int DP = D / 4;                     // dims per part: 32 or 16
    const float* ob = obs + part * DP;
    bool live = true;
    const int first_row = c0 + tbeg * kFuKeys;   // cache row of key 0 of tile 0
    float ln_next = 0.f;
    if (lnh && tbeg * kFuKeys + kr < 2 * P) ln_next = lnh[first_row + kr];
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % ST, buf = i & 1;
      const int tile = tbeg + i;
      const int krow = tile * kFuKeys + kr;       // this thread's key, relative to c0
      const int t = c0 + krow;                    // its cache row
      const bool kval = krow < 2 * P;
      const float lnt = ln_next * kLog2e;
      if (lnh && i + 1 < ntiles) {
        const int kn = krow + kFuKeys;
        ln_next = kn < 2 * P ? lnh[c0 + kn] : 0.f;
      }
      live = live && mbar_wait_ab(&s_full[buf], (i / 2) & 1, s_abort);
      live = __all_sync(0xffffffffu, live);
      float sv[NC];
      if (live) {
        tc_fence_after();
        const uint32_t ta = tmem + lane_base + (uint32_t)(buf * kFuKeys + qc0);
        tmem_ld32(ta, *reinterpret_cast<float(*)[32]>(sv));
        tmem_ld32(ta + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
      } else {
#pragma unroll
        for (int j = 0; j < NC; ++j) sv[j] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[buf]);
      // p_qt = 2^(s q.k + lnt - Z_q); query q sees the key when t <= L - W + (q mod W)
      if (kval) {
#pragma unroll
        for (int j = 0; j < NC; j += 2) {
          const float2 z = *reinterpret_cast<const float2*>(&zq[qc0 + j]);
          const float2 x = ffma2(make_float2(sv[j], sv[j + 1]), make_float2(qscale, qscale),
                                 make_float2(lnt - z.x, lnt - z.y));
          sv[j] = ex2_ftz(x.x);
          sv[j + 1] = ex2_ftz(x.y);
        }
        const int hide = t - (L - W);             // queries with q mod W < hide miss it
        if (hide > 0) {
#pragma unroll
          for (int j = 0; j < NC; ++j)
            if (qmod[qc0 + j] < hide) sv[j] = 0.f;
        }
      } else {
#pragma unroll
        for (int j = 0; j < NC; ++j) sv[j] = 0.f;
      }
      const unsigned char* kt = base + S::kStageOff + s * S::kStageBytes;
      const unsigned char* vt = kt + S::kTile;
      bool sok = live && mbar_wait_ab(&full[s], (i / ST) & 1, s_abort);   // K, V rows landed
      sok = __all_sync(0xffffffffu, sok);
      live = live && sok;
      if constexpr (!PERQ) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < NC; ++j) acc[j & 3] += sv[j];
        abar[(buf * 2 + half) * 128 + kr] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        named_bar(1, kFuSoftThreads);
      }
      // the tile's pair pp: rows 2 pp, 2 pp + 1; this thread: dims [DP part, DP part + DP):
      // |k_b - k_a|^2, |v_a - o_bar|^2, |v_b - o_bar|^2, |v_a + v_b - 2 o_bar|^2
      float dd = 0.f, ea = 0.f, eb = 0.f, ec = 0.f;
      const int ra = 2 * pp, rb = ra + 1;
#pragma unroll
      for (int ch = 0; ch < DP / 8; ++ch) {
        const int dim = part * DP + ch * 8;
        const int bx = dim >> 6, cc = (dim & 63) >> 3;
        const uint4 ka = *reinterpret_cast<const uint4*>(kt + bx * S::kBox + swz128(ra, cc));
        const uint4 kb = *reinterpret_cast<const uint4*>(kt + bx * S::kBox + swz128(rb, cc));
        const uint4 va = *reinterpret_cast<const uint4*>(vt + bx * S::kBox + swz128(ra, cc));
        const uint4 vb = *reinterpret_cast<const uint4*>(vt + bx * S::kBox + swz128(rb, cc));
        const uint32_t kaw[4] = {ka.x, ka.y, ka.z, ka.w}, kbw[4] = {kb.x, kb.y, kb.z, kb.w};
        const uint32_t vaw[4] = {va.x, va.y, va.z, va.w}, vbw[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 o2 = *reinterpret_cast<const float2*>(ob + ch * 8 + 2 * e);
          const float2 dk = make_float2(bf16_lo(kbw[e]) - bf16_lo(kaw[e]), bf16_hi(kbw[e]) - bf16_hi(kaw[e]));
          const float2 ra2 = make_float2(bf16_lo(vaw[e]) - o2.x, bf16_hi(vaw[e]) - o2.y);
          const float2 rb2 = make_float2(bf16_lo(vbw[e]) - o2.x, bf16_hi(vbw[e]) - o2.y);
          const float2 rc2 = fadd2(ra2, rb2);
          dd = fmaf(dk.x, dk.x, fmaf(dk.y, dk.y, dd));
          ea = fmaf(ra2.x, ra2.x, fmaf(ra2.y, ra2.y, ea));
          eb = fmaf(rb2.x, rb2.x, fmaf(rb2.y, rb2.y, eb));
          ec = fmaf(rc2.x, rc2.x, fmaf(rc2.y, rc2.y, ec));
        }
      }
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        dd += __shfl_xor_sync(0xffffffffu, dd, o);
        ea += __shfl_xor_sync(0xffffffffu, ea, o);
        eb += __shfl_xor_sync(0xffffffffu, eb, o);
        ec += __shfl_xor_sync(0xffffffffu, ec, o);
      }
      const int pglob = tile * (kFuKeys / 2) + pp;
      if constexpr (!PERQ) {
        if (part == 0 && pglob < P && live) {
          const float* ab = abar + buf * 256;
          const float aa = (ab[ra] + ab[128 + ra]) * inv_qv;
          const float bb = (ab[rb] + ab[128 + rb]) * inv_qv;
          const float n11 = fabsf(aa * (1.f - 2.f * aa)) * sqrtf(ea);
          const float n22 = fabsf(bb * (1.f - 2.f * bb)) * sqrtf(eb);
          const float n12 = aa * bb * sqrtf(ec);
          float w, sc;
          pair_weight_score(n11, n12, n22, dd, form, w, sc);
          const size_t at = (size_t)unit * (T_cap / 2) + pglob;
          score[at] = sc;
          w_b[at] = w;
        }
      } else {
        // per-query window form: U = V E^T gives v_t . e_q on the key's lane
        bool uok = live && mbar_wait_ab(u_full, i & 1, s_abort);
        uok = __all_sync(0xffffffffu, uok);
        live = live && uok;
        float uv[NC];
        if (uok) {
          tc_fence_after();
          const uint32_t ta = tmem + lane_base + (uint32_t)(256 + qc0);
          tmem_ld32(ta, *reinterpret_cast<float(*)[32]>(uv));
          tmem_ld32(ta + 32, *reinterpret_cast<float(*)[32]>(uv + 32));
        } else {
#pragma unroll
          for (int j = 0; j < NC; ++j) uv[j] = 0.f;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(u_empty);
        if (part == 0) {
          terms[pp * 4 + 0] = dd;
          terms[pp * 4 + 1] = ea;
          terms[pp * 4 + 2] = eb;
          terms[pp * 4 + 3] = ec;
        }
        named_bar(1, kFuSoftThreads);
        // per window query of this half: lane a (even key) takes N11 and N12, lane b N22
        const int pl = kr >> 1;
        const bool is_a = (kr & 1) == 0;
        const float t_own = is_a ? terms[pl * 4 + 1] : terms[pl * 4 + 2];
        const float t_ab = terms[pl * 4 + 3];
        float n_self = 0.f, n_cpl = 0.f;
#pragma unroll 8
        for (int j = 0; j < NC; ++j) {
          const float p = sv[j], u = uv[j];
          const float p_o = __shfl_xor_sync(0xffffffffu, p, 1);
          const float u_o = __shfl_xor_sync(0xffffffffu, u, 1);
          const float z = on2[qc0 + j], wq = on2[128 + qc0 + j];
          n_self = fmaf(fabsf(p * (1.f - 2.f * p)),
                        sqrtf(fmaxf(0.f, fmaf(-2.f, u - wq, t_own) + z)), n_self);
          if (is_a)
            n_cpl = fmaf(p * p_o, sqrtf(fmaxf(0.f, fmaf(-4.f, u + u_o - 2.f * wq, t_ab) + 4.f * z)),
                         n_cpl);
        }
        norms[(half * 64 + pl) * 3 + (is_a ? 0 : 2)] = n_self;
        if (is_a) norms[(half * 64 + pl) * 3 + 1] = n_cpl;
        named_bar(1, kFuSoftThreads);
        if (part == 0 && pglob < P && live) {
          const float* n0 = norms + pp * 3;
          const float* n1 = norms + (64 + pp) * 3;
          const float n11 = (n0[0] + n1[0]) * inv_qv;
          const float n12 = (n0[1] + n1[1]) * inv_qv;
          const float n22 = (n0[2] + n1[2]) * inv_qv;
          float w, sc;
          pair_weight_score(n11, n12, n22, terms[pp * 4], form, w, sc);
          const size_t at = (size_t)unit * (T_cap / 2) + pglob;
          score[at] = sc;
          w_b[at] = w;
        }
        named_bar(1, kFuSoftThreads);             // terms / norms are rewritten next tile
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (!live) set_flag(flags, KVS_FLAG_TIMEOUT);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kScTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

static int fused_splits(int units) {
  int s = 148 / units;            // one CTA per SM, one wave
  if (s < 1) s = 1;
  return s;
}

bool window_fused_supported(const kvs_cache_desc& d, int W) {
  const unsigned long long rows = (unsigned long long)d.B * d.H_kv * (unsigned long long)d.T_cap;
  const unsigned long long qrows = (unsigned long long)d.B * d.H_q * (unsigned long long)W;
  const unsigned long long orows = (unsigned long long)d.B * d.H_kv * 128ull;
  return d.dtype == KVS_BF16 && (d.d == 64 || d.d == 128) && (d.H_q / d.H_kv) * W <= 128 &&
         rows < (1ull << 31) && qrows < (1ull << 31) && orows < (1ull << 31) &&
         tensor_map_encoder() != nullptr;
}

template <int D>
static cudaError_t launch_fused_t(const kvs_cache_desc& d, const void* K, const void* V,
                                  const float* logn, const int32_t* len,
                                  const int32_t* cand_begin, int n_recent, const void* Qw, int W,
                                  int form, int stats_form, const ScoreLayout& Ly, char* ws,
                                  float* score, float* w_b, cudaStream_t st) {
  const unsigned long long rows = (unsigned long long)d.B * d.H_kv * (unsigned long long)d.T_cap;
  const unsigned long long qrows = (unsigned long long)d.B * d.H_q * (unsigned long long)W;
  const int units = d.B * d.H_kv;
  bf16* oq_hi = reinterpret_cast<bf16*>(ws + Ly.oq_hi);
  bf16* oq_lo = reinterpret_cast<bf16*>(ws + Ly.oq_lo);
  CUtensorMap mQ, mK, mV, mOh, mOl;
  if (!encode_rows_map(&mQ, Qw, qrows, D, 128) || !encode_rows_map(&mK, K, rows, D, kFuKeys) ||
      !encode_rows_map(&mV, V, rows, D, kFuKeys) ||
      !encode_rows_map(&mOh, oq_hi, (unsigned long long)units * 128, D, 128) ||
      !encode_rows_map(&mOl, oq_lo, (unsigned long long)units * 128, D, 128))
    return cudaErrorInvalidValue;
  const int nsa = fused_splits(units) < Ly.nsplit ? fused_splits(units) : Ly.nsplit;
  const int Qn = Ly.Qn;
  int32_t* flags = reinterpret_cast<int32_t*>(ws);
  float* part_ml = reinterpret_cast<float*>(ws + Ly.part_ml);
  float* part_o = reinterpret_cast<float*>(ws + Ly.part_o);
  float* stats = reinterpret_cast<float*>(ws + Ly.stats);
  float* obar = reinterpret_cast<float*>(ws + Ly.obar);
  float* on2 = reinterpret_cast<float*>(ws + Ly.on2);
  float* owq = reinterpret_cast<float*>(ws + Ly.owq);

  auto ka = window_fa_kernel<D>;
  if (!ensure_smem_attr((const void*)ka, FaShape<D>::kSmem)) return cudaErrorInvalidValue;
  ka<<<dim3(nsa, units), kFuThreads, FaShape<D>::kSmem, st>>>(
      mQ, mK, mV, logn, len, d.H_kv, d.H_q, W, d.T_cap, nsa, part_ml, part_o, flags);
  const size_t csm = (size_t)Qn * nsa * sizeof(float);
  auto kc = fa_combine_kernel<D>;
  if (!ensure_smem_attr((const void*)kc, csm)) return cudaErrorInvalidValue;
  kc<<<units, D, csm, st>>>(part_ml, part_o, Qn, nsa, stats, obar, on2, owq, oq_hi, oq_lo);
  const int nsb = fused_splits(units);
  if (stats_form == KVS_FORM_PER_QUERY) {
    auto kb = window_score_kernel<D, true>;
    if (!ensure_smem_attr((const void*)kb, ScShape<D, true>::kSmem)) return cudaErrorInvalidValue;
    kb<<<dim3(nsb, units), kFuThreads, ScShape<D, true>::kSmem, st>>>(
        mQ, mK, mV, mOh, mOl, logn, len, cand_begin, n_recent, d.H_kv, d.H_q, W, d.T_cap, nsb,
        form, stats, obar, on2, owq, score, w_b, flags);
  } else {
    auto kb = window_score_kernel<D, false>;
    if (!ensure_smem_attr((const void*)kb, ScShape<D, false>::kSmem)) return cudaErrorInvalidValue;
    kb<<<dim3(nsb, units), kFuThreads, ScShape<D, false>::kSmem, st>>>(
        mQ, mK, mV, mOh, mOl, logn, len, cand_begin, n_recent, d.H_kv, d.H_q, W, d.T_cap, nsb,
        form, stats, obar, on2, owq, score, w_b, flags);
  }
  count_launches(3);
  return cudaGetLastError();
}

cudaError_t launch_score_fused(const kvs_cache_desc& d, const void* K, const void* V,
                               const float* logn, const int32_t* len, const int32_t* cand_begin,
                               int n_recent, const void* Qw, int W, int form, int stats_form,
                               const ScoreLayout& Ly, char* ws, float* score, float* w_b,
                               cudaStream_t st) {
  if (d.d == 128)
    return launch_fused_t<128>(d, K, V, logn, len, cand_begin, n_recent, Qw, W, form, stats_form,
                               Ly, ws, score, w_b, st);
  return launch_fused_t<64>(d, K, V, logn, len, cand_begin, n_recent, Qw, W, form, stats_form, Ly,
                            ws, score, w_b, st);
}

}  // namespace kvs
