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
//     multiplied by V) so that O keeps close to fp32 accuracy; it goes back into tensor
//     memory over the tile's S and feeds the P V MMAs from there. The reference maximum
//     of a row moves only when a tile exceeds it by 2^8 (the accumulator is then
//     rescaled in tensor memory), so P <= 2^8 between moves.
//   fa_query_kernel (per window query and KV head): the partials' (m, l, O) -> (M, L)
//     and o_q; fa_center_kernel: o_bar = mean_q o_q, and for pass B's per-query form
//     e_q = o_q - o_bar as bf16 hi / mid / lo rows with |e_q|^2 and o_bar . e_q.
//   pass B (window_score_kernel, per KV head and candidate split): S^T = K Q^T with the
//     keys on the tensor-memory lanes, so that a thread owns one key and its row of
//     window probabilities p_qt = 2^(s_qt - M_q) / L_q: alpha_bar_t is a sum over the
//     thread's own columns. A candidate pair is two adjacent rows of the same 128-row
//     tile (tiles start at the candidate span's first row), so the pair norms, weight
//     and score come straight from the K and V rows already in shared memory, the two
//     rows of a pair on two lanes of one warp.
//     Window form "mean" (the plain reading): the one-query norms at (alpha_bar, o_bar).
//     Window form "per query": the one-query norms of every window query, averaged.
//     With e_q = o_q - o_bar, |v - o_q|^2 = |v - o_bar|^2 - 2 (v.e_q - o_bar.e_q) + |e_q|^2
//     and |v_a + v_b - 2 o_q|^2 = |v_a + v_b - 2 o_bar|^2 - 4 (v_a.e_q + v_b.e_q
//     - 2 o_bar.e_q) + 4 |e_q|^2: the row terms are taken directly in fp32 as in the mean
//     form and U = V E^T (E as three bf16 parts) on the tensor cores. Where a query's
//     output sits near the row (attention concentrated on it), the expansion cancels:
//     its result is then far below the terms it is formed from, and the distance is
//     recomputed directly from the value rows and e_q (rarely: at most a few keys per
//     query can hold most of its attention).
//
// Warp roles (both passes): warp 0 issues the TMA loads (128-byte swizzle, no
// multicast), warp 1 owns the tensor memory and one of its threads issues tcgen05.mma,
// warps 2-5 and 6-9 are two softmax groups that take alternate tiles (one warp per
// tensor-memory lane quarter, one row per thread), each with its own tensor-memory
// buffers and barriers, so that no CTA-wide barrier sits in the per-tile path and one
// group computes while the other waits for its data. Every wait is bounded.
#include <cudaTypedefs.h>

#include "kvs_common.cuh"
#include "kvs_kernels.h"
#include "ptx.cuh"

namespace kvs {

constexpr int kFuKeys = 128;            // keys per tile
constexpr int kFuGroupWarps = 4;        // softmax warps per group: one per lane quarter
constexpr int kFuThreads = (2 + 2 * kFuGroupWarps) * 32;
constexpr float kRescaleSlack = 8.f;    // log2 units
constexpr uint32_t kFuTmemCols = 512;

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) &
                                          ~static_cast<uintptr_t>(1023));
}

// 16 consecutive 32-bit columns of this thread's tensor-memory lane, stored from registers
// (warp-collective) without waiting; tmem_st_wait() waits for all of the thread's stores.
__device__ __forceinline__ void tmem_st16_async(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// The same from every other register of w, starting at w[OFF] (16 columns).
template <int OFF>
__device__ __forceinline__ void tmem_st16_pairs(uint32_t taddr, const uint32_t (&w)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(w[OFF]), "r"(w[OFF + 2]), "r"(w[OFF + 4]), "r"(w[OFF + 6]), "r"(w[OFF + 8]),
      "r"(w[OFF + 10]), "r"(w[OFF + 12]), "r"(w[OFF + 14]), "r"(w[OFF + 16]), "r"(w[OFF + 18]),
      "r"(w[OFF + 20]), "r"(w[OFF + 22]), "r"(w[OFF + 24]), "r"(w[OFF + 26]), "r"(w[OFF + 28]),
      "r"(w[OFF + 30])
      : "memory");
}
// CW (16 or 32) consecutive fp32 columns of this thread's lane, loaded and waited for.
template <int CW>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, float (&v)[CW]) {
  if constexpr (CW == 32) {
    tmem_ld32(taddr, v);
  } else {
    static_assert(CW == 16, "chunk width");
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  }
}

// One fp32 column of this thread's lane (warp-collective), waited for.
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr) : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r) : : "memory");
  return __uint_as_float(r);
}

// Two columns of this thread's lane: store (no wait), and load (waits).
__device__ __forceinline__ void tmem_st2(uint32_t taddr, uint32_t a, uint32_t b) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(a), "r"(b)
               : "memory");
}
__device__ __forceinline__ void tmem_ld2(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(taddr)
               : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]) : : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 consecutive 32-bit columns of this thread's lane, loaded without waiting; the values
// are defined only after tmem_ld_wait on the same registers (which ties them to the wait,
// so that no use is scheduled before it).
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// ---------------------------------------------------------------------------
// Pass A: per-split softmax statistics and unnormalised window outputs
// ---------------------------------------------------------------------------

template <int D>
struct FaShape {
  static constexpr int kBoxes = D / 64;
  static constexpr int kBox = 128 * 128;                 // 128 rows x 128 bytes
  static constexpr int kTile = kBoxes * kBox;            // a Q, K or V tile
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr int kLnSlot = kFuKeys * 4 + 16;       // log-counts of a tile + their maximum
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTile;
  static constexpr int kVOff = kKOff + kStages * kTile;
  static constexpr int kLnOff = kVOff + kStages * kTile;
  static constexpr int kSmallOff = kLnOff + kStages * kLnSlot;
  static constexpr int kSmem = kSmallOff + 256 + 16 + 1024;   // barriers, misc, alignment
  static_assert(kSmem <= 232448, "shared memory");
  // TMA tile destinations with 128-byte swizzling start on 1024-byte boundaries; the
  // log-count slots take 16-byte vector stores; the barriers (1 + 4 ST + 6) fit 256 bytes
  static_assert(kKOff % 1024 == 0 && kVOff % 1024 == 0 && kTile % 1024 == 0, "tile alignment");
  static_assert(kLnOff % 16 == 0 && kLnSlot % 16 == 0 && kSmallOff % 8 == 0, "slot alignment");
  static_assert(8 * (1 + 4 * kStages + 6) <= 256, "barrier room");
};

// Tensor memory of pass A, per softmax group g: S_g at columns [128 g, 128 g + 128) --
// once read, a 32-key chunk c of it holds that chunk's P as bf16 pairs, hi in columns
// [32 c, 32 c + 16) and lo in [32 c + 16, 32 c + 32), the A operand of the group's P V
// MMAs -- and O_g at [256 + D g, 256 + D g + D).
template <int D>
__global__ void __launch_bounds__(kFuThreads, 1)
window_fa_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const float* __restrict__ logn,
                 const int32_t* __restrict__ len, int H_kv, int H_q, int W, int T_cap, int nsplit,
                 int cap_chunks, float* __restrict__ part_ml, float* __restrict__ part_o,
                 int32_t* __restrict__ flags) {
  using S = FaShape<D>;
  constexpr int ST = S::kStages;
  extern __shared__ unsigned char dsm[];
  unsigned char* base = align1024(dsm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::kSmallOff);
  uint64_t* q_full = bars;              // 1
  uint64_t* k_full = q_full + 1;        // ST
  uint64_t* k_empty = k_full + ST;      // ST: the QK^T MMA of the stage is done
  uint64_t* v_full = k_empty + ST;      // ST: V rows (TMA) and log-counts (producer lanes)
  uint64_t* v_empty = v_full + ST;      // ST: the P V MMAs of the stage are done
  uint64_t* s_full = v_empty + ST;      // 2 (per group)
  uint64_t* p_full = s_full + 2;        // 2: the group's four warps have written P
  uint64_t* pv_done = p_full + 2;       // 2: the group's P V MMAs of a tile are done
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(base + S::kSmallOff + 256);
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
  // split s takes one chunk of the head's rows: a share of its length, or (cap_chunks) of
  // the capacity, so that a head shorter than the capacity leaves its last CTAs idle
  int chunk = ((cap_chunks ? T_cap : L) + nsplit - 1) / nsplit;
  chunk = (chunk + kFuKeys - 1) / kFuKeys * kFuKeys;
  const int t0 = split * chunk, t1 = min(L, t0 + chunk);
  const int ntiles = t1 > t0 ? (t1 - t0 + kFuKeys - 1) / kFuKeys : 0;
  if (ntiles == 0) {   // nothing of the head in this split: an empty partial (uniform over the CTA)
    float* pm = part_ml + ((size_t)unit * nsplit + split) * Qn * 2;
    float* po = part_o + ((size_t)unit * nsplit + split) * Qn * D;
    for (int i = tid; i < Qn; i += kFuThreads) {
      pm[2 * i] = -INFINITY;
      pm[2 * i + 1] = 0.f;
    }
    for (int i = tid; i < Qn * D / 4; i += kFuThreads)
      reinterpret_cast<float4*>(po)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const int q_row0 = (b * H_q + h * G) * W;
  const int k_row0 = unit * T_cap + t0;
  const bool has_ln = logn != nullptr;
  const float* lnh = has_ln ? logn + (size_t)unit * T_cap : nullptr;

  if (tid == 0) {
    *s_abort = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1 + 32);     // the TMA transaction, then each producer lane
      mbar_init(&v_empty[s], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&p_full[g], kFuGroupWarps);
      mbar_init(&pv_done[g], 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(s_tmem, kFuTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ---------------- producer warp ----------------
    // lane 0 issues the TMA loads; every lane loads four log-counts of each tile into the
    // V stage's slot (plain loads, one tile ahead) and arrives on the stage's barrier
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(q_full, S::kTile);
#pragma unroll
      for (int bx = 0; bx < S::kBoxes; ++bx)
        tma_load_2d(base + S::kQOff + bx * S::kBox, &tmQ, bx * 64, q_row0, q_full);
    }
    auto ln4 = [&](int i) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (has_ln && i < ntiles) {
        const int t = t0 + i * kFuKeys + 4 * lane;
        v.x = t < t1 ? lnh[t] * kLog2e : 0.f;
        v.y = t + 1 < t1 ? lnh[t + 1] * kLog2e : 0.f;
        v.z = t + 2 < t1 ? lnh[t + 2] * kLog2e : 0.f;
        v.w = t + 3 < t1 ? lnh[t + 3] * kLog2e : 0.f;
      }
      return v;
    };
    float4 ln_next = ln4(0);
    int issued_k = 0, issued_v = 0;
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % ST;
      const uint32_t ph = ((i / ST) - 1) & 1;
      bool ok = true;
      if (lane == 0) {
        ok = i < ST || mbar_wait_ab(&k_empty[s], ph, s_abort);
        if (ok) {
          mbar_arrive_expect_tx(&k_full[s], S::kTile);
#pragma unroll
          for (int bx = 0; bx < S::kBoxes; ++bx)
            tma_load_2d(base + S::kKOff + s * S::kTile + bx * S::kBox, &tmK, bx * 64,
                        k_row0 + i * kFuKeys, &k_full[s]);
        }
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      issued_k = i + 1;
      ok = i < ST || mbar_wait_ab(&v_empty[s], ph, s_abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&v_full[s], S::kTile);
#pragma unroll
        for (int bx = 0; bx < S::kBoxes; ++bx)
          tma_load_2d(base + S::kVOff + s * S::kTile + bx * S::kBox, &tmV, bx * 64,
                      k_row0 + i * kFuKeys, &v_full[s]);
      }
      *reinterpret_cast<float4*>(base + S::kLnOff + s * S::kLnSlot + 16 * lane) = ln_next;
      {
        // the tile's largest log-count (entries past the split read as 0 <= every
        // log-count): with the row maximum of S it bounds the tile's logits from above
        float lm = fmaxf(fmaxf(ln_next.x, ln_next.y), fmaxf(ln_next.z, ln_next.w));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lm = fmaxf(lm, __shfl_xor_sync(0xffffffffu, lm, o));
        if (lane == 0)
          *reinterpret_cast<float*>(base + S::kLnOff + s * S::kLnSlot + kFuKeys * 4) = lm;
      }
      mbar_arrive(&v_full[s]);
      ln_next = ln4(i + 1);
      issued_v = i + 1;
    }
    if (lane == 0) {
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
      int pv_issued = 0;
      // O_g += P_hi V + P_lo V for tile j (group g = j & 1): P from the group's tensor
      // memory, V from the ring (MN-major: keys are the K dimension)
      auto issue_pv = [&](int j) -> bool {
        const int g = j & 1, kj = j >> 1, vs = j % ST;
        if (!mbar_wait_ab(&p_full[g], kj & 1, s_abort) ||
            !mbar_wait_ab(&v_full[vs], (j / ST) & 1, s_abort))
          return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(base + S::kVOff + vs * S::kTile);
        const uint32_t p_tm = tmem + (uint32_t)(g * kFuKeys);
        const uint32_t o_tm = tmem + 256 + (uint32_t)(g * D);
#pragma unroll
        for (int ks = 0; ks < kFuKeys / 16; ++ks) {
          const uint64_t bdesc = umma_desc_mn_sw128(v_addr + ks * 2048, S::kBox);
          const uint32_t a = p_tm + 32 * (ks >> 1) + 8 * (ks & 1);
          umma_bf16_ts(o_tm, a, bdesc, idesc_pv, (kj > 0 || ks > 0) ? 1u : 0u);
          umma_bf16_ts(o_tm, a + 16, bdesc, idesc_pv, 1u);
        }
        umma_commit(&pv_done[g]);
        umma_commit(&v_empty[vs]);
        pv_issued = j + 1;
        return true;
      };
      bool ok = mbar_wait_ab(q_full, 0, s_abort);
      for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % ST, g = i & 1, k = i >> 1;
        // S of tile i overwrites the P that the group's previous P V MMAs read
        if (!mbar_wait_ab(&k_full[s], (i / ST) & 1, s_abort) ||
            (k >= 1 && !mbar_wait_ab(&pv_done[g], (k - 1) & 1, s_abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(base + S::kKOff + s * S::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (uint32_t)((ks >> 2) * S::kBox + (ks & 3) * 32);
          umma_bf16_ss(tmem + g * kFuKeys, umma_desc_k_sw128(q_addr + off),
                       umma_desc_k_sw128(k_addr + off), idesc_qk, ks > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[g]);
        umma_commit(&k_empty[s]);
        if (i >= 1) ok = issue_pv(i - 1);
      }
      if (ok && ntiles > 0) ok = issue_pv(ntiles - 1);
      if (!ok) set_flag(flags, KVS_FLAG_TIMEOUT);
      // the last MMAs of each group (each P V follows that tile's QK^T) must finish before
      // the tensor memory is released
      for (int g = 0; g < 2; ++g) {
        const int n_g = pv_issued > g ? (pv_issued - 1 - g) / 2 + 1 : 0;
        if (n_g > 0 && !mbar_wait(&pv_done[g], (n_g - 1) & 1)) set_flag(flags, KVS_FLAG_TIMEOUT);
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax groups ----------------
    // group g takes tiles g, g + 2, ...; warp (warp & 3) of it owns window-query rows
    // r = 32 (warp & 3) + lane, all 128 keys of a tile (four 32-key chunks) and the row
    // of O_g
    const int g = (warp - 2) >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int pos = L - W + (r % W);
    const bool row_ok = r < Qn && pos >= 0;
    const float qscale = kLog2e / sqrtf((float)D);
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_cols = tmem + lane_base + (uint32_t)(g * kFuKeys);
    const uint32_t o_cols = tmem + lane_base + 256 + (uint32_t)(g * D);
    float m_ref = -INFINITY, l = 0.f;
    bool live = true;
    int n_mine = 0;
    for (int i = g; i < ntiles; i += 2) {
      const int k = i >> 1, s = i % ST;
      const int tb = t0 + i * kFuKeys;
      ++n_mine;
      live = live && mbar_wait_ab(&s_full[g], k & 1, s_abort);
      live = live && mbar_wait_ab(&v_full[s], (i / ST) & 1, s_abort);   // log-counts, V
      live = __all_sync(0xffffffffu, live);          // tcgen05.ld / st are warp-collective
      const float* lnb = reinterpret_cast<const float*>(base + S::kLnOff + s * S::kLnSlot);
      // logits x = s q.k + log2(e) logn in the log2 domain; masks only on the split's last
      // tile and on keys the causal window hides from some queries
      const bool interior = tb + kFuKeys <= t1 && tb + kFuKeys - 1 <= L - W;
      auto logits = [&](uint32_t (&w)[32], int c) {
        if (interior && row_ok) {
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 ln2 = has_ln ? *reinterpret_cast<const float2*>(lnb + 32 * c + j)
                                      : make_float2(0.f, 0.f);
            const float2 x = ffma2(make_float2(__uint_as_float(w[j]), __uint_as_float(w[j + 1])),
                                   make_float2(qscale, qscale), ln2);
            w[j] = __float_as_uint(x.x);
            w[j + 1] = __float_as_uint(x.y);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = tb + 32 * c + j;
            const bool vis = row_ok && t < t1 && t <= pos;
            w[j] = __float_as_uint(vis ? fmaf(__uint_as_float(w[j]), qscale, has_ln ? lnb[32 * c + j] : 0.f)
                                       : -INFINITY);
          }
        }
      };
      // P = 2^(x - m) as bf16 hi and lo parts over the chunk's own S columns, computed in
      // place over the chunk's logits: pair j/2 leaves hi in w[j] and lo in w[j + 1]
      auto exps = [&](uint32_t (&w)[32], int c, float m, float& lsum) {
        float2 ps = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float pa = m > -INFINITY ? ex2_ftz(__uint_as_float(w[j]) - m) : 0.f;
          const float pb = m > -INFINITY ? ex2_ftz(__uint_as_float(w[j + 1]) - m) : 0.f;
          const float2 p2 = make_float2(pa, pb);
          ps = fadd2(ps, p2);
          const uint32_t hh = pack_bf16x2(pa, pb);
          const float2 r2 = ffma2(make_float2(bf16_lo(hh), bf16_hi(hh)), make_float2(-1.f, -1.f), p2);
          w[j] = hh;
          w[j + 1] = pack_bf16x2(r2.x, r2.y);
        }
        lsum += ps.x + ps.y;
        tmem_st16_pairs<0>(s_cols + 32 * c, w);
        tmem_st16_pairs<1>(s_cols + 32 * c + 16, w);
      };
      float lsum = 0.f, cfac = 1.f, m_new = m_ref;
      // a warp with no valid row leaves its P lanes as they are: an MMA row only feeds the
      // same row of O, and those rows are never read
      if (live && __any_sync(0xffffffffu, row_ok)) {
        tc_fence_after();
        // sweep 1: the tile's row maximum (one chunk of S in registers at a time: a whole
        // row does not fit beside the rest without spilling)
        // On a tile without masked keys an upper bound serves as well as the maximum (the
        // reference only has to be at least every logit): the row maximum of the raw S
        // times the scale, plus the tile's largest log-count, costs one max per element.
        float mt = -INFINITY;
        const bool bound = interior;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t w[32];
          tmem_ld32_async(s_cols + 32 * c, w);
          tmem_ld_wait(w);
          if (!bound) logits(w, c);
          float m4[4] = {__uint_as_float(w[0]), __uint_as_float(w[1]), __uint_as_float(w[2]),
                         __uint_as_float(w[3])};
#pragma unroll
          for (int j = 4; j < 32; ++j) m4[j & 3] = fmaxf(m4[j & 3], __uint_as_float(w[j]));
          mt = fmaxf(mt, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
        }
        if (bound) mt = fmaf(mt, qscale, lnb[kFuKeys]);
        // the reference maximum moves only when the tile exceeds it by 2^8; O_g, which the
        // group's previous P V MMAs update, is then rescaled
        m_new = (mt > m_ref + kRescaleSlack) ? mt : m_ref;
        const bool resc = m_new != m_ref && m_ref > -INFINITY;
        cfac = resc ? ex2_ftz(m_ref - m_new) : 1.f;
        if (__any_sync(0xffffffffu, resc)) {
          live = live && mbar_wait_ab(&pv_done[g], (k - 1) & 1, s_abort);
          live = __all_sync(0xffffffffu, live);
          if (live) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              float ov[32];
              tmem_ld32(o_cols + 32 * c, ov);
#pragma unroll
              for (int j = 0; j < 32; ++j) ov[j] *= cfac;
              tmem_st32(o_cols + 32 * c, ov);
            }
          }
        }
        // sweep 2: P chunk by chunk (stores in flight until the one wait below)
        if (live) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t w[32];
            tmem_ld32_async(s_cols + 32 * c, w);
            tmem_ld_wait(w);
            logits(w, c);
            exps(w, c, m_new, lsum);
          }
        }
        tmem_st_wait();
      }
      l = l * cfac + lsum;
      // value rows past the split's end may hold anything (even non-finite): zero them,
      // since their probability is 0 and 0 x inf is not (this group's four warps split it)
      const int nvalid = min(kFuKeys, t1 - tb);
      if (nvalid < kFuKeys && live) {
        unsigned char* vt = base + S::kVOff + s * S::kTile;
        const int nz = (kFuKeys - nvalid) * S::kBoxes * 8;    // 16-byte chunks
        for (int idx = quarter * 32 + lane; idx < nz; idx += 128) {
          const int rr = nvalid + idx / (S::kBoxes * 8);
          const int rem = idx % (S::kBoxes * 8);
          *reinterpret_cast<uint4*>(vt + (rem >> 3) * S::kBox + rr * 128 + (rem & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();                    // generic writes -> tensor-core reads
      tc_fence_before();                           // tensor-memory stores -> the MMA's reads
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[g]);
      m_ref = m_new;
    }
    if (!live) set_flag(flags, KVS_FLAG_TIMEOUT);
    // The CTA's partial, the two groups merged: group 1 leaves its (m, l) per row in two
    // columns of its S buffer (free once its last P V MMAs are done; the same lanes), and
    // the group-0 warp of the same lane quarter combines both O rows from tensor memory
    // (the two warps meet at a named barrier of their own).
    bool got = n_mine > 0 && live && mbar_wait_ab(&pv_done[g], (n_mine - 1) & 1, s_abort);
    got = __all_sync(0xffffffffu, got);
    if (n_mine > 0 && !got) set_flag(flags, KVS_FLAG_TIMEOUT);
    const bool any = got && row_ok && m_ref > -INFINITY && l > 0.f;
    const uint32_t ml1_cols = tmem + lane_base + (uint32_t)kFuKeys;   // S_1, columns 0-1
    if (g == 1) {
      tmem_st2(ml1_cols, __float_as_uint(any ? m_ref : -INFINITY), __float_as_uint(any ? l : 0.f));
      tmem_st_wait();
      tc_fence_before();
    }
    named_bar(1 + quarter, 2 * 32);
    if (g == 0) {
      tc_fence_after();
      uint32_t ml[2];
      tmem_ld2(ml1_cols, ml);
      const float m1 = __uint_as_float(ml[0]), l1 = __uint_as_float(ml[1]);
      const bool any1 = l1 > 0.f;
      const float m0 = any ? m_ref : -INFINITY;
      const float M = fmaxf(m0, m1);
      const float f0 = any ? ex2_ftz(m0 - M) : 0.f, f1 = any1 ? ex2_ftz(m1 - M) : 0.f;
      const bool both = any || any1;
      const float Ls = (any ? f0 * l : 0.f) + (any1 ? f1 * l1 : 0.f);
      const size_t prow = ((size_t)unit * nsplit + split) * Qn + r;
      if (r < Qn) {
        part_ml[prow * 2 + 0] = both ? M : -INFINITY;
        part_ml[prow * 2 + 1] = both ? Ls : 0.f;
      }
      const uint32_t o1_cols = tmem + lane_base + 256 + (uint32_t)D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o0[32], o1[32];
        if (__any_sync(0xffffffffu, any)) {
          tmem_ld32(o_cols + 32 * c, o0);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o0[j] = 0.f;
        }
        if (__any_sync(0xffffffffu, any1)) {
          tmem_ld32(o1_cols + 32 * c, o1);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o1[j] = 0.f;
        }
        if (r < Qn) {
          float* po = part_o + prow * D + 32 * c;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float4 v4;
            v4.x = (any ? f0 * o0[j] : 0.f) + (any1 ? f1 * o1[j] : 0.f);
            v4.y = (any ? f0 * o0[j + 1] : 0.f) + (any1 ? f1 * o1[j + 1] : 0.f);
            v4.z = (any ? f0 * o0[j + 2] : 0.f) + (any1 ? f1 * o1[j + 2] : 0.f);
            v4.w = (any ? f0 * o0[j + 3] : 0.f) + (any1 ? f1 * o1[j + 3] : 0.f);
            *reinterpret_cast<float4*>(po + j) = v4;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kFuTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Combine, in two small kernels with many CTAs (a per-head CTA walking all partials of
// all queries was latency-bound: one launch took longer than both passes together).
//   fa_query_kernel (one CTA per window query and head): the partials' (m, l, O) ->
//     (M, L) and o_q.
//   fa_center_kernel (per head, and per block of queries in the per-query form):
//     o_bar = mean_q o_q over the queries with a visible key, and e_q = o_q - o_bar as
//     bf16 hi / mid / lo rows with |e_q|^2 and o_bar . e_q.
// ---------------------------------------------------------------------------

// One CTA per block of QB window queries of a head (QB grows with the number of heads,
// so that the grid stays near a thousand CTAs): the warps take the block's queries in
// turn for (M, L), then every thread (one column) sums its column of the partials' O rows
// for each query of the block, the loads independent of one another.
constexpr int kQueryBlockMax = 16;

template <int D>
__global__ void __launch_bounds__(D, 8)
fa_query_kernel(const float* __restrict__ part_ml, const float* __restrict__ part_o, int Qn,
                int nparts, int QB, float* __restrict__ stats, float* __restrict__ oq) {
  extern __shared__ float fac[];                 // [QB][nparts] weights 2^(m - M) / L
  const int unit = blockIdx.y, c = threadIdx.x, lane = c & 31, warp = c >> 5;
  const int q0 = blockIdx.x * QB, nq = min(QB, Qn - q0);
  const float* e = part_ml + (size_t)unit * nparts * Qn * 2;
  for (int j = warp; j < nq; j += D / 32) {
    const int q = q0 + j;
    float M = -INFINITY;
    for (int s = lane; s < nparts; s += 32) {
      const float ls = e[((size_t)s * Qn + q) * 2 + 1];
      if (ls > 0.f) M = fmaxf(M, e[((size_t)s * Qn + q) * 2]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Ls = 0.f;
    if (M > -INFINITY)
      for (int s = lane; s < nparts; s += 32) {
        const float ls = e[((size_t)s * Qn + q) * 2 + 1];
        if (ls > 0.f) Ls = fmaf(ls, exp2f(e[((size_t)s * Qn + q) * 2] - M), Ls);
      }
    Ls = warp_sum(Ls);
    const bool valid = Ls > 0.f;
    for (int s = lane; s < nparts; s += 32) {
      const float ls = e[((size_t)s * Qn + q) * 2 + 1];
      fac[j * nparts + s] = (valid && ls > 0.f) ? exp2f(e[((size_t)s * Qn + q) * 2] - M) / Ls : 0.f;
    }
    if (lane == 0) {
      stats[((size_t)unit * Qn + q) * 2 + 0] = M;
      stats[((size_t)unit * Qn + q) * 2 + 1] = Ls;
    }
  }
  __syncthreads();
  // o_q = sum over partials of weight x O row, with the loads of a batch independent of
  // one another: eight partials of one query at a time when there are many partials, all
  // the block's queries of one partial at a time when there are few
  const size_t stride = (size_t)Qn * D;
  const float* pb = part_o + ((size_t)unit * nparts * Qn + q0) * D + c;
  if (nparts >= 8 || nq == 1) {
    for (int j = 0; j < nq; ++j) {
      const float* po = pb + (size_t)j * D;
      const float* f = fac + j * nparts;
      float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      int s = 0;
      for (; s + 8 <= nparts; s += 8) {
#pragma unroll
        for (int k = 0; k < 8; ++k) a8[k] = fmaf(f[s + k], po[(s + k) * stride], a8[k]);
      }
      for (; s < nparts; ++s) a8[s & 7] = fmaf(f[s], po[s * stride], a8[s & 7]);
      oq[((size_t)unit * 128 + q0 + j) * D + c] =
          ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
    }
  } else {
    float acc[kQueryBlockMax];
#pragma unroll
    for (int j = 0; j < kQueryBlockMax; ++j) acc[j] = 0.f;
    for (int s = 0; s < nparts; ++s) {
#pragma unroll
      for (int j = 0; j < kQueryBlockMax; ++j)
        if (j < nq) acc[j] = fmaf(fac[j * nparts + s], pb[s * stride + (size_t)j * D], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < kQueryBlockMax; ++j)
      if (j < nq) oq[((size_t)unit * 128 + q0 + j) * D + c] = acc[j];
  }
}

// One CTA per 32 columns of a head: 8 warps x 32 columns, warp w summing the queries
// q = w, w + 8, ... in a fixed order, so o_bar is the same on every run.
constexpr int kCenterWarps = 8;

template <int D>
__global__ void __launch_bounds__(kCenterWarps * 32)
fa_center_kernel(const float* __restrict__ stats, const float* __restrict__ oq, int Qn,
                 int with_e, float* __restrict__ obar, float* __restrict__ zpart,
                 float* __restrict__ wpart, bf16* __restrict__ e_hi, bf16* __restrict__ e_mid,
                 bf16* __restrict__ e_lo) {
  __shared__ float s_sum[kCenterWarps][32];
  __shared__ float s_ob[32];
  __shared__ int s_valid;                        // queries with a visible key
  const int cb = blockIdx.x, unit = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, qg = tid >> 5;
  const int c = 32 * cb + lane;
  if (tid == 0) s_valid = 0;
  __syncthreads();
  int nv = 0;
  for (int q = tid; q < Qn; q += kCenterWarps * 32) nv += stats[((size_t)unit * Qn + q) * 2 + 1] > 0.f;
  if (nv) atomicAdd(&s_valid, nv);
  const float* col = oq + (size_t)unit * 128 * D + c;
  float a = 0.f;
#pragma unroll 4
  for (int q = qg; q < Qn; q += kCenterWarps) a += col[(size_t)q * D];
  s_sum[qg][lane] = a;
  __syncthreads();
  if (qg == 0) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kCenterWarps; ++w) t += s_sum[w][lane];
    const float ob = s_valid > 0 ? t / (float)s_valid : 0.f;
    s_ob[lane] = ob;
    obar[(size_t)unit * D + c] = ob;
  }
  if (!with_e) return;
  __syncthreads();
  // e_q = o_q - o_bar for this CTA's 32 columns of every (padded) query row, and the
  // column block's share of |e_q|^2 and o_bar . e_q (pass B adds the D / 32 shares)
  const float ob = s_ob[lane];
  for (int q = qg; q < 128; q += kCenterWarps) {
    const float e = q < Qn ? col[(size_t)q * D] - ob : 0.f;
    const bf16 hi = __float2bfloat16_rn(e);
    const float r1 = e - __bfloat162float(hi);
    const bf16 mid = __float2bfloat16_rn(r1);
    const size_t at = ((size_t)unit * 128 + q) * D + c;
    e_hi[at] = hi;
    e_mid[at] = mid;
    e_lo[at] = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    const float z = warp_sum(e * e), wv = warp_sum(ob * e);
    if (lane == 0) {
      zpart[((size_t)unit * (D / 32) + cb) * 128 + q] = z;
      wpart[((size_t)unit * (D / 32) + cb) * 128 + q] = wv;
    }
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
  static constexpr int kStages = PERQ ? (D == 128 ? 1 : 2) : (D == 128 ? 3 : 4);
  static constexpr int kQOff = 0;
  static constexpr int kEOff = kTile;                        // per query form: E hi, mid, lo
  static constexpr int kStageOff = kEOff + (PERQ ? 3 * kTile : 0);
  static constexpr int kStageBytes = 2 * kTile;              // K tile, then V tile
  static constexpr int kSmallOff = kStageOff + kStages * kStageBytes;
  // barriers (256 B), Z_q = M_q + log2 L_q [128], o_bar [D], q mod W [128], and for the
  // per-query form |e_q|^2 and o_bar . e_q [2][128]; tensor-memory address, abort flag
  static constexpr int kZOff = kSmallOff + 256;
  static constexpr int kObOff = kZOff + 128 * 4;
  static constexpr int kQmodOff = kObOff + 128 * 4;
  static constexpr int kEqOff = kQmodOff + 128 * 4;
  static constexpr int kMiscOff = kEqOff + (PERQ ? 3 * 128 * 4 : 0);
  static constexpr int kSmem = kMiscOff + 16 + 1024;
  static_assert(kSmem <= 232448, "shared memory");
  // TMA tile destinations with 128-byte swizzling start on 1024-byte boundaries; the
  // barriers (1 + 2 ST + 8) fit the 256 bytes before Z_q; the float2 reads of Z_q and
  // o_bar are 8-byte aligned
  static_assert(kEOff % 1024 == 0 && kStageOff % 1024 == 0 && kStageBytes % 1024 == 0,
                "tile alignment");
  static_assert(8 * (1 + 2 * kStages + 8) <= kZOff - kSmallOff, "barrier room");
  static_assert(kSmallOff % 8 == 0 && kZOff % 8 == 0 && kObOff % 8 == 0, "array alignment");
};

// Tensor memory of pass B, per softmax group g: S^T_g at [128 g, 128 g + 128) and, per
// query form, U_g = V E^T at [256 + 128 g, 256 + 128 g + 128).

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

// Square root on the special-function unit (PTX sqrt.approx.ftz: relative error of a few
// units in the last place of fp32, far inside the score tolerance; subnormals flush to 0).
__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Per-query form, taken directly where the expansion around o_bar cancels:
// |x - k e_q|^2 with x = (v_a - o_bar) (+ (v_b - o_bar) when vb is given), the value rows
// read from the cache, o_bar and e_q = hi + mid + lo from shared memory (E tiles with
// 128-byte swizzling, query q's row).
template <int D>
__device__ __noinline__ float direct_sq(const bf16* __restrict__ va, const bf16* __restrict__ vb,
                                        const float* obs, const unsigned char* et, int q, float k) {
  constexpr int kBox = 128 * 128, kTile = (D / 64) * kBox;
  float acc = 0.f;
#pragma unroll 2
  for (int ch = 0; ch < D / 8; ++ch) {
    const int dim = ch * 8, bx = dim >> 6, cc = (dim & 63) >> 3;
    float fa[8], fb[8], eh[8], em[8], el[8];
    load_vec(va + dim, fa);
    if (vb) {
      load_vec(vb + dim, fb);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) fb[e] = 0.f;
    }
    const uint32_t off = (uint32_t)(bx * kBox) + swz128(q, cc);
    load_vec(reinterpret_cast<const bf16*>(et + off), eh);
    load_vec(reinterpret_cast<const bf16*>(et + kTile + off), em);
    load_vec(reinterpret_cast<const bf16*>(et + 2 * kTile + off), el);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float o = obs[dim + e];
      const float x = vb ? (fa[e] - o) + (fb[e] - o) : fa[e] - o;
      const float dlt = fmaf(-k, (el[e] + em[e]) + eh[e], x);
      acc = fmaf(dlt, dlt, acc);
    }
  }
  return acc;
}

// A squared distance from the expansion is recomputed directly when it is below this
// fraction of the magnitude of the terms it was formed from (a bound on their error).
constexpr float kRedoFrac = 1.f / 16.f;

template <int D, bool PERQ>
__global__ void __launch_bounds__(kFuThreads, 1)
window_score_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmEh,
                    const __grid_constant__ CUtensorMap tmEm, const __grid_constant__ CUtensorMap tmEl,
                    const bf16* __restrict__ Vg, const float* __restrict__ logn,
                    const int32_t* __restrict__ len,
                    const int32_t* __restrict__ cand_begin, int n_recent, int H_kv, int H_q,
                    int W, int T_cap, int nsplit, int cap_chunks, int form,
                    const float* __restrict__ stats,
                    const float* __restrict__ obar, const float* __restrict__ zqg,
                    const float* __restrict__ wqg, float* __restrict__ score,
                    float* __restrict__ w_b, int32_t* __restrict__ flags) {
  using S = ScShape<D, PERQ>;
  constexpr int ST = S::kStages;
  extern __shared__ unsigned char dsm[];
  unsigned char* base = align1024(dsm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::kSmallOff);
  uint64_t* q_full = bars;              // 1 (Q and, per query, E hi / mid / lo)
  uint64_t* full = q_full + 1;          // ST: K and V tiles of a stage landed
  uint64_t* empty = full + ST;          // ST: the four warps of the tile's group are done
  uint64_t* s_full = empty + ST;        // 2 (per group)
  uint64_t* s_empty = s_full + 2;       // 2
  uint64_t* u_full = s_empty + 2;       // 2 (per query form)
  uint64_t* u_empty = u_full + 2;       // 2
  float* zq = reinterpret_cast<float*>(base + S::kZOff);
  float* obs = reinterpret_cast<float*>(base + S::kObOff);
  int* qmod = reinterpret_cast<int*>(base + S::kQmodOff);
  float* eqs = reinterpret_cast<float*>(base + S::kEqOff);        // |e_q|^2, o_bar.e_q, |e_q|
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
  // split s takes a share of the head's candidate tiles, or (cap_chunks) a fixed number of
  // tiles of the capacity's, so that a short head leaves its last CTAs idle
  int tbeg, tend;
  if (cap_chunks) {
    const int cap_tiles = (T_cap / 2 + kFuKeys / 2 - 1) / (kFuKeys / 2);
    const int per = (cap_tiles + nsplit - 1) / nsplit;
    tbeg = min(ntot, split * per);
    tend = min(ntot, tbeg + per);
  } else {
    tbeg = (int)((long long)split * ntot / nsplit);
    tend = (int)((long long)(split + 1) * ntot / nsplit);
  }
  const int ntiles = tend - tbeg;
  if (ntiles <= 0) return;                           // uniform over the CTA
  const int q_row0 = (b * H_q + h * G) * W;
  const int e_row0 = unit * 128;
  const int k_row0 = unit * T_cap + c0 + tbeg * kFuKeys;

  if (tid == 0) {
    *s_abort = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFuGroupWarps);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&s_empty[g], kFuGroupWarps);
      mbar_init(&u_full[g], 1);
      mbar_init(&u_empty[g], kFuGroupWarps);
    }
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
      float z = 0.f, wv = 0.f;
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        z += zqg[((size_t)unit * (D / 32) + cb) * 128 + q];
        wv += wqg[((size_t)unit * (D / 32) + cb) * 128 + q];
      }
      eqs[q] = z;
      eqs[128 + q] = wv;
      eqs[256 + q] = sqrtf(z);
    }
  }
  if (warp == 1) tmem_alloc(s_tmem, kFuTmemCols);
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
      mbar_arrive_expect_tx(q_full, PERQ ? 4 * S::kTile : S::kTile);
#pragma unroll
      for (int bx = 0; bx < S::kBoxes; ++bx) {
        tma_load_2d(base + S::kQOff + bx * S::kBox, &tmQ, bx * 64, q_row0, q_full);
        if (PERQ) {
          tma_load_2d(base + S::kEOff + bx * S::kBox, &tmEh, bx * 64, e_row0, q_full);
          tma_load_2d(base + S::kEOff + S::kTile + bx * S::kBox, &tmEm, bx * 64, e_row0, q_full);
          tma_load_2d(base + S::kEOff + 2 * S::kTile + bx * S::kBox, &tmEl, bx * 64, e_row0,
                      q_full);
        }
      }
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % ST;
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
    // ---------------- MMA issuer: S^T = K Q^T (and U = V E^T) ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(kFuKeys, 128);
      const uint32_t q_addr = smem_u32(base + S::kQOff);
      const uint32_t e_addr = smem_u32(base + S::kEOff);
      bool ok = mbar_wait_ab(q_full, 0, s_abort);
      int done = 0;
      for (int i = 0; ok && i < ntiles; ++i) {
        const int s = i % ST, g = i & 1, k = i >> 1;
        if (!mbar_wait_ab(&full[s], (i / ST) & 1, s_abort) ||
            (k >= 1 && !mbar_wait_ab(&s_empty[g], (k - 1) & 1, s_abort)) ||
            (PERQ && k >= 1 && !mbar_wait_ab(&u_empty[g], (k - 1) & 1, s_abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(base + S::kStageOff + s * S::kStageBytes);
        const uint32_t v_addr = k_addr + S::kTile;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (uint32_t)((ks >> 2) * S::kBox + (ks & 3) * 32);
          umma_bf16_ss(tmem + g * kFuKeys, umma_desc_k_sw128(k_addr + off),
                       umma_desc_k_sw128(q_addr + off), idesc, ks > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[g]);
        if (PERQ) {
#pragma unroll
          for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const uint32_t off = (uint32_t)((ks >> 2) * S::kBox + (ks & 3) * 32);
              umma_bf16_ss(tmem + 256 + g * kFuKeys, umma_desc_k_sw128(v_addr + off),
                           umma_desc_k_sw128(e_addr + part * S::kTile + off), idesc,
                           (part > 0 || ks > 0) ? 1u : 0u);
            }
          umma_commit(&u_full[g]);
        }
        done = i + 1;
      }
      if (!ok) set_flag(flags, KVS_FLAG_TIMEOUT);
      for (int g = 0; g < 2; ++g) {
        const int n_g = done > g ? (done - 1 - g) / 2 + 1 : 0;
        if (n_g > 0 && !mbar_wait(&s_full[g], (n_g - 1) & 1)) set_flag(flags, KVS_FLAG_TIMEOUT);
        if (PERQ && n_g > 0 && !mbar_wait(&u_full[g], (n_g - 1) & 1))
          set_flag(flags, KVS_FLAG_TIMEOUT);
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax groups ----------------
    // group g takes tiles g, g + 2, ...; warp (warp & 3) of it owns the keys
    // kr = 32 (warp & 3) + lane of a tile with all 128 window-query columns, and its 16
    // pairs: lanes 2 j and 2 j + 1 are the pair's two rows, and each of the two takes
    // half of the head dimension for the row terms
    const int g = (warp - 2) >> 2, quarter = warp & 3;
    const int kr = quarter * 32 + lane;
    const float qscale = kLog2e / sqrtf((float)D);
    const float* lnh = logn ? logn + (size_t)unit * T_cap : nullptr;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_cols = tmem + lane_base + (uint32_t)(g * kFuKeys);
    const uint32_t u_cols = tmem + lane_base + 256 + (uint32_t)(g * kFuKeys);
    const bool is_a = (lane & 1) == 0;
    const int ra = quarter * 32 + (lane & ~1), rb = ra + 1;   // the pair's rows in the tile
    constexpr int DH = D / 2;                                  // dims per lane of a pair
    const int dim0 = (lane & 1) * DH;
    bool live = true;
    float ln_next = 0.f;
    if (lnh && g < ntiles) {
      const int kn = (tbeg + g) * kFuKeys + kr;
      if (kn < 2 * P) ln_next = lnh[c0 + kn];
    }
    for (int i = g; i < ntiles; i += 2) {
      const int k = i >> 1, s = i % ST;
      const int tile = tbeg + i;
      const int krow = tile * kFuKeys + kr;       // this thread's key, relative to c0
      const int t = c0 + krow;                    // its cache row
      const bool kval = krow < 2 * P;
      const float lnt = ln_next * kLog2e;
      if (lnh && i + 2 < ntiles) {
        const int kn = krow + 2 * kFuKeys;
        ln_next = kn < 2 * P ? lnh[c0 + kn] : 0.f;
      }
      const int hide = t - (L - W);               // queries with q mod W < hide miss the key
      // With an even stage count every use of a stage is this group's (tiles i, i + ST,
      // ... have i's parity), so the group has seen the stage's previous phase and may wait
      // on `full` first: the row terms below then overlap the tile's S^T MMA. With an odd
      // count consecutive uses of a stage go to different groups and a parity wait on
      // `full` could match the previous phase, so the group waits for its S^T first (the
      // MMA was issued only after the stage's rows had landed, so the stage then holds
      // this tile and the wait on `full` can only match this tile's phase).
      constexpr bool kOwnStages = (ST % 2) == 0;
      if (!kOwnStages) live = live && mbar_wait_ab(&s_full[g], k & 1, s_abort);
      live = live && mbar_wait_ab(&full[s], (i / ST) & 1, s_abort);
      live = __all_sync(0xffffffffu, live);
      // the pair's row terms from the stage: |k_b - k_a|^2, |v_a - o_bar|^2,
      // |v_b - o_bar|^2, |v_a + v_b - 2 o_bar|^2 (this lane's half of the dims)
      // packed fp32 pairs: the two dims of a bf16 pair in one register pair
      const float2 neg1 = make_float2(-1.f, -1.f);
      float2 dd2 = make_float2(0.f, 0.f), ea2 = dd2, eb2 = dd2, ec2 = dd2, na2 = dd2, nb2 = dd2;
      if (live) {
        const unsigned char* kt = base + S::kStageOff + s * S::kStageBytes;
        const unsigned char* vt = kt + S::kTile;
#pragma unroll
        for (int ch = 0; ch < DH / 8; ++ch) {
          const int dim = dim0 + ch * 8;
          const int bx = dim >> 6, cc = (dim & 63) >> 3;
          const uint4 ka = *reinterpret_cast<const uint4*>(kt + bx * S::kBox + swz128(ra, cc));
          const uint4 kb = *reinterpret_cast<const uint4*>(kt + bx * S::kBox + swz128(rb, cc));
          const uint4 va = *reinterpret_cast<const uint4*>(vt + bx * S::kBox + swz128(ra, cc));
          const uint4 vb = *reinterpret_cast<const uint4*>(vt + bx * S::kBox + swz128(rb, cc));
          const uint32_t kaw[4] = {ka.x, ka.y, ka.z, ka.w}, kbw[4] = {kb.x, kb.y, kb.z, kb.w};
          const uint32_t vaw[4] = {va.x, va.y, va.z, va.w}, vbw[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 o2 = *reinterpret_cast<const float2*>(obs + dim + 2 * e);
            const float2 ka2 = make_float2(bf16_lo(kaw[e]), bf16_hi(kaw[e]));
            const float2 kb2 = make_float2(bf16_lo(kbw[e]), bf16_hi(kbw[e]));
            const float2 va2 = make_float2(bf16_lo(vaw[e]), bf16_hi(vaw[e]));
            const float2 vb2 = make_float2(bf16_lo(vbw[e]), bf16_hi(vbw[e]));
            const float2 dk = ffma2(ka2, neg1, kb2);
            const float2 ra2 = ffma2(o2, neg1, va2);
            const float2 rb2 = ffma2(o2, neg1, vb2);
            const float2 rc2 = fadd2(ra2, rb2);
            dd2 = ffma2(dk, dk, dd2);
            ea2 = ffma2(ra2, ra2, ea2);
            eb2 = ffma2(rb2, rb2, eb2);
            ec2 = ffma2(rc2, rc2, ec2);
            if (PERQ) {
              na2 = ffma2(va2, va2, na2);
              nb2 = ffma2(vb2, vb2, nb2);
            }
          }
        }
      }
      float dd = dd2.x + dd2.y, ea = ea2.x + ea2.y, eb = eb2.x + eb2.y, ec = ec2.x + ec2.y;
      float na = na2.x + na2.y, nb = nb2.x + nb2.y;
      dd += __shfl_xor_sync(0xffffffffu, dd, 1);
      ea += __shfl_xor_sync(0xffffffffu, ea, 1);
      eb += __shfl_xor_sync(0xffffffffu, eb, 1);
      ec += __shfl_xor_sync(0xffffffffu, ec, 1);
      if (PERQ) {
        na += __shfl_xor_sync(0xffffffffu, na, 1);
        nb += __shfl_xor_sync(0xffffffffu, nb, 1);
      }
      // window probabilities p_qt = 2^(s q.k + lnt - Z_q), the key's row of S^T
      if (kOwnStages) live = live && mbar_wait_ab(&s_full[g], k & 1, s_abort);
      if (PERQ) live = live && mbar_wait_ab(&u_full[g], k & 1, s_abort);
      live = __all_sync(0xffffffffu, live);
      // the stage's rows are read, here and by the tile's MMAs (done: S^T, U landed)
      if (lane == 0) mbar_arrive(&empty[s]);
      if (live) tc_fence_after();
      float acc = 0.f, n_self = 0.f, n_cpl = 0.f;
      const float t_own = is_a ? ea : eb;
      // per query form: the magnitudes that bound the expansion's error (U carries the
      // tensor cores' accumulation error, of order |v| |e_q|), and the value rows that a
      // direct recomputation reads
      const float vn_own = sqrtf(is_a ? na : nb), vn_pair = sqrtf(na) + sqrtf(nb);
      const bf16* v_own = Vg + ((size_t)unit * T_cap + (kval ? t : 0)) * D;
      const bf16* v_next = v_own + D;
      // chunks of CW window queries (16 in the per-query form, whose per-element work
      // keeps two chunk-wide arrays live: a narrower chunk keeps them in registers)
      constexpr int CW = PERQ ? 16 : 32;
#pragma unroll 1
      for (int c = 0; c < 128 / CW; ++c) {
        float v[CW];
        if (live) {
          tmem_ld_n<CW>(s_cols + CW * c, v);
        } else {
#pragma unroll
          for (int j = 0; j < CW; ++j) v[j] = 0.f;
        }
        if (kval) {
#pragma unroll
          for (int j = 0; j < CW; j += 2) {
            const float2 z = *reinterpret_cast<const float2*>(&zq[CW * c + j]);
            const float2 x = ffma2(make_float2(v[j], v[j + 1]), make_float2(qscale, qscale),
                                   make_float2(lnt - z.x, lnt - z.y));
            v[j] = ex2_ftz(x.x);
            v[j + 1] = ex2_ftz(x.y);
          }
          if (hide > 0) {
#pragma unroll
            for (int j = 0; j < CW; ++j)
              if (qmod[CW * c + j] < hide) v[j] = 0.f;
          }
        } else {
#pragma unroll
          for (int j = 0; j < CW; ++j) v[j] = 0.f;
        }
        if constexpr (!PERQ) {
          float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < CW; ++j) a4[j & 3] += v[j];
          acc += (a4[0] + a4[1]) + (a4[2] + a4[3]);
        } else {
          // per window query: lane a (even key) takes N11 and N12, lane b N22
          float u[CW];
          if (live) {
            tmem_ld_n<CW>(u_cols + CW * c, u);
          } else {
#pragma unroll
            for (int j = 0; j < CW; ++j) u[j] = 0.f;
          }
          // fully unrolled: v[] and u[] stay in registers (a partly unrolled loop indexes
          // them at run time, which puts them in local memory). The terms whose expansion
          // cancels are only marked here and taken directly afterwards, outside the loop.
          uint32_t redo_s = 0u, redo_c = 0u;
#pragma unroll
          for (int j = 0; j < CW; ++j) {
            const int q = CW * c + j;
            const float p = v[j], uu = u[j];
            const float p_o = __shfl_xor_sync(0xffffffffu, p, 1);
            const float u_o = __shfl_xor_sync(0xffffffffu, uu, 1);
            const float z = eqs[q], wq = eqs[128 + q], se = eqs[256 + q];
            // |v - o_q|^2 and |v_a + v_b - 2 o_q|^2 by the expansion, unless it cancels
            // (a query whose output sits near the row)
            const float xs = uu - wq, xc = uu + u_o - 2.f * wq;
            const float rs = fmaf(-2.f, xs, t_own) + z;
            const float rc = fmaf(-4.f, xc, ec) + 4.f * z;
            const float ms = t_own + z + 2.f * fabsf(xs) + 2.f * vn_own * se;
            const float mc = ec + 4.f * z + 4.f * fabsf(xc) + 4.f * vn_pair * se;
            const bool ds = p != 0.f && rs < kRedoFrac * ms;
            const bool dc = is_a && p * p_o != 0.f && rc < kRedoFrac * mc;
            redo_s |= (uint32_t)ds << j;
            redo_c |= (uint32_t)dc << j;
            n_self = fmaf(ds ? 0.f : fabsf(p * (1.f - 2.f * p)), sqrt_approx(fmaxf(0.f, rs)), n_self);
            if (is_a) n_cpl = fmaf(dc ? 0.f : p * p_o, sqrt_approx(fmaxf(0.f, rc)), n_cpl);
          }
          // the marked terms, directly from the value rows and e_q (rare: only keys that
          // hold much of some query's attention); the query's column of S^T is loaded
          // again by the whole warp and p recomputed with the same arithmetic
          uint32_t todo = __reduce_or_sync(0xffffffffu, redo_s | redo_c);
          const unsigned char* et = base + S::kEOff;
          while (todo) {
            const int j = __ffs(todo) - 1;
            todo &= todo - 1u;
            const int q = CW * c + j;
            float sv = tmem_ld1(s_cols + q);
            float p = 0.f;
            if (kval) {
              p = ex2_ftz(fmaf(sv, qscale, lnt - zq[q]));
              if (hide > 0 && qmod[q] < hide) p = 0.f;
            }
            const float p_o = __shfl_xor_sync(0xffffffffu, p, 1);
            if ((redo_s >> j) & 1u)
              n_self = fmaf(fabsf(p * (1.f - 2.f * p)),
                            sqrt_approx(direct_sq<D>(v_own, nullptr, obs, et, q, 1.f)), n_self);
            if ((redo_c >> j) & 1u)
              n_cpl = fmaf(p * p_o, sqrt_approx(direct_sq<D>(v_own, v_next, obs, et, q, 2.f)),
                           n_cpl);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_empty[g]);
        if (PERQ) mbar_arrive(&u_empty[g]);
      }
      // the pair's weight and score (lane a writes them)
      float n11, n12, n22;
      if constexpr (!PERQ) {
        const float al = acc * inv_qv;
        const float aa = __shfl_sync(0xffffffffu, al, lane & ~1);
        const float bb = __shfl_sync(0xffffffffu, al, lane | 1);
        n11 = fabsf(aa * (1.f - 2.f * aa)) * sqrtf(ea);
        n22 = fabsf(bb * (1.f - 2.f * bb)) * sqrtf(eb);
        n12 = aa * bb * sqrtf(ec);
      } else {
        const float other = __shfl_xor_sync(0xffffffffu, n_self, 1);
        n11 = (is_a ? n_self : other) * inv_qv;
        n22 = (is_a ? other : n_self) * inv_qv;
        n12 = n_cpl * inv_qv;
      }
      const int pglob = tile * (kFuKeys / 2) + (ra >> 1);
      if (is_a && pglob < P && live) {
        float w, sc;
        pair_weight_score(n11, n12, n22, dd, form, w, sc);
        const size_t at = (size_t)unit * (T_cap / 2) + pglob;
        score[at] = sc;
        w_b[at] = w;
      }
    }
    if (!live) set_flag(flags, KVS_FLAG_TIMEOUT);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kFuTmemCols);
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

// Many heads over a large capacity: a few splits per head over fixed chunks of the
// capacity instead of one share of each head's length. With ragged lengths (a serving
// batch) a head's CTAs then carry at most a chunk each and the short heads' spare CTAs
// return at once, so the SMs even the load out over the waves; a single CTA per head
// would leave the longest heads setting the time.
static bool cap_chunked(int units, int T_cap) { return units >= 74 && T_cap >= 8192; }
static int cap_splits(int T_cap) { return T_cap / 2048 < 4 ? T_cap / 2048 : 4; }

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
  bf16* e_hi = reinterpret_cast<bf16*>(ws + Ly.oq_hi);
  bf16* e_mid = reinterpret_cast<bf16*>(ws + Ly.oq_mid);
  bf16* e_lo = reinterpret_cast<bf16*>(ws + Ly.oq_lo);
  CUtensorMap mQ, mK, mV, mEh, mEm, mEl;
  const unsigned long long erows = (unsigned long long)units * 128;
  if (!encode_rows_map(&mQ, Qw, qrows, D, 128) || !encode_rows_map(&mK, K, rows, D, kFuKeys) ||
      !encode_rows_map(&mV, V, rows, D, kFuKeys) || !encode_rows_map(&mEh, e_hi, erows, D, 128) ||
      !encode_rows_map(&mEm, e_mid, erows, D, 128) || !encode_rows_map(&mEl, e_lo, erows, D, 128))
    return cudaErrorInvalidValue;
  // pass A: one partial per CTA (its two softmax groups merged), as many CTAs per head as
  // the layout has partial slots at most
  const bool capc = cap_chunked(units, d.T_cap);
  int nsa = capc ? cap_splits(d.T_cap) : fused_splits(units);
  if (nsa > Ly.part_slots) nsa = Ly.part_slots;
  const int Qn = Ly.Qn;
  int32_t* flags = reinterpret_cast<int32_t*>(ws);
  float* part_ml = reinterpret_cast<float*>(ws + Ly.part_ml);
  float* part_o = reinterpret_cast<float*>(ws + Ly.part_o);
  float* stats = reinterpret_cast<float*>(ws + Ly.stats);
  float* obar = reinterpret_cast<float*>(ws + Ly.obar);
  float* zq = reinterpret_cast<float*>(ws + Ly.on2);
  float* wq = reinterpret_cast<float*>(ws + Ly.owq);

  auto ka = window_fa_kernel<D>;
  if (!ensure_smem_attr((const void*)ka, FaShape<D>::kSmem)) return cudaErrorInvalidValue;
  ka<<<dim3(nsa, units), kFuThreads, FaShape<D>::kSmem, st>>>(
      mQ, mK, mV, logn, len, d.H_kv, d.H_q, W, d.T_cap, nsa, capc ? 1 : 0, part_ml, part_o,
      flags);
  float* oq = reinterpret_cast<float*>(ws + Ly.oq);
  // queries per CTA: about a thousand CTAs in all
  int QB = 1;
  while (QB < kQueryBlockMax && (long long)units * Qn / (2 * QB) >= 1024) QB *= 2;
  const size_t qsm = (size_t)QB * nsa * sizeof(float);
  auto kq = fa_query_kernel<D>;
  if (!ensure_smem_attr((const void*)kq, qsm)) return cudaErrorInvalidValue;
  kq<<<dim3((Qn + QB - 1) / QB, units), D, qsm, st>>>(part_ml, part_o, Qn, nsa, QB, stats, oq);
  const bool perq = stats_form == KVS_FORM_PER_QUERY;
  fa_center_kernel<D><<<dim3(D / 32, units), kCenterWarps * 32, 0, st>>>(
      stats, oq, Qn, perq ? 1 : 0, obar, zq, wq, e_hi, e_mid, e_lo);
  const int nsb = capc ? cap_splits(d.T_cap) : fused_splits(units);
  if (perq) {
    auto kb = window_score_kernel<D, true>;
    if (!ensure_smem_attr((const void*)kb, ScShape<D, true>::kSmem)) return cudaErrorInvalidValue;
    kb<<<dim3(nsb, units), kFuThreads, ScShape<D, true>::kSmem, st>>>(
        mQ, mK, mV, mEh, mEm, mEl, (const bf16*)V, logn, len, cand_begin, n_recent, d.H_kv,
        d.H_q, W, d.T_cap, nsb, capc ? 1 : 0, form, stats, obar, zq, wq, score, w_b, flags);
  } else {
    auto kb = window_score_kernel<D, false>;
    if (!ensure_smem_attr((const void*)kb, ScShape<D, false>::kSmem)) return cudaErrorInvalidValue;
    kb<<<dim3(nsb, units), kFuThreads, ScShape<D, false>::kSmem, st>>>(
        mQ, mK, mV, mEh, mEm, mEl, (const bf16*)V, logn, len, cand_begin, n_recent, d.H_kv,
        d.H_q, W, d.T_cap, nsb, capc ? 1 : 0, form, stats, obar, zq, wq, score, w_b, flags);
  }
  count_launches(4);
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
