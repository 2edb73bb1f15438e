// Split-K GQA decode over a bf16 cache: TMA-fed shared-memory pipeline and
// warp-level tensor-core MMAs.
//
// Attention of the KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程",
// §数学主线三) with the log-count logit bias of merged rows; the decoder stage the
// pages time (Figure 5). The step is HBM-bound (about 4 flop per byte), so the
// design goal is to keep every byte of K and V moving: one producer warp issues
// 2D TMA tile loads (128-byte swizzle, no multicast, L2 evict-first) of 16 * NC
// cache rows of K and V into a ring of shared-memory stages guarded by mbarriers;
// NC consumer warps each take 16 rows of a stage. The problem is computed
// transposed so that the cache rows fill the MMA's M dimension and the G query
// heads its N = 8 columns: S^T = K Q^T by m16n8k16 MMAs, the online softmax on the
// accumulator fragments, the probability tile transposed in registers (movmatrix)
// and O^T += V^T P^T by a second set of MMAs.
//
// Two launch shapes share the main loop:
//  - split grid (NC = 4, two CTAs per SM, nsplit splits per KV head): each CTA
//    publishes a partial row, and the last CTA of a head to arrive combines them
//    (decode_common.cuh); no CTA waits on another;
//  - cluster grid (NC = 8, one CTA per SM): the C splits of a KV head form one
//    thread-block cluster and combine their partials through distributed shared
//    memory, with no global partials and no arrival counter. Used when every head's
//    cluster fits on the GPU at once (few heads, as in single-sequence decode).
#include <cudaTypedefs.h>

#include <map>
#include <type_traits>
#include <mutex>
#include <utility>

#include "decode_common.cuh"
#include "kvs_common.cuh"
#include "kvs_kernels.h"
#include "ptx.cuh"

namespace kvs {


// Lazy reference of the decode's online softmax: it moves when a logit exceeds it by this
// much (log2 units), so probabilities stay <= 2^8 between moves.
constexpr float kDecodeSlack = 8.f;

template <int D, int NC, int STAGES, int EXTRA>
struct TcShape {
  static constexpr int kTile = 16 * NC;                    // cache rows per stage
  static constexpr int kThreads = (NC + 1 + EXTRA) * 32;   // consumers, producer, extra
  static constexpr int kBoxes = D / 64;                    // 128-byte boxes per row
  static constexpr int kBoxBytes = kTile * 128;            // one box of one stage
  static constexpr int kTileBytes = kBoxes * kBoxBytes;    // K (or V) rows of one stage
  static constexpr int kStageBytes = 2 * kTileBytes;       // K then V
  static constexpr int kRingBytes = STAGES * kStageBytes;
  // log-counts of a stage: kTile + 4 floats from a 16-byte aligned start (TMA needs
  // the start coordinate of an fp32 box to be a multiple of 4), one slot per stage
  static constexpr int kLnBox = kTile + 4;
  static constexpr int kLnSlot = 1024;
  static_assert(kLnBox * 4 <= kLnSlot, "log-count slot");
  static constexpr int kSmem = kRingBytes + STAGES * kLnSlot + (2 * STAGES + 1) * 8 + 1024;
  // the split combine stages all splits of at least one query head in the ring
  static_assert(kMaxDecodeSplits * (D + kPartPad) * 4 <= kRingBytes, "combine staging");
};

// the two launch shapes (the cluster shape adds the warp that pre-runs the combine)
template <int D> using SplitShape = TcShape<D, 4, 3, 0>;
template <int D> using ClusterShape = TcShape<D, 8, D == 64 ? 6 : 3, 1>;

template <int D, int G, int NC, int STAGES, bool kCluster>
__global__ void __launch_bounds__((NC + (kCluster ? 2 : 1)) * 32, kCluster ? 1 : 2)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmL, int ln_lead,
                 const bf16* __restrict__ q, bf16* K, bf16* V, float* logn, int32_t* len,
                 const bf16* __restrict__ k_new, const bf16* __restrict__ v_new,
                 bf16* __restrict__ out, int T_cap, int nsplit, int32_t* counters, float* part,
                 int32_t* flags) {
  using S = TcShape<D, NC, STAGES, kCluster ? 1 : 0>;
  constexpr int kTile = S::kTile, kThreads = S::kThreads;
  static_assert(NC * G * D * 4 <= S::kRingBytes, "warp partials fit the ring");
  extern __shared__ unsigned char dsm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(dsm) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* ln_ring = base + S::kRingBytes;   // STAGES log-count slots
  uint64_t* full = reinterpret_cast<uint64_t*>(ln_ring + STAGES * S::kLnSlot);
  uint64_t* empty = full + STAGES;
  uint64_t* cbar = empty + STAGES;                 // the split combine's bulk copies
  __shared__ __align__(16) float qs[G][D];
  __shared__ float s_m[NC][G], s_l[NC][G];
  __shared__ float s_new[G];
  __shared__ float s_fac[G][kMaxDecodeSplits];
  __shared__ float s_gstat[G][2];
  __shared__ int s_last;
  // cluster shape: the inbox peers push into, the scratch of the warm-up run, and the
  // appended row (k, v) staged at kernel start
  using Inbox = std::conditional_t<kCluster, ClusterInbox<D, G>, char>;
  __shared__ Inbox s_inbox[2];
  __shared__ __align__(16) bf16 s_kvnew[kCluster ? 2 : 1][kCluster ? D : 8];
  __shared__ uint64_t s_inbar[2];   // cluster shape: the inbox's barrier, the scratch inbox's
  // after the main loop the stage buffers hold the consumer warps' partial outputs
  float(*s_acc)[G][D] = reinterpret_cast<float(*)[G][D]>(base);

  // Launched with programmatic stream serialisation: the grid may be scheduled before the
  // previous kernel of the stream has finished, but every access waits for that kernel's
  // completion and memory here, so ordering is as in plain stream order; the early
  // trigger lets the next decode launch be scheduled in turn.
  griddep_wait();
  griddep_launch_dependents();
  const int head = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == NC * 32) {   // the producer: descriptor fetches overlap the length load
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    if (logn != nullptr) prefetch_tmap(&tmL);
  }
  // Every global load of the prologue goes out before the length comes back: this
  // thread's share of the query (staged in shared memory below), the appended row (the
  // cluster shape stages it whatever the length turns out to be; `append` gates its
  // use) and, in the consumer warps, the query fragments of the S^T MMAs.
  constexpr int kQPer = (G * D + kThreads - 1) / kThreads;
  float qv[kQPer];
#pragma unroll
  for (int r = 0; r < kQPer; ++r) {
    const int i = tid + r * kThreads;
    qv[r] = i < G * D ? to_f32(q[(size_t)head * G * D + i]) : 0.f;
  }
  const bool want_append = k_new != nullptr && v_new != nullptr;
  static_assert(!kCluster || 2 * D <= kThreads, "one appended element per thread");
  bf16 kvv = __float2bfloat16_rn(0.f);
  // element loads: the API does not require these rows to be 16-byte aligned
  if (kCluster && want_append && tid < 2 * D)
    kvv = (tid < D ? k_new : v_new)[(size_t)head * D + tid % D];
  // B operand of S^T = K Q^T in consumer lane (grp, tig): column n = grp holds query
  // head grp (zero past G)
  uint32_t qb[D / 16][2];
  {
    const int grp = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      if (warp < NC && grp < G) {
        const bf16* qr = q + ((size_t)head * G + grp) * D + ks * 16 + tig * 2;
        qb[ks][0] = *reinterpret_cast<const uint32_t*>(qr);
        qb[ks][1] = *reinterpret_cast<const uint32_t*>(qr + 8);
      } else {
        qb[ks][0] = qb[ks][1] = 0u;
      }
    }
  }
  int L = len[head];
  const bool bad = L < 0 || L > T_cap;
  if (bad) {
    if (split == 0 && tid == 0) set_flag(flags, KVS_FLAG_BAD_LENGTH);
    L = 0;
  }
  // whole tiles per split, the remainder spread one tile each (at most one tile of
  // imbalance, whatever the length)
  const long long T = (L + kTile - 1) / kTile;
  const int tb = (int)(split * T / nsplit), te = (int)((split + 1) * T / nsplit);
  const int t0 = tb * kTile, t1 = min(L, te * kTile);
  const int ntiles = t1 > t0 ? te - tb : 0;
  const int row0 = head * T_cap + t0;            // B*H_kv*T_cap < 2^31 (host check)
  // log-counts of tile i start at element e = ln_lead + row0 + i * kTile of the
  // log-count map; its box starts at e rounded down to a multiple of 4 (so every
  // tile's offset is (ln_lead + row0) & 3, kTile being a multiple of 4)
  const bool has_ln = logn != nullptr;
  const int ln_off = (ln_lead + row0) & 3;

  const bool append = want_append && !bad;
  // One thread issues every TMA load of the ring: stage i % STAGES takes the K and V rows
  // of tile i (and its log-counts) and signals full[s] when they have landed.
  const bool producer = tid == NC * 32;
  const uint64_t once = policy_evict_first();   // K and V are read once per step
  auto issue = [&](int i) {
    const int s = i % STAGES;
    unsigned char* st = base + s * S::kStageBytes;
    mbar_arrive_expect_tx(&full[s], S::kStageBytes + (has_ln ? S::kLnBox * 4 : 0));
    if (has_ln)
      tma_load_1d_hint(ln_ring + s * S::kLnSlot, &tmL, ln_lead + row0 + i * kTile - ln_off,
                       &full[s], once);
#pragma unroll
    for (int bx = 0; bx < S::kBoxes; ++bx) {
      tma_load_2d_hint(st + bx * S::kBoxBytes, &tmK, bx * 64, row0 + i * kTile, &full[s], once);
      tma_load_2d_hint(st + S::kTileBytes + bx * S::kBoxBytes, &tmV, bx * 64, row0 + i * kTile,
                       &full[s], once);
    }
  };
  // The producer sets up the barriers and fills the ring as soon as the length is known,
  // before it takes its share of the query and appended-row staging that the CTA barrier
  // below waits for: the first stages are in flight while those loads complete.
  int issued = 0;
  if (producer) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NC);
    }
    mbar_init(cbar, 1);
    if constexpr (kCluster) {
      mbar_init(&s_inbar[0], 1);
      mbar_init(&s_inbar[1], 1);
    }
    fence_mbar_init();
    for (; issued < STAGES && issued < ntiles; ++issued) issue(issued);
    if constexpr (kCluster) {
      constexpr int NU = G * D / 4;
      mbar_arrive_expect_tx(&s_inbar[0], inbox_bytes<G>(NU, nsplit, (int)cluster_ctarank()));
      mbar_arrive_expect_tx(&s_inbar[1], dry_inbox_bytes<G>(NU, nsplit));
    }
  }
  const float qscale = kLog2e / sqrtf((float)D);
#pragma unroll
  for (int r = 0; r < kQPer; ++r) {
    const int i = tid + r * kThreads;
    if (i < G * D) qs[i / D][i % D] = qv[r] * qscale;
  }
  if (kCluster && want_append && tid < 2 * D) s_kvnew[tid / D][tid % D] = kvv;
  __syncthreads();
  // every CTA's inbox barrier is initialised before any peer pushes into it (the combine
  // opens with the matching wait)
  if constexpr (kCluster) cluster_arrive_relaxed();

  // per consumer lane: two query-head columns n0 = 2 tig, n1 = 2 tig + 1 of the
  // transposed problem (running max, this lane's share of the sum) and the
  // transposed output O^T[d][n] for d = 16 j + grp (+8)
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float O[D / 16][4];
#pragma unroll
  for (int j = 0; j < D / 16; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;

  if (kCluster && warp == NC + 1) {
    // ---------------- the extra warp, while the others stream: the appended row's
    // logits (read by the combine), then the combine's code run dry ----------------
    if constexpr (kCluster) {
      if (append && L < T_cap) {
        for (int g = 0; g < G; ++g) {
          float sp = 0.f;
          for (int c = lane; c < D; c += 32) sp = fmaf(qs[g][c], to_f32(s_kvnew[0][c]), sp);
          sp = warp_sum(sp);
          if (lane == 0) s_new[g] = sp;
        }
      }
      cluster_combine<bf16, D, G, NC>(s_m, s_l, s_acc, s_new, &s_inbox[1], &s_inbar[1], nsplit,
                                      (int)cluster_ctarank(), lane, 32, /*dry=*/true, 0, L, T_cap,
                                      append, K, V, logn, len, s_kvnew[0], s_kvnew[kCluster ? 1 : 0],
                                      reinterpret_cast<bf16*>(&s_inbox[1]), flags);
      // its pushes into the scratch inbox have all landed before the CTA can leave
      if (lane == 0 && !mbar_wait(&s_inbar[1], 0)) set_flag(flags, KVS_FLAG_TIMEOUT);
    }
  } else if (warp == NC) {
    // ---------------- producer: one thread issues every TMA load ----------------
    if (lane == 0) {
      // the first STAGES tiles went out before the CTA barrier; the rest wait for a free stage
      for (int i = issued; i < ntiles; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&empty[s], ((i / STAGES) - 1) & 1)) {
          set_flag(flags, KVS_FLAG_TIMEOUT);
          break;
        }
        issue(i);
        issued = i + 1;
      }
      // the last load issued into each stage must land before the buffers are reused
      for (int i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
        if (!mbar_wait(&full[i % STAGES], (i / STAGES) & 1)) set_flag(flags, KVS_FLAG_TIMEOUT);
    }
    __syncwarp();   // reconverge before the CTA-wide barrier after the main loop
  } else if (warp < NC) {
    // ---------------- consumers: 16 rows of each stage per warp ----------------
    const int grp = lane >> 2;                       // fragment row
    const int mi = lane >> 3, ri = lane & 7;         // ldmatrix: matrix index, row in matrix
    const int r0 = warp * 16;                        // this warp's rows inside a stage
    const uint32_t ring = smem_u32(base);
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % STAGES;
      // ldmatrix / mma are warp-collective: the whole warp leaves together
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / STAGES) & 1))) {
        set_flag(flags, KVS_FLAG_TIMEOUT);
        break;
      }
      const uint32_t kb = ring + s * S::kStageBytes;
      const uint32_t vb = kb + S::kTileBytes;
      const int tok0 = t0 + i * kTile + r0;
      const int nval = min(16, t1 - tok0);
      if (nval > 0) {
        if (nval < 16) {
          // rows past the split's end may hold anything: zero their values so that
          // 0-probability x value stays 0 (keys are masked below)
          unsigned char* vrow = base + s * S::kStageBytes + S::kTileBytes;
          for (int idx = lane; idx < (16 - nval) * S::kBoxes * 8; idx += 32) {
            const int rr = r0 + nval + idx / (S::kBoxes * 8);
            const int rem = idx % (S::kBoxes * 8);
            *reinterpret_cast<uint4*>(vrow + (rem >> 3) * S::kBoxBytes + rr * 128 + (rem & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        // The warp's V fragments (A operands of O^T += V^T P^T) first, kept in registers,
        // then its K fragments straight into the S^T MMAs, and the stage's log-counts: the
        // warp is then done with the stage's shared memory and releases it before its
        // softmax and P V MMAs, so the producer refills it while they run.
        uint32_t vf[D / 16][4];
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          const int row = r0 + ((mi >> 1) << 3) + ri;
          const int el = j * 16 + ((mi & 1) << 3);
          ldsm_x4_trans(vb + (el >> 6) * S::kBoxBytes + swz128(row, (el & 63) >> 3), vf[j][0],
                        vf[j][1], vf[j][2], vf[j][3]);
        }
        // S^T (16 rows x 8 columns): A = the K rows, two accumulators to halve the chain
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int row = r0 + ((mi & 1) << 3) + ri;
          const int el = ks * 16 + ((mi >> 1) << 3);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kb + (el >> 6) * S::kBoxBytes + swz128(row, (el & 63) >> 3), a0, a1, a2, a3);
          if (ks & 1)
            mma_bf16_16816(sb, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
          else
            mma_bf16_16816(sa, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
        }
        // log-counts of this lane's rows grp and grp + 8 (landed with the stage)
        float2 ln_cur = make_float2(0.f, 0.f);
        if (has_ln) {
          const float* lns = reinterpret_cast<const float*>(ln_ring + s * S::kLnSlot) + ln_off + r0;
          ln_cur = make_float2(lns[grp], lns[grp + 8]);
        }
        // every shared-memory read of the stage is issued (the arrive orders them before it)
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        const bool v0 = grp < nval, v1 = grp + 8 < nval;
        const float x0 = v0 ? fmaf(sa[0] + sb[0], qscale, ln_cur.x * kLog2e) : -INFINITY;
        const float x1 = v0 ? fmaf(sa[1] + sb[1], qscale, ln_cur.x * kLog2e) : -INFINITY;
        const float x2 = v1 ? fmaf(sa[2] + sb[2], qscale, ln_cur.y * kLog2e) : -INFINITY;
        const float x3 = v1 ? fmaf(sa[3] + sb[3], qscale, ln_cur.y * kLog2e) : -INFINITY;
        // The reference maximum of a column moves only when a logit exceeds it by 2^8
        // (so P <= 2^8 between moves); the column maxima over the 16 rows (the 8 lanes
        // sharing tig) and the rescale of l and O are taken only when some lane's logit
        // does, which after the first stages is rare.
        const bool up = x0 > m0 + kDecodeSlack || x2 > m0 + kDecodeSlack ||
                        x1 > m1 + kDecodeSlack || x3 > m1 + kDecodeSlack;
        if (__any_sync(0xffffffffu, up)) {
          float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
          }
          const float mn0 = mx0 > m0 + kDecodeSlack ? mx0 : m0;
          const float mn1 = mx1 > m1 + kDecodeSlack ? mx1 : m1;
          // factors of the old reference (0 when there was none: l and O are still 0)
          const float c0 = mn0 == m0 ? 1.f : ex2_ftz(m0 - mn0);
          const float c1 = mn1 == m1 ? 1.f : ex2_ftz(m1 - mn1);
          l0 *= c0;
          l1 *= c1;
#pragma unroll
          for (int j = 0; j < D / 16; ++j) {
            O[j][0] *= c0; O[j][1] *= c1; O[j][2] *= c0; O[j][3] *= c1;
          }
          m0 = mn0;
          m1 = mn1;
        }
        const float b0 = m0 == -INFINITY ? 0.f : m0;       // all -inf so far: keep zeros
        const float b1 = m1 == -INFINITY ? 0.f : m1;
        const float p0 = ex2_ftz(x0 - b0), p1 = ex2_ftz(x1 - b1);
        const float p2 = ex2_ftz(x2 - b0), p3 = ex2_ftz(x3 - b1);
        l0 += p0 + p2;
        l1 += p1 + p3;
        // P^T as the B operand: transpose the two 8x8 bf16 blocks (rows 0-7, 8-15)
        const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));
        const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));
#pragma unroll
        for (int j = 0; j < D / 16; ++j) mma_bf16_16816(O[j], vf[j][0], vf[j][1], vf[j][2], vf[j][3], pb0, pb1);
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);   // no rows of this warp in the stage
      }
    }
    // the lanes sharing tig hold disjoint rows' shares of the column sums
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
  }

  // every TMA write has landed and every read is done: reuse the ring for partials
  __syncthreads();
  if (warp < NC) {
    const int grp = lane >> 2, n0 = 2 * (lane & 3), n1 = n0 + 1;
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      if (n0 < G) {
        s_acc[warp][n0][16 * j + grp] = O[j][0];
        s_acc[warp][n0][16 * j + grp + 8] = O[j][2];
      }
      if (n1 < G) {
        s_acc[warp][n1][16 * j + grp] = O[j][1];
        s_acc[warp][n1][16 * j + grp + 8] = O[j][3];
      }
    }
    if (grp == 0) {
      if (n0 < G) { s_m[warp][n0] = m0; s_l[warp][n0] = l0; }
      if (n1 < G) { s_m[warp][n1] = m1; s_l[warp][n1] = l1; }
    }
  }
  __syncthreads();
  const DecodeSmem<D, G, NC> Sm{s_m, s_l, s_acc, qs, s_new, s_fac, s_gstat, &s_last};
  const DecodeArgs<bf16> a{head, split, nsplit, L, T_cap, bad, K, V, logn, len, k_new, v_new,
                           out, counters, part, flags};
  if constexpr (kCluster) {
    cluster_combine<bf16, D, G, NC>(s_m, s_l, s_acc, s_new, &s_inbox[0], &s_inbar[0], nsplit,
                                    (int)cluster_ctarank(), tid, kThreads, /*dry=*/false, head, L,
                                    T_cap, append, K, V, logn, len, s_kvnew[0],
                                    s_kvnew[kCluster ? 1 : 0], out, flags);
  } else {
    decode_epilogue_staged<bf16, D, G, NC>(Sm, base, S::kRingBytes, cbar, a, tid, kThreads);
  }
}


// ---------------------------------------------------------------------------
// Host side: tensor maps over the whole cache ([B*H_kv*T_cap rows, d] bf16) and launch
// ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool encode_rows_map(CUtensorMap* map, const void* base, unsigned long long rows, int d,
                     int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * sizeof(bf16)};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 1D map over the log-counts, starting at the 16-byte boundary at or below `logn`;
// *lead = the elements between that boundary and logn (0..3). Elements past the end
// read as zero; the few before logn lie in the same 16-byte chunk, so the same page.
static bool encode_ln_map(CUtensorMap* map, const float* logn, unsigned long long n, int box,
                          int* lead) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const uintptr_t a = reinterpret_cast<uintptr_t>(logn);
  const uintptr_t b = a & ~static_cast<uintptr_t>(15);
  *lead = (int)((a - b) / sizeof(float));
  cuuint64_t dims[1] = {(cuuint64_t)(n + *lead)};
  cuuint64_t strides[1] = {0};
  cuuint32_t boxd[1] = {(cuuint32_t)box};
  cuuint32_t estr[1] = {1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, reinterpret_cast<void*>(b), dims, strides,
             boxd, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool decode_tc_supported(const kvs_cache_desc& d) {
  const unsigned long long rows = (unsigned long long)d.B * d.H_kv * (unsigned long long)d.T_cap;
  return d.dtype == KVS_BF16 && (d.d == 64 || d.d == 128) && rows < (1ull << 31) &&
         tensor_map_encoder() != nullptr;
}

// Cluster size for a cluster launch over `units` KV heads on the current device, or
// 0 when the split grid is to be used: the largest C <= 16 with C * units <= SM count
// for which the occupancy calculator places all `units` clusters at once.
template <int D, int G>
static int cluster_size_for(int units) {
  using CS = ClusterShape<D>;
  auto kfn = decode_tc_kernel<D, G, 8, (D == 64 ? 6 : 3), true>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_pair(dev, units);
  const auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int C = units > 0 ? sms / units : 0;
  if (C > kMaxClusterSize) C = kMaxClusterSize;
  if (!ensure_smem_attr((const void*)kfn, CS::kSmem)) C = 0;
  if (C > 8 && !ensure_nonportable_cluster((const void*)kfn)) C = 8;
  for (; C >= 2; --C) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, units);
    cfg.blockDim = dim3(CS::kThreads);
    cfg.dynamicSmemBytes = CS::kSmem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = C;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (const void*)kfn, &cfg) == cudaSuccess && n >= units) break;
  }
  (void)cudaGetLastError();   // a refused query leaves no error behind
  if (C < 2) C = 0;
  cache[key] = C;
  return C;
}

template <int D, int G, int NC, int STAGES, bool kCluster>
static cudaError_t launch_shape(const kvs_cache_desc& d, const void* q, void* K, void* V,
                                float* logn, int32_t* len, const void* k_new, const void* v_new,
                                void* out, int nsplit, const DecodeLayout& Ly, char* ws,
                                cudaStream_t st) {
  using S = TcShape<D, NC, STAGES, kCluster ? 1 : 0>;
  auto kfn = decode_tc_kernel<D, G, NC, STAGES, kCluster>;
  // per device, cached (the first call on a device must precede any capture)
  if (!ensure_smem_attr((const void*)kfn, S::kSmem)) return cudaErrorInvalidValue;
  if (kCluster && nsplit > 8 && !ensure_nonportable_cluster((const void*)kfn))
    return cudaErrorInvalidValue;
  const unsigned long long rows = (unsigned long long)d.B * d.H_kv * (unsigned long long)d.T_cap;
  CUtensorMap mK, mV, mL;
  if (!encode_rows_map(&mK, K, rows, d.d, S::kTile) || !encode_rows_map(&mV, V, rows, d.d, S::kTile))
    return cudaErrorInvalidValue;
  int ln_lead = 0;
  if (logn) {
    if (!encode_ln_map(&mL, logn, rows, S::kLnBox, &ln_lead)) return cudaErrorInvalidValue;
  } else {
    mL = mK;   // never read
  }
  // Programmatic stream serialisation: this grid is scheduled while the previous one
  // finishes (the kernel waits for it before any access); measured 0.35 us less per
  // 128K decode launch than plain stream order.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nsplit, d.B * d.H_kv);
  cfg.blockDim = dim3(S::kThreads);
  cfg.dynamicSmemBytes = S::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = nsplit;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = kCluster ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, kfn, mK, mV, mL, ln_lead, (const bf16*)q, (bf16*)K, (bf16*)V, logn, len, (const bf16*)k_new,
      (const bf16*)v_new, (bf16*)out, d.T_cap, nsplit,
      reinterpret_cast<int32_t*>(ws + Ly.counters), reinterpret_cast<float*>(ws + Ly.part),
      reinterpret_cast<int32_t*>(ws));
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D, int G>
static cudaError_t launch_tc(const kvs_cache_desc& d, const void* q, void* K, void* V,
                             float* logn, int32_t* len, const void* k_new, const void* v_new,
                             void* out, const DecodeLayout& Ly, char* ws, cudaStream_t st) {
  const int C = cluster_size_for<D, G>(d.B * d.H_kv);
  if (C >= 2)
    return launch_shape<D, G, 8, (D == 64 ? 6 : 3), true>(d, q, K, V, logn, len, k_new, v_new, out,
                                                          C, Ly, ws, st);
  return launch_shape<D, G, 4, 3, false>(d, q, K, V, logn, len, k_new, v_new, out, Ly.nsplit, Ly,
                                         ws, st);
}

cudaError_t launch_decode_tc(const kvs_cache_desc& d, const void* q, void* K, void* V, float* logn,
                             int32_t* len, const void* k_new, const void* v_new, void* out,
                             const DecodeLayout& Ly, char* ws, cudaStream_t st) {
  const int G = d.H_q / d.H_kv;
#define KVS_TC(DD, GG) \
  if (d.d == DD && G == GG) return launch_tc<DD, GG>(d, q, K, V, logn, len, k_new, v_new, out, Ly, ws, st)
  KVS_TC(128, 1); KVS_TC(128, 2); KVS_TC(128, 4); KVS_TC(128, 8);
  KVS_TC(64, 1); KVS_TC(64, 2); KVS_TC(64, 4); KVS_TC(64, 8);
#undef KVS_TC
  return cudaErrorInvalidValue;
}

}  // namespace kvs
