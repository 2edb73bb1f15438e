// Split-K GQA decode over a bf16 cache: TMA-fed shared-memory pipeline and
// warp-level tensor-core MMAs.
//
// Attention of the KVSlimmer deep dive ("论文专题讲解：KVSlimmer：非对称 KV 合并的数学与工程",
// §数学主线三) with the log-count logit bias of merged rows; the decoder stage the
// pages time (Figure 5). The step is HBM-bound (about 4 flop per byte), so the
// design goal is to keep every byte of K and V moving: one producer warp issues
// 2D TMA tile loads (128-byte swizzle, no multicast) of 64 cache rows of K and V
// into a 3-stage ring of shared-memory buffers guarded by mbarriers; four consumer
// warps each take 16 rows of a stage, compute the logits of the G query heads with
// m16n8k16 MMAs (the G heads padded to the 16-row A tile), run the online softmax
// in registers, and accumulate P V with a second set of MMAs whose A operand is the
// probability tile repacked from the logit accumulators. Two CTAs fit on an SM, and
// the grid covers every (KV head, split) once. The split partials are combined by
// the last CTA to arrive (decode_common.cuh); no CTA waits on another.
#include <cudaTypedefs.h>

#include "decode_common.cuh"
#include "kvs_common.cuh"
#include "kvs_kernels.h"
#include "ptx.cuh"

namespace kvs {

constexpr int kTcTile = 64;                        // cache rows per pipeline stage
constexpr int kTcStages = 3;
constexpr int kTcConsumers = 4;                    // consumer warps, 16 rows each
constexpr int kTcThreads = (kTcConsumers + 1) * 32;

template <int D>
struct TcShape {
  static constexpr int kBoxes = D / 64;                    // 128-byte boxes per row
  static constexpr int kBoxBytes = kTcTile * 128;          // one box of one stage
  static constexpr int kTileBytes = kBoxes * kBoxBytes;    // K (or V) rows of one stage
  static constexpr int kStageBytes = 2 * kTileBytes;       // K then V
  static constexpr int kSmem = kTcStages * kStageBytes + 2 * kTcStages * 8 + 1024;
};

template <int D, int G>
__global__ void __launch_bounds__(kTcThreads, 2)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const bf16* __restrict__ q, bf16* K, bf16* V, float* logn, int32_t* len,
                 const bf16* __restrict__ k_new, const bf16* __restrict__ v_new,
                 bf16* __restrict__ out, int T_cap, int nsplit, int32_t* counters,
                 float* part_ml, float* part_acc, int32_t* flags) {
  using S = TcShape<D>;
  static_assert(G * D * 4 * kTcConsumers <= kTcStages * S::kStageBytes, "epilogue overlay");
  extern __shared__ unsigned char dsm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(dsm) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kTcStages * S::kStageBytes);
  uint64_t* empty = full + kTcStages;
  __shared__ __align__(16) float qs[G][D];
  __shared__ float s_m[kTcConsumers][G], s_l[kTcConsumers][G];
  __shared__ float s_new[G];
  __shared__ int s_last;
  // after the main loop the stage buffers hold the consumer warps' partial outputs
  float(*s_acc)[G][D] = reinterpret_cast<float(*)[G][D]>(base);

  const int head = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_trigger();
  pdl_wait();     // nothing above this line touches global memory
  int L = len[head];
  const bool bad = L < 0 || L > T_cap;
  if (bad) {
    if (split == 0 && tid == 0) set_flag(flags, KVS_FLAG_BAD_LENGTH);
    L = 0;
  }
  int chunk = (L + nsplit - 1) / nsplit;
  chunk = (chunk + kTcTile - 1) / kTcTile * kTcTile;
  const int t0 = split * chunk, t1 = min(L, t0 + chunk);
  const int ntiles = t1 > t0 ? (t1 - t0 + kTcTile - 1) / kTcTile : 0;
  const int row0 = head * T_cap + t0;            // B*H_kv*T_cap < 2^31 (host check)

  const float qscale = kLog2e / sqrtf((float)D);
  for (int i = tid; i < G * D; i += kTcThreads) {
    const int g = i / D, c = i - g * D;
    qs[g][c] = to_f32(q[((size_t)head * G + g) * D + c]) * qscale;
  }
  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kTcConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();

  float m_run = -INFINITY, l_run = 0.f;
  float O[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.f;

  if (warp == kTcConsumers) {
    // ---------------- producer: one thread issues every TMA load ----------------
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % kTcStages;
        if (i >= kTcStages && !mbar_wait(&empty[s], ((i / kTcStages) - 1) & 1)) {
          set_flag(flags, KVS_FLAG_TIMEOUT);
          break;
        }
        unsigned char* st = base + s * S::kStageBytes;
        mbar_arrive_expect_tx(&full[s], S::kStageBytes);
#pragma unroll
        for (int bx = 0; bx < S::kBoxes; ++bx) {
          tma_load_2d(st + bx * S::kBoxBytes, &tmK, bx * 64, row0 + i * kTcTile, &full[s]);
          tma_load_2d(st + S::kTileBytes + bx * S::kBoxBytes, &tmV, bx * 64, row0 + i * kTcTile,
                      &full[s]);
        }
        issued = i + 1;
      }
      // the last load issued into each stage must land before the buffers are reused
      for (int i = issued > kTcStages ? issued - kTcStages : 0; i < issued; ++i)
        if (!mbar_wait(&full[i % kTcStages], (i / kTcStages) & 1)) set_flag(flags, KVS_FLAG_TIMEOUT);
    }
    __syncwarp();   // reconverge before the CTA-wide barrier after the main loop
  } else {
    // ---------------- consumers: 16 rows of each stage per warp ----------------
    const int grp = lane >> 2, tig = lane & 3;       // MMA fragment row / column pair
    const int mi = lane >> 3, ri = lane & 7;         // ldmatrix: matrix index, row in matrix
    // query A fragments: row grp (< G) of the 16-row tile, k pairs (2 tig, +1) and (+8);
    // rows 8..15 of the tile are padding and stay zero
    uint32_t qa[D / 16][2];
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      if (grp < G) {
        const bf16* qr = q + ((size_t)head * G + grp) * D + ks * 16 + tig * 2;
        qa[ks][0] = *reinterpret_cast<const uint32_t*>(qr);
        qa[ks][1] = *reinterpret_cast<const uint32_t*>(qr + 8);
      } else {
        qa[ks][0] = qa[ks][1] = 0u;
      }
    }
    const float* lnh = logn ? logn + (size_t)head * T_cap : nullptr;
    const int r0 = warp * 16;                        // this warp's rows inside a stage
    const uint32_t ring = smem_u32(base);
    // log-counts of this lane's four rows of a tile, fetched one tile ahead so the
    // global-memory latency overlaps the previous tile's work (rows 8j + 2 tig + e;
    // the row index is even, so each pair is one aligned 8-byte load)
    auto fetch_ln = [&](int tile, float2 (&dst)[2]) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int tok = t0 + tile * kTcTile + r0 + 8 * j + 2 * tig;
        dst[j] = (lnh && tile < ntiles && tok < t1) ? *reinterpret_cast<const float2*>(lnh + tok)
                                                    : make_float2(0.f, 0.f);
      }
    };
    float2 ln_cur[2], ln_next[2];
    fetch_ln(0, ln_cur);
    for (int i = 0; i < ntiles; ++i) {
      fetch_ln(i + 1, ln_next);
      const int s = i % kTcStages;
      // ldmatrix / mma are warp-collective: the whole warp leaves together
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / kTcStages) & 1))) {
        set_flag(flags, KVS_FLAG_TIMEOUT);
        break;
      }
      const uint32_t kb = ring + s * S::kStageBytes;
      const uint32_t vb = kb + S::kTileBytes;
      const int tok0 = t0 + i * kTcTile + r0;
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
        // logits of the 16 rows: two 8-row n-tiles
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int row = r0 + ((mi >> 1) << 3) + ri;
          const int el = ks * 16 + ((mi & 1) << 3);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + (el >> 6) * S::kBoxBytes + swz128(row, (el & 63) >> 3), b0, b1, b2, b3);
          mma_bf16_16816(sc[0], qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
          mma_bf16_16816(sc[1], qa[ks][0], 0u, qa[ks][1], 0u, b2, b3);
        }
        // online softmax on row grp: this lane holds rows tok0 + 8j + 2 tig + e
        float p[2][2];
        float mloc = -INFINITY;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tok = tok0 + 8 * j + 2 * tig + e;
            float sv = -INFINITY;
            const float lnv = e ? ln_cur[j].y : ln_cur[j].x;
            if (tok < t1) sv = fmaf(sc[j][e], qscale, lnv * kLog2e);
            p[j][e] = sv;
            mloc = fmaxf(mloc, sv);
          }
        }
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
        const float m_new = fmaxf(m_run, mloc);
        const float corr = exp2f(m_run - m_new);
        float psum = 0.f;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            p[j][e] = exp2f(p[j][e] - m_new);
            psum += p[j][e];
          }
        psum += __shfl_xor_sync(0xffffffffu, psum, 1);
        psum += __shfl_xor_sync(0xffffffffu, psum, 2);
        l_run = l_run * corr + psum;
        m_run = m_new;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          O[n][0] *= corr;
          O[n][1] *= corr;
        }
        // P (bf16) as the A operand: k = the 16 rows, row grp; padding rows zero
        const uint32_t pa0 = pack_bf16x2(p[0][0], p[0][1]);
        const uint32_t pa2 = pack_bf16x2(p[1][0], p[1][1]);
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          const int row = r0 + ((mi & 1) << 3) + ri;
          const int el = j * 16 + ((mi >> 1) << 3);
          uint32_t v0, v1, v2, v3;
          ldsm_x4_trans(vb + (el >> 6) * S::kBoxBytes + swz128(row, (el & 63) >> 3), v0, v1, v2, v3);
          mma_bf16_16816(O[2 * j], pa0, 0u, pa2, 0u, v0, v1);
          mma_bf16_16816(O[2 * j + 1], pa0, 0u, pa2, 0u, v2, v3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      ln_cur[0] = ln_next[0];
      ln_cur[1] = ln_next[1];
    }
  }

  // every TMA write has landed and every read is done: reuse the ring for partials
  __syncthreads();
  if (warp < kTcConsumers) {
    const int grp = lane >> 2, tig = lane & 3;
    if (grp < G) {
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        s_acc[warp][grp][n * 8 + tig * 2] = O[n][0];
        s_acc[warp][grp][n * 8 + tig * 2 + 1] = O[n][1];
      }
      if (tig == 0) {
        s_m[warp][grp] = m_run;
        s_l[warp][grp] = l_run;
      }
    }
  }
  __syncthreads();
  // the combine scratch sits in the ring after the warp partials
  float* scratch = reinterpret_cast<float*>(base) + kTcConsumers * G * D;
  static_assert((kTcConsumers * G * D + 2 * G * 64 + 2 * G) * 4 <= kTcStages * S::kStageBytes,
                "combine scratch fits the ring");
  decode_epilogue<bf16, D, G, kTcConsumers>(s_m, s_l, s_acc, qs, s_new, &s_last, scratch, tid,
                                            kTcThreads, head, split, nsplit, L, bad, T_cap, K, V,
                                            logn, len, k_new, v_new, out, counters, part_ml,
                                            part_acc, flags);
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

bool decode_tc_supported(const kvs_cache_desc& d) {
  const unsigned long long rows = (unsigned long long)d.B * d.H_kv * (unsigned long long)d.T_cap;
  return d.dtype == KVS_BF16 && (d.d == 64 || d.d == 128) && rows < (1ull << 31) &&
         tensor_map_encoder() != nullptr;
}

template <int D, int G>
static cudaError_t launch_tc(const kvs_cache_desc& d, const CUtensorMap& mK, const CUtensorMap& mV,
                             const void* q, void* K, void* V, float* logn, int32_t* len,
                             const void* k_new, const void* v_new, void* out,
                             const DecodeLayout& Ly, char* ws, cudaStream_t st) {
  auto kfn = decode_tc_kernel<D, G>;
  static bool attr = false;   // set once per process, before any capture
  if (!attr) {
    if (cudaFuncSetAttribute((const void*)kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             TcShape<D>::kSmem) != cudaSuccess)
      return cudaErrorInvalidValue;
    attr = true;
  }
  // programmatic serialization lets this grid launch while the previous one drains;
  // the kernel waits for it (griddepcontrol.wait) before any global-memory access
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(Ly.nsplit, d.B * d.H_kv);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = TcShape<D>::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, kfn, mK, mV, (const bf16*)q, (bf16*)K, (bf16*)V, logn, len, (const bf16*)k_new,
      (const bf16*)v_new, (bf16*)out, d.T_cap, Ly.nsplit,
      reinterpret_cast<int32_t*>(ws + Ly.counters), reinterpret_cast<float*>(ws + Ly.part_ml),
      reinterpret_cast<float*>(ws + Ly.part_acc), reinterpret_cast<int32_t*>(ws));
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_decode_tc(const kvs_cache_desc& d, const void* q, void* K, void* V, float* logn,
                             int32_t* len, const void* k_new, const void* v_new, void* out,
                             const DecodeLayout& Ly, char* ws, cudaStream_t st) {
  const unsigned long long rows = (unsigned long long)d.B * d.H_kv * (unsigned long long)d.T_cap;
  CUtensorMap mK, mV;
  if (!encode_rows_map(&mK, K, rows, d.d, kTcTile) || !encode_rows_map(&mV, V, rows, d.d, kTcTile))
    return cudaErrorInvalidValue;
  const int G = d.H_q / d.H_kv;
#define KVS_TC(DD, GG) \
  if (d.d == DD && G == GG) return launch_tc<DD, GG>(d, mK, mV, q, K, V, logn, len, k_new, v_new, out, Ly, ws, st)
  KVS_TC(128, 1); KVS_TC(128, 2); KVS_TC(128, 4); KVS_TC(128, 8);
  KVS_TC(64, 1); KVS_TC(64, 2); KVS_TC(64, 4); KVS_TC(64, 8);
#undef KVS_TC
  return cudaErrorInvalidValue;
}

}  // namespace kvs
