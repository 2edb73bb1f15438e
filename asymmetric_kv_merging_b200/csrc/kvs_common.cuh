// Shared device helpers for the KVSlimmer kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvs.h"

namespace kvs {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kTargetCtas = 296;         // 2 resident CTAs on each of the 148 SMs
constexpr size_t kWsAlign = 256;
constexpr int kMergePairsPerBlock = 128;  // pairs handled by one merge CTA
constexpr int kInplaceMaxSpan = 8192;     // rows an in-place merge may rewrite per head

typedef __nv_bfloat16 bf16;

// Host-side count of kernel launches (see kvs_launch_count).
void count_launches(int n);

// Launch with programmatic stream serialisation: the grid may be scheduled while the
// previous kernel of the stream is still running, so the kernel must execute
// griddepcontrol.wait (griddep_wait) before its first access to memory that earlier work
// writes -- the kernels launched this way do so first thing -- and it triggers its own
// dependents right after. Returns the launch's error.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kfn)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kfn, static_cast<Args&&>(args)...);
}

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Elements of T that fit one 16-byte vector.
template <typename T> struct Vec16;
template <> struct Vec16<float> { static constexpr int n = 4; };
template <> struct Vec16<bf16> { static constexpr int n = 8; };

// bf16 -> fp32 is a 16-bit left shift of the bit pattern (exact).
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Load 16 bytes (Vec16<T>::n elements) and widen to fp32.
__device__ __forceinline__ void load_vec(const float* p, float* f) {
  float4 v = *reinterpret_cast<const float4*>(p);
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
__device__ __forceinline__ void load_vec(const bf16* p, float* f) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z); f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}
// Same, streaming through L2 only (data read once).
__device__ __forceinline__ void load_vec_cs(const float* p, float* f) {
  float4 v = __ldcs(reinterpret_cast<const float4*>(p));
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
__device__ __forceinline__ void load_vec_cs(const bf16* p, float* f) {
  uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z); f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

// Narrow fp32 -> T (round to nearest even) and store 16 bytes.
__device__ __forceinline__ void store_vec(float* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void store_vec(bf16* p, const float* f) {
  uint4 u;
  u.x = pack_bf16x2(f[0], f[1]); u.y = pack_bf16x2(f[2], f[3]);
  u.z = pack_bf16x2(f[4], f[5]); u.w = pack_bf16x2(f[6], f[7]);
  *reinterpret_cast<uint4*>(p) = u;
}

// Raw 16-byte copy.
__device__ __forceinline__ uint4 load_raw(const void* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void store_raw(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Order-preserving map of a pair score to an unsigned key: NaN ranks as +inf,
// -0 as +0, then the usual sign-magnitude flip so unsigned order = float order.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7fffffffu) > 0x7f800000u) u = 0x7f800000u;   // NaN -> +inf
  if ((u & 0x7fffffffu) == 0u) u = 0u;                     // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void set_flag(int32_t* flags, int32_t bit) { atomicOr(flags, bit); }

// ---------------------------------------------------------------------------
// Workspace layouts (host and device agree through these structs).
// ---------------------------------------------------------------------------

struct SelUnit {       // one selection unit (a head, or a sequence in pooled scope)
  uint32_t thr_key;    // pairs with key < thr_key are merged
  int32_t need_eq;     // ... plus the first need_eq pairs (unit order) with key == thr_key
  int32_t R;           // pairs merged in the unit
  int32_t P;           // candidate pairs in the unit
};

struct HeadInfo {      // one (b, h)
  int32_t len_in;      // length before the round (-1: head skipped)
  int32_t P;           // candidate pairs
  int32_t R;           // pairs merged in this head
  int32_t c0;          // candidate span start
  int32_t lt0, eq0;    // unit-wide exclusive scans at this head's first block
  int32_t pad0, pad1;
};

struct ScoreLayout {
  size_t part_ml, part_o, stats, obar, alpha, oq, oq_hi, oq_mid, oq_lo, on2, owq, total;
  int nsplit, Qn;
  int part_slots;   // window partials per head the layout holds (>= nsplit, >= 2)
};
struct MergeLayout {
  size_t sel, head, blk, total;
  int nblk;
};
// Decode split partials: one row of kPartPad + d floats per (query head, split),
// query-head major, so that every split of a query head is one contiguous block:
// [acc[0..d) | m | l | pad | pad]. Rows are 16-byte multiples (d in {64, 128}).
constexpr int kPartPad = 4;
struct DecodeLayout {
  size_t counters, part, total;
  int nsplit;
};

inline int window_splits(const kvs_cache_desc& d) {
  int units = d.B * d.H_kv;
  int s = (kTargetCtas + units - 1) / units;
  int cap = d.T_cap / 256 > 1 ? d.T_cap / 256 : 1;
  if (s > cap) s = cap;
  if (s > 64) s = 64;
  return s < 1 ? 1 : s;
}

constexpr int kMaxDecodeSplits = 64;      // the combine gives each lane two splits
constexpr int kMaxClusterSize = 16;       // CTAs of one KV head in a cluster launch

inline int decode_splits(const kvs_cache_desc& d) {
  // as many splits as keep the grid to one wave of two CTAs per SM
  int units = d.B * d.H_kv;
  int s = kTargetCtas / units;
  int cap = d.T_cap / 128 > 1 ? d.T_cap / 128 : 1;
  if (s > cap) s = cap;
  if (s > kMaxDecodeSplits) s = kMaxDecodeSplits;
  return s < 1 ? 1 : s;
}

// Every layout starts with the same persistent region: the device flag word in the
// first 256 bytes, then one arrival counter per KV head for the decode combine. No
// op writes this region except through its own flags / counters, so one zeroed
// workspace can be shared by all ops on a stream.
inline size_t persistent_bytes(const kvs_cache_desc& d) {
  return kWsAlign + align_up((size_t)d.B * d.H_kv * sizeof(int32_t), kWsAlign);
}

inline ScoreLayout score_layout(const kvs_cache_desc& d, int W) {
  ScoreLayout L;
  size_t units = (size_t)d.B * d.H_kv;
  L.Qn = (d.H_q / d.H_kv) * W;
  L.nsplit = window_splits(d);
  L.part_slots = L.nsplit > 2 ? L.nsplit : 2;
  L.part_ml = persistent_bytes(d);
  L.part_o = align_up(L.part_ml + units * L.part_slots * L.Qn * 2 * sizeof(float), kWsAlign);
  L.stats = align_up(L.part_o + units * L.part_slots * L.Qn * (size_t)d.d * sizeof(float), kWsAlign);
  L.obar = align_up(L.stats + units * L.Qn * 2 * sizeof(float), kWsAlign);
  L.alpha = align_up(L.obar + units * (size_t)d.d * sizeof(float), kWsAlign);
  // window outputs of the bf16 path: o_q (fp32, rows of 128 padded queries per head),
  // and relative to their mean, e_q = o_q - o_bar, as bf16 hi / mid / lo parts with
  // |e_q|^2 and o_bar . e_q in shares per block of 32 columns
  L.oq = align_up(L.alpha + units * (size_t)d.T_cap * sizeof(float), kWsAlign);
  L.oq_hi = align_up(L.oq + units * 128 * (size_t)d.d * sizeof(float), kWsAlign);
  L.oq_mid = align_up(L.oq_hi + units * 128 * (size_t)d.d * 2, kWsAlign);
  L.oq_lo = align_up(L.oq_mid + units * 128 * (size_t)d.d * 2, kWsAlign);
  L.on2 = align_up(L.oq_lo + units * 128 * (size_t)d.d * 2, kWsAlign);
  L.owq = align_up(L.on2 + units * 128 * (size_t)(d.d / 32) * sizeof(float), kWsAlign);
  L.total = align_up(L.owq + units * 128 * (size_t)(d.d / 32) * sizeof(float), kWsAlign);
  return L;
}

inline MergeLayout merge_layout(const kvs_cache_desc& d) {
  MergeLayout L;
  size_t heads = (size_t)d.B * d.H_kv;
  L.nblk = (d.T_cap / 2 + kMergePairsPerBlock - 1) / kMergePairsPerBlock;
  if (L.nblk < 1) L.nblk = 1;
  L.sel = persistent_bytes(d);
  L.head = align_up(L.sel + heads * sizeof(SelUnit), kWsAlign);
  L.blk = align_up(L.head + heads * sizeof(HeadInfo), kWsAlign);
  L.total = align_up(L.blk + heads * L.nblk * sizeof(int2), kWsAlign);
  return L;
}

inline DecodeLayout decode_layout(const kvs_cache_desc& d) {
  DecodeLayout L;
  size_t qheads = (size_t)d.B * d.H_q;
  L.nsplit = decode_splits(d);
  L.counters = kWsAlign;
  L.part = persistent_bytes(d);
  L.total = align_up(L.part + qheads * L.nsplit * (size_t)(d.d + kPartPad) * sizeof(float),
                     kWsAlign);
  return L;
}

// Chunked prefill: the score and merge scratch share one region (the score scratch is
// dead once the pairs are scored), followed by the round's pair scores and weights and
// the per-head candidate starts and targets.
struct PrefillLayout {
  ScoreLayout score;
  MergeLayout merge;
  size_t score_arr, w_b_arr, cand, target, total;
};

inline PrefillLayout prefill_layout(const kvs_cache_desc& d, int W) {
  PrefillLayout L;
  L.score = score_layout(d, W);
  L.merge = merge_layout(d);
  const size_t heads = (size_t)d.B * d.H_kv;
  const size_t pairs = heads * (size_t)(d.T_cap / 2);
  const size_t scratch_end = L.score.total > L.merge.total ? L.score.total : L.merge.total;
  L.score_arr = align_up(scratch_end, kWsAlign);
  L.w_b_arr = align_up(L.score_arr + pairs * sizeof(float), kWsAlign);
  L.cand = align_up(L.w_b_arr + pairs * sizeof(float), kWsAlign);
  L.target = align_up(L.cand + heads * sizeof(int32_t), kWsAlign);
  L.total = align_up(L.target + heads * sizeof(int32_t), kWsAlign);
  return L;
}

}  // namespace kvs
