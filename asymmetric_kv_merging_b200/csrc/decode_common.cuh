// Epilogue shared by the decode kernels: merge the CTA's per-warp softmax partials,
// publish the split's partial, and let the last CTA of a head combine all splits,
// attend and append the new row, and reset the head's arrival counter.
//
// Softmax partials are (m, l, acc) in the log2 domain: m the running maximum of
// s = log2(e) (q.k / sqrt(d) + logn), l = sum 2^(s - m), acc = sum 2^(s - m) v.
// A split's partial of query head g is one row of D + kPartPad floats,
// [acc | m | l | pad pad], and the splits of one query head are consecutive rows.
#pragma once

#include "kvs_common.cuh"
#include "ptx.cuh"

namespace kvs {

template <typename T>
__device__ __forceinline__ void store_out(T* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<bf16>(bf16* p, float v) { *p = __float2bfloat16_rn(v); }

// Shared-memory state of the epilogue, owned by the calling kernel.
template <int D, int G, int NW>
struct DecodeSmem {
  float (*sm)[G];                  // [NW][G] warp maxima
  float (*sl)[G];                  // [NW][G] warp sums
  float (*sacc)[G][D];             // [NW][G][D] warp accumulators
  float (*qs)[D];                  // [G][D] scaled queries (log2 domain)
  float* s_new;                    // [G] logit of the appended row
  float (*fac)[kMaxDecodeSplits];  // [G][64] split scale factors
  float (*gstat)[2];               // [G] combined (M, 1/L)
  int* s_last;
};

// Arguments of one decode call that the epilogue needs.
template <typename T>
struct DecodeArgs {
  int head, split, nsplit, L, T_cap;
  bool bad;
  T *K, *V;
  float* logn;
  int32_t* len;
  const T *k_new, *v_new;
  T* out;
  int32_t* counters;
  float* part;
  int32_t* flags;
};

// Write the CTA's partial row for every query head of the KV head, then count the
// arrival. Returns true in the last CTA of the head to arrive, for which every other
// split's row is visible after the return. `async_reuse`: the caller will overwrite
// the warp partials with bulk copies (async proxy) afterwards.
template <int D, int G, int NW, bool async_reuse>
__device__ __forceinline__ bool publish_split(const DecodeSmem<D, G, NW>& S, int tid, int nthreads,
                                              int head, int split, int nsplit, float* part,
                                              int32_t* counters) {
  constexpr int RS = D + kPartPad;
  float* ph = part + (size_t)head * G * nsplit * RS;
  for (int i = tid; i < G * D; i += nthreads) {
    const int g = i / D, c = i - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, S.sm[w][g]);
    float Ls = 0.f, A = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float f = exp2f(S.sm[w][g] - M);
        Ls = fmaf(S.sl[w][g], f, Ls);
        A = fmaf(S.sacc[w][g][c], f, A);
      }
    }
    float* row = ph + ((size_t)g * nsplit + split) * RS;
    row[c] = A;
    if (c == 0) {
      row[D] = M;
      row[D + 1] = Ls;
    }
  }
  if (async_reuse) fence_proxy_async_smem();
  // one device-scope release/acquire by one thread publishes the whole CTA's rows
  // (ordered before it by the barrier) and, in the last CTA, acquires all others'
  __syncthreads();
  if (tid == 0) *S.s_last = atom_add_acq_rel_gpu(&counters[head], 1) == nsplit - 1;
  __syncthreads();
  return *S.s_last != 0;
}

// Scale factors of the nsplit partials of one query head from their (m, l), with the
// appended row's logit sn (-inf when there is none). Executed by one whole warp.
__device__ __forceinline__ void split_factors(const float* m_of, const float* l_of, int stride,
                                              int nsplit, float sn, float* fac, float* gstat,
                                              int lane) {
  float mA = -INFINITY, lA = 0.f, mB = -INFINITY, lB = 0.f;
  if (lane < nsplit) {
    mA = m_of[lane * stride];
    lA = l_of[lane * stride];
  }
  if (lane + 32 < nsplit) {
    mB = m_of[(lane + 32) * stride];
    lB = l_of[(lane + 32) * stride];
  }
  float M = fmaxf(lA > 0.f ? mA : -INFINITY, lB > 0.f ? mB : -INFINITY);
  M = fmaxf(warp_max(M), sn);
  const bool live = M > -INFINITY;
  const float fA = (lA > 0.f && live) ? exp2f(mA - M) : 0.f;
  const float fB = (lB > 0.f && live) ? exp2f(mB - M) : 0.f;
  float Ls = warp_sum(lA * fA + lB * fB);
  if (sn > -INFINITY) Ls += exp2f(sn - M);
  if (lane < nsplit) fac[lane] = fA;
  if (lane + 32 < nsplit) fac[lane + 32] = fB;
  if (lane == 0) {
    gstat[0] = M;
    gstat[1] = Ls > 0.f ? 1.f / Ls : 0.f;
  }
}

// Logits of the appended row for the G query heads (count 1: no bias).
template <typename T, int D, int G, int NW>
__device__ __forceinline__ void appended_logits(const DecodeSmem<D, G, NW>& S, const T* kn,
                                                int warp, int lane, int nwarps) {
  for (int g = warp; g < G; g += nwarps) {
    float sp = 0.f;
    for (int c = lane; c < D; c += 32) sp = fmaf(S.qs[g][c], to_f32(kn[c]), sp);
    sp = warp_sum(sp);
    if (lane == 0) S.s_new[g] = sp;
  }
}

// Output columns c..c+3 of query head g from the scaled split rows (`rows` points at
// column c of split 0, `rs` floats between splits).
template <typename T, int D, bool kShared>
__device__ __forceinline__ void combine_columns(const float* rows, int rs, int nsplit,
                                                const float* fac, const float* gstat, float sn,
                                                const T* vn, int c, T* o) {
  float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 16
  for (int s = 0; s < nsplit; ++s) {
    const float f = fac[s];
    const float4 v = kShared ? *reinterpret_cast<const float4*>(rows + (size_t)s * rs)
                             : __ldcg(reinterpret_cast<const float4*>(rows + (size_t)s * rs));
    A.x = fmaf(v.x, f, A.x); A.y = fmaf(v.y, f, A.y);
    A.z = fmaf(v.z, f, A.z); A.w = fmaf(v.w, f, A.w);
  }
  if (vn) {
    const float f = exp2f(sn - gstat[0]);
    A.x = fmaf(to_f32(vn[c]), f, A.x); A.y = fmaf(to_f32(vn[c + 1]), f, A.y);
    A.z = fmaf(to_f32(vn[c + 2]), f, A.z); A.w = fmaf(to_f32(vn[c + 3]), f, A.w);
  }
  const float inv = gstat[1];
  store_out<T>(o, A.x * inv); store_out<T>(o + 1, A.y * inv);
  store_out<T>(o + 2, A.z * inv); store_out<T>(o + 3, A.w * inv);
}

// Append the new row (count 1), advance the length and re-arm the arrival counter.
template <typename T, int D>
__device__ __forceinline__ void finish_head(const DecodeArgs<T>& a, bool append, bool fits,
                                            int tid, int nthreads) {
  const int head = a.head, L = a.L;
  if (append) {
    if (fits) {
      const T* kn = a.k_new + (size_t)head * D;
      const T* vn = a.v_new + (size_t)head * D;
      for (int c = tid; c < D; c += nthreads) {
        a.K[((size_t)head * a.T_cap + L) * D + c] = kn[c];
        a.V[((size_t)head * a.T_cap + L) * D + c] = vn[c];
      }
      if (tid == 0 && a.logn) a.logn[(size_t)head * a.T_cap + L] = 0.f;
    } else if (tid == 0) {
      set_flag(a.flags, KVS_FLAG_OUT_CAPACITY);
    }
  }
  __syncthreads();
  if (tid == 0) {
    if (append && fits) a.len[head] = L + 1;
    a.counters[head] = 0;
  }
}

// Epilogue with a global-load combine: the last CTA stages every split's (m, l) in
// shared memory, turns them into scale factors one warp per query head, then reduces
// the accumulator rows four columns per thread with independent L2 loads. For
// kernels without a large free shared-memory buffer.
template <typename T, int D, int G, int NW>
__device__ __forceinline__ void decode_epilogue(const DecodeSmem<D, G, NW>& S, float* ml_stage,
                                                const DecodeArgs<T>& a, int tid, int nthreads) {
  constexpr int RS = D + kPartPad;
  const int lane = tid & 31, warp = tid >> 5, nwarps = nthreads / 32;
  if (!publish_split<D, G, NW, false>(S, tid, nthreads, a.head, a.split, a.nsplit, a.part,
                                      a.counters))
    return;
  const int nsplit = a.nsplit;
  const bool append = a.k_new != nullptr && a.v_new != nullptr && !a.bad;
  const bool fits = a.L < a.T_cap;
  const bool attend_new = append && fits;
  const float* ph = a.part + (size_t)a.head * G * nsplit * RS;
  // (m, l) of every split: ml_stage[2 * (g * nsplit + s) + {0, 1}]
  for (int i = tid; i < G * nsplit; i += nthreads) {
    const float2 ml = __ldcg(reinterpret_cast<const float2*>(ph + (size_t)i * RS + D));
    ml_stage[2 * i] = ml.x;
    ml_stage[2 * i + 1] = ml.y;
  }
  if (attend_new) appended_logits<T, D, G, NW>(S, a.k_new + (size_t)a.head * D, warp, lane, nwarps);
  __syncthreads();
  for (int g = warp; g < G; g += nwarps)
    split_factors(ml_stage + 2 * g * nsplit, ml_stage + 2 * g * nsplit + 1, 2, nsplit,
                  attend_new ? S.s_new[g] : -INFINITY, S.fac[g], S.gstat[g], lane);
  __syncthreads();
  const T* vn = attend_new ? a.v_new + (size_t)a.head * D : nullptr;
  for (int e = tid; e < G * (D / 4); e += nthreads) {
    const int g = e / (D / 4), c = (e - g * (D / 4)) * 4;
    combine_columns<T, D, false>(ph + (size_t)g * nsplit * RS + c, RS, nsplit, S.fac[g],
                                 S.gstat[g], attend_new ? S.s_new[g] : 0.f, vn, c,
                                 a.out + ((size_t)a.head * G + g) * D + c);
  }
  finish_head<T, D>(a, append, fits, tid, nthreads);
}

// Epilogue with a staged combine: the last CTA pulls the rows of as many query heads
// as fit in `stage` (a free shared-memory buffer of `stage_bytes`, 16-byte aligned)
// with one bulk copy, so the whole combine costs one L2 round trip per chunk instead
// of one per batch of loads. `cbar` is an initialised mbarrier (count 1) that has not
// been used before.
template <typename T, int D, int G, int NW>
__device__ __forceinline__ void decode_epilogue_staged(const DecodeSmem<D, G, NW>& S,
                                                       unsigned char* stage, uint32_t stage_bytes,
                                                       uint64_t* cbar, const DecodeArgs<T>& a,
                                                       int tid, int nthreads) {
  constexpr int RS = D + kPartPad;
  const int lane = tid & 31, warp = tid >> 5, nwarps = nthreads / 32;
  if (!publish_split<D, G, NW, true>(S, tid, nthreads, a.head, a.split, a.nsplit, a.part,
                                     a.counters))
    return;
  const int nsplit = a.nsplit;
  const bool append = a.k_new != nullptr && a.v_new != nullptr && !a.bad;
  const bool fits = a.L < a.T_cap;
  const bool attend_new = append && fits;
  const float* ph = a.part + (size_t)a.head * G * nsplit * RS;
  const uint32_t g_bytes = (uint32_t)nsplit * RS * sizeof(float);
  int gpc = (int)(stage_bytes / g_bytes);          // query heads per chunk (>= 1, host-checked)
  if (gpc > G) gpc = G;
  if (tid == 0) fence_proxy_async_global();        // rows acquired above, read by bulk copies
  const float* st = reinterpret_cast<const float*>(stage);
  uint32_t phase = 0;
  for (int g0 = 0; g0 < G; g0 += gpc) {
    const int ng = G - g0 < gpc ? G - g0 : gpc;
    if (g0 > 0) {
      fence_proxy_async_smem();                    // generic reads of the last chunk are done
      __syncthreads();
    }
    if (tid == 0) {
      const uint32_t bytes = (uint32_t)ng * g_bytes;
      mbar_arrive_expect_tx(cbar, bytes);
      const unsigned char* src = reinterpret_cast<const unsigned char*>(ph + (size_t)g0 * nsplit * RS);
      for (uint32_t off = 0; off < bytes; off += 32768u) {
        const uint32_t n = bytes - off < 32768u ? bytes - off : 32768u;
        bulk_load(stage + off, src + off, n, cbar);
      }
    }
    if (g0 == 0 && attend_new)                     // overlaps the copy
      appended_logits<T, D, G, NW>(S, a.k_new + (size_t)a.head * D, warp, lane, nwarps);
    if (!mbar_wait(cbar, phase)) {
      // the copy is still writing the buffer: record it and give it one more bound
      if (lane == 0) set_flag(a.flags, KVS_FLAG_TIMEOUT);
      mbar_wait(cbar, phase);
    }
    phase ^= 1u;
    __syncthreads();                               // s_new visible
    for (int gg = warp; gg < ng; gg += nwarps) {
      const int g = g0 + gg;
      const float* rows = st + (size_t)gg * nsplit * RS;
      split_factors(rows + D, rows + D + 1, RS, nsplit, attend_new ? S.s_new[g] : -INFINITY,
                    S.fac[g], S.gstat[g], lane);
    }
    __syncthreads();
    const T* vn = attend_new ? a.v_new + (size_t)a.head * D : nullptr;
    for (int e = tid; e < ng * (D / 4); e += nthreads) {
      const int gg = e / (D / 4), c = (e - gg * (D / 4)) * 4, g = g0 + gg;
      combine_columns<T, D, true>(st + (size_t)gg * nsplit * RS + c, RS, nsplit, S.fac[g],
                                  S.gstat[g], attend_new ? S.s_new[g] : 0.f, vn, c,
                                  a.out + ((size_t)a.head * G + g) * D + c);
    }
  }
  finish_head<T, D>(a, append, fits, tid, nthreads);
}

// Shared-memory inbox of a cluster combine: the partial columns and (m, l) that the C
// CTAs of a cluster push to the CTA owning an output slice. A dedicated region (not
// the ring), because peers may push while this CTA is still streaming.
template <int D, int G>
struct __align__(16) ClusterInbox {
  float acc[G * D + 4 * kMaxClusterSize];               // [C][G*D/(4C) + 1] 4-column units
  float ml[kMaxClusterSize][G][2];                      // [C][G] (m, l)
};

// Output slice of rank r among C CTAs: units [n*r/C, n*(r+1)/C) of n.
__device__ __forceinline__ int slice_lo(int n, int r, int C) { return (int)((unsigned)n * r / C); }
__device__ __forceinline__ int slice_owner(int n, int col, int C) {
  return (int)(((unsigned)(col + 1) * C - 1) / n);
}
// Bytes that land in the inbox of rank r: every CTA's units of r's slice, and every
// CTA's (m, l) per query head.
template <int G>
__device__ __forceinline__ uint32_t inbox_bytes(int n, int C, int r) {
  return (uint32_t)(C * (slice_lo(n, r + 1, C) - slice_lo(n, r, C)) * 16 + C * G * 8);
}
// Bytes the dry run pushes into its own scratch inbox: all n units and C copies of (m, l).
template <int G>
__device__ __forceinline__ uint32_t dry_inbox_bytes(int n, int C) {
  return (uint32_t)(n * 16 + C * G * 8);
}

// Cluster combine of a decode step in which the C CTAs of a cluster are all the splits
// of one KV head: no global partials, no arrival counter, no last CTA. Every CTA
// merges its warp partials, four output columns per thread, and pushes each 4-column
// unit to the CTA owning that unit's output slice, and its (m, l) to every CTA, with
// asynchronous distributed shared-memory stores that count their bytes on the
// receiver's inbox barrier. Each CTA combines its slice as soon as its own inbox
// barrier says every push into it has landed (no cluster-wide barrier on that path), and
// the CTA of rank 0 appends the new row. The cluster barrier's arrive follows the pushes
// and its wait ends the function, so no CTA leaves while a push into it may still be in
// flight. The loop over warps is unrolled, so that its shared-memory loads and
// exponentials overlap; the slice takes one lane per source CTA and unit.
//
// Protocol with the caller: every CTA initialises `inbar` (count 1) at kernel start and
// arrives on it once with expect_tx = inbox_bytes<G>(NU, C, rank), then every thread
// arrives (relaxed, after the barrier-init fence) on the cluster barrier; the combine
// begins with the matching wait.
// s_new: the appended row's logit per query head (read when append && L < T_cap);
// vn: its value row, staged in shared memory at kernel start (nullable when !append).
// `dry`: run the same instructions with every store aimed at this CTA's scratch
// (`inbox`, `inbar` and `out` point there, head is 0) and without the barriers, the
// inbox wait or the append, from a single warp while the other warps stream (its loads
// of the warp partials see stage data in flight; the values are discarded). A kernel
// launch starts with cold instruction caches; the dry run pulls this code in before the
// real combine needs it. The scratch barrier expects dry_inbox_bytes<G>(NU, C).
template <typename T, int D, int G, int NW>
__device__ __noinline__ void cluster_combine(
    float (*sm)[G], float (*sl)[G], float (*sacc)[G][D], const float* s_new,
    ClusterInbox<D, G>* inbox, uint64_t* inbar, int C, int rank, int tid, int nthreads, bool dry,
    int head, int L, int T_cap, bool append, T* K, T* V, float* logn, int32_t* len, const T* kn,
    const T* vn, T* out, int32_t* flags) {
  constexpr int NU = G * D / 4;                        // 4-column output units
  const bool fits = L < T_cap;
  const bool attend_new = append && fits;
  const int slice_w = NU / C + 1;                      // inbox row stride in units (>= any slice)
  const uint32_t in_acc = smem_u32(inbox->acc), in_ml = smem_u32(&inbox->ml[0][0][0]);
  const uint32_t in_bar = smem_u32(inbar);
  if (!dry) cluster_wait();                            // every CTA's inbox barrier is set up
  // merge the warps unit by unit and push each unit to its owner
  for (int u = tid; u < NU; u += nthreads) {
    const int g = (u * 4) / D, c = u * 4 - g * D;
    float mw[NW];
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      mw[w] = sm[w][g];
      M = fmaxf(M, mw[w]);
    }
    float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M > -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float f = exp2f(mw[w] - M);
        const float4 v = *reinterpret_cast<const float4*>(&sacc[w][g][c]);
        A.x = fmaf(v.x, f, A.x); A.y = fmaf(v.y, f, A.y);
        A.z = fmaf(v.z, f, A.z); A.w = fmaf(v.w, f, A.w);
      }
    }
    const int owner = slice_owner(NU, u, C);
    const int at = rank * slice_w + (u - slice_lo(NU, owner, C));
    const uint32_t dst = dry ? rank : owner;
    st_async_f32x4(cluster_map(in_acc + (uint32_t)at * 16u, dst), A, cluster_map(in_bar, dst));
  }
  // push (m, l) of every query head to every CTA: ml[rank][g] in CTA j (the threads past
  // the unit loop's last take these first)
  const int k0 = (tid + nthreads - NU % nthreads) % nthreads;
  for (int k = k0; k < C * G; k += nthreads) {
    const int j = k / G, g = k - j * G;
    float mw[NW];
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      mw[w] = sm[w][g];
      M = fmaxf(M, mw[w]);
    }
    float Ls = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) Ls = fmaf(sl[w][g], exp2f(mw[w] - M), Ls);
    }
    const uint32_t dst = dry ? rank : j;
    st_async_f32x2(cluster_map(in_ml + (uint32_t)((rank * G + g) * 2) * 4u, dst), M, Ls,
                   cluster_map(in_bar, dst));
  }
  if (!dry) cluster_arrive();                          // this CTA's pushes; the wait is at the end
  // combine this CTA's slice from its inbox, once every push into it has landed: 16
  // lanes per unit, lane j of a half-warp taking source CTA j (C <= 16), max and sums
  // by shuffles within the half-warp; whole warps take part, so that the shuffles are
  // warp-uniform
  const int lo = slice_lo(NU, rank, C), hi = slice_lo(NU, rank + 1, C);
  const int nunits = hi - lo, warp = tid >> 5, nwarps = nthreads >> 5;
  // (thread 0 waits whatever its share, so the CTA outlives every push into it)
  if (!dry && (tid == 0 || 2 * warp < nunits) && !mbar_wait(inbar, 0))
    set_flag(flags, KVS_FLAG_TIMEOUT);
  const int j = tid & 15;
  for (int b0 = 2 * warp; b0 < nunits; b0 += 2 * nwarps) {
    const int b = b0 + ((tid >> 4) & 1);
    const bool act = b < nunits;
    const int u = lo + (act ? b : 0);
    const int g = (u * 4) / D, c = u * 4 - g * D;
    float m = -INFINITY, l = 0.f;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (act && j < C) {
      const float2 ml = *reinterpret_cast<const float2*>(&inbox->ml[j][g][0]);
      v = *reinterpret_cast<const float4*>(&inbox->acc[(j * slice_w + b) * 4]);
      if (ml.y > 0.f) {
        m = ml.x;
        l = ml.y;
      }
    }
    const float sn = attend_new ? s_new[g] : -INFINITY;
    float M = fmaxf(m, sn);
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float f = (l > 0.f && M > -INFINITY) ? exp2f(m - M) : 0.f;
    float Ls = l * f;
    float4 A = make_float4(v.x * f, v.y * f, v.z * f, v.w * f);
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) {
      Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
      A.x += __shfl_xor_sync(0xffffffffu, A.x, off);
      A.y += __shfl_xor_sync(0xffffffffu, A.y, off);
      A.z += __shfl_xor_sync(0xffffffffu, A.z, off);
      A.w += __shfl_xor_sync(0xffffffffu, A.w, off);
    }
    if (act && j == 0) {
      if (attend_new && M > -INFINITY) {
        const float fn = exp2f(sn - M);
        Ls += fn;
        A.x = fmaf(to_f32(vn[c]), fn, A.x);
        A.y = fmaf(to_f32(vn[c + 1]), fn, A.y);
        A.z = fmaf(to_f32(vn[c + 2]), fn, A.z);
        A.w = fmaf(to_f32(vn[c + 3]), fn, A.w);
      }
      T* o = out + ((size_t)head * G + g) * D + c;
      store_out<T>(o, Ls > 0.f ? A.x / Ls : 0.f);
      store_out<T>(o + 1, Ls > 0.f ? A.y / Ls : 0.f);
      store_out<T>(o + 2, Ls > 0.f ? A.z / Ls : 0.f);
      store_out<T>(o + 3, Ls > 0.f ? A.w / Ls : 0.f);
    }
  }
  if (!dry && rank == 0 && append) {
    if (fits) {
      for (int c = tid; c < D; c += nthreads) {
        K[((size_t)head * T_cap + L) * D + c] = kn[c];
        V[((size_t)head * T_cap + L) * D + c] = vn[c];
      }
      if (tid == 0 && logn) logn[(size_t)head * T_cap + L] = 0.f;
      if (tid == 0) len[head] = L + 1;
    } else if (tid == 0) {
      set_flag(flags, KVS_FLAG_OUT_CAPACITY);
    }
  }
  if (!dry) cluster_wait();                            // every push of the cluster has landed
}

}  // namespace kvs
