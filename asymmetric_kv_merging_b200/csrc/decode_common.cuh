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
  float acc[G * D + kMaxClusterSize];                   // [C][G*D/C + 1]
  float ml[kMaxClusterSize][G][2];                      // [C][G] (m, l)
};

// Output slice of rank r among C CTAs: columns [G*D*r/C, G*D*(r+1)/C).
__device__ __forceinline__ int slice_lo(int n, int r, int C) { return (int)((unsigned)n * r / C); }
__device__ __forceinline__ int slice_owner(int n, int col, int C) {
  return (int)(((unsigned)(col + 1) * C - 1) / n);
}

// Cluster combine of a decode step in which the C CTAs of a cluster are all the splits
// of one KV head: no global partials, no arrival counter, no last CTA. Every CTA
// merges its warp partials and pushes each column to the CTA owning that column's
// output slice (distributed shared-memory stores into the owner's inbox), and its
// (m, l) to every CTA; after one cluster barrier each CTA combines its slice from its
// own inbox, and the CTA of rank 0 appends the new row. Nothing is read remotely, so
// a CTA may leave as soon as its slice is written.
//
// kn, vn: the appended row of this head (nullable when !append); the caller stages it
// in shared memory at kernel start, so the combine waits on no global load.
// `dry`: run the same instructions with every store aimed at this CTA's scratch
// (`inbox` and `out` point there, head is 0) and without barriers or the append,
// from a single warp while the other warps stream (its loads of the warp partials see
// stage data in flight; the values are discarded). A kernel launch starts with cold
// instruction caches; the dry run pulls this code in before the real combine needs it.
template <typename T, int D, int G, int NW>
__device__ __noinline__ void cluster_combine(
    float (*sm)[G], float (*sl)[G], float (*sacc)[G][D], float (*qs)[D], float* s_cml,
    float* s_new, ClusterInbox<D, G>* inbox, int C, int rank, int tid, int nthreads, bool dry,
    int head, int L, int T_cap, bool append, T* K, T* V, float* logn, int32_t* len,
    const T* kn, const T* vn, T* out, int32_t* flags) {
  constexpr int N = G * D;
  const int lane = tid & 31, warp = tid >> 5, nwarps = nthreads / 32;
  const bool fits = L < T_cap;
  const bool attend_new = append && fits;
  const int slice_w = N / C + 1;                       // inbox row stride (>= any slice)
  // this CTA's (m, l) per query head
  for (int g = tid; g < G; g += nthreads) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sm[w][g]);
    float Ls = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) Ls = fmaf(sl[w][g], exp2f(sm[w][g] - M), Ls);
    }
    s_cml[2 * g] = M;
    s_cml[2 * g + 1] = Ls;
  }
  if (attend_new) appended_logits<T, D, G, NW>(DecodeSmem<D, G, NW>{sm, sl, sacc, qs, s_new, nullptr, nullptr, nullptr},
                                               kn, warp, lane, nwarps);
  if (!dry) __syncthreads();
  const uint32_t in_acc = smem_u32(inbox->acc), in_ml = smem_u32(&inbox->ml[0][0][0]);
  // push (m, l) of every query head to every CTA: ml[rank][g] in CTA j
  for (int k = tid; k < C * G; k += nthreads) {
    const int j = k / G, g = k - j * G;
    const uint32_t dst = cluster_map(in_ml + (uint32_t)((rank * G + g) * 2) * 4u, dry ? rank : j);
    st_cluster_f32x2(dst, s_cml[2 * g], s_cml[2 * g + 1]);
  }
  // merge the warps column by column and push each column to its owner
  for (int i = tid; i < N; i += nthreads) {
    const int g = i / D, c = i - g * D;
    const float M = s_cml[2 * g];
    float A = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) A = fmaf(sacc[w][g][c], exp2f(sm[w][g] - M), A);
    }
    const int owner = slice_owner(N, i, C);
    const int at = rank * slice_w + (i - slice_lo(N, owner, C));
    st_cluster_f32(cluster_map(in_acc + (uint32_t)at * 4u, dry ? rank : owner), A);
  }
  if (!dry) {
    cluster_arrive();
    cluster_wait();                                    // every push to this CTA landed
  }
  // combine this CTA's slice from its inbox
  const int lo = slice_lo(N, rank, C), hi = slice_lo(N, rank + 1, C);
  for (int col = lo + tid; col < hi; col += nthreads) {
    const int g = col / D, c = col - g * D;
    const float sn = attend_new ? s_new[g] : -INFINITY;
    float M = sn;
    for (int j = 0; j < C; ++j)
      if (inbox->ml[j][g][1] > 0.f) M = fmaxf(M, inbox->ml[j][g][0]);
    float Ls = 0.f, A = 0.f;
    if (M > -INFINITY) {
      for (int j = 0; j < C; ++j) {
        const float lj = inbox->ml[j][g][1];
        const float f = lj > 0.f ? exp2f(inbox->ml[j][g][0] - M) : 0.f;
        Ls = fmaf(lj, f, Ls);
        A = fmaf(inbox->acc[j * slice_w + (col - lo)], f, A);
      }
      if (attend_new) {
        const float f = exp2f(sn - M);
        Ls += f;
        A = fmaf(to_f32(vn[c]), f, A);
      }
    }
    store_out<T>(out + ((size_t)head * G + g) * D + c, Ls > 0.f ? A / Ls : 0.f);
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
}

}  // namespace kvs
