// Internal launchers shared between the kernel files and the C-ABI layer.
#pragma once

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "kvs.h"
#include "kvs_common.cuh"

namespace kvs {

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the current
// device (cudaFuncSetAttribute applies per device). The value set is cached per
// (device, kernel) under a mutex, so later calls make no CUDA call; the first call for
// a device must come before any stream capture.
bool ensure_smem_attr(const void* fn, size_t bytes);
// Allow cluster sizes above 8 for a kernel on the current device (cached the same way).
bool ensure_nonportable_cluster(const void* fn);

// Window statistics: (m, l) per window query, o_bar and alpha_bar into the score workspace.
cudaError_t launch_window_stats(const kvs_cache_desc& d, const void* K, const void* V,
                                const float* logn, const int32_t* len, const void* Qw, int W,
                                const ScoreLayout& Ly, char* ws, cudaStream_t st);

// Pair norms, merge weight and score from alpha_bar / o_bar.
cudaError_t launch_pair_score(const kvs_cache_desc& d, const void* K, const void* V,
                              const int32_t* len, const int32_t* cand_begin, int n_recent,
                              int form, const ScoreLayout& Ly, char* ws, float* score,
                              float* w_b, cudaStream_t st);

// Selection to the budget, then merge + compaction (out-of-place or in-place).
cudaError_t launch_select(const kvs_cache_desc& d, const float* score, const int32_t* len,
                          const int32_t* cand_begin, int n_recent, const int32_t* target,
                          int scope, const MergeLayout& Ly, char* ws, cudaStream_t st);

cudaError_t launch_merge(const kvs_cache_desc& d, const void* K, const void* V, const float* logn,
                         const float* score, const float* w_b, int scope, int T_cap_out,
                         bool inplace, void* K_out, void* V_out, float* logn_out,
                         int32_t* len_out, uint8_t* dbg_sel, int32_t* dbg_off, float* dbg_km,
                         const MergeLayout& Ly, char* ws, cudaStream_t st);

// Chunked prefill: append n rows of a chunk ([B, H_kv, n, d]) at row L of every head
// whose length is L (others: KVS_FLAG_BAD_LENGTH), then len = L + n; fill two int32
// arrays with constants.
cudaError_t launch_append_rows(const kvs_cache_desc& d, void* K, void* V, float* logn,
                               int32_t* len, int L, const void* k_rows, const void* v_rows, int n,
                               char* ws, cudaStream_t st);
cudaError_t launch_fill2(int32_t* a, int32_t va, int32_t* b, int32_t vb, int n, cudaStream_t st);

// Split-K GQA decode with fused split combine and optional append.
cudaError_t launch_decode(const kvs_cache_desc& d, const void* q, void* K, void* V, float* logn,
                          int32_t* len, const void* k_new, const void* v_new, void* out,
                          const DecodeLayout& Ly, char* ws, cudaStream_t st);

// Driver entry point for tensor maps, and a 2D map over a [rows, d] bf16 array with
// boxes of 64 elements x box_rows rows and 128-byte swizzling (rows past the end read 0).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
bool encode_rows_map(CUtensorMap* map, const void* base, unsigned long long rows, int d,
                     int box_rows);

// Window statistics and pair scores for bf16 caches in two fused tensor-core passes
// (G*W <= 128): form is KVS_FORM_FULL or KVS_FORM_DIAGONAL; stats_form is 0 (window
// mean) or KVS_FORM_PER_QUERY.
bool window_fused_supported(const kvs_cache_desc& d, int W);
cudaError_t launch_score_fused(const kvs_cache_desc& d, const void* K, const void* V,
                               const float* logn, const int32_t* len, const int32_t* cand_begin,
                               int n_recent, const void* Qw, int W, int form, int stats_form,
                               const ScoreLayout& Ly, char* ws, float* score, float* w_b,
                               cudaStream_t st);

// The same step for bf16 caches on the TMA + tensor-core kernel.
bool decode_tc_supported(const kvs_cache_desc& d);
cudaError_t launch_decode_tc(const kvs_cache_desc& d, const void* q, void* K, void* V, float* logn,
                             int32_t* len, const void* k_new, const void* v_new, void* out,
                             const DecodeLayout& Ly, char* ws, cudaStream_t st);

// Measurement helper: stream `rows` rows of a [rows, d] bf16 array through shared
// memory with the decode kernel's TMA pattern on `ctas` CTAs, computing nothing.
cudaError_t launch_stream_probe(const void* buf, long long rows, int d, int ctas, char* ws,
                                cudaStream_t st);

}  // namespace kvs
