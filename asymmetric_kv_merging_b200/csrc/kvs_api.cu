// C ABI of libkvs.so: host-side validation, workspace layout and kernel launches.
// The operations and their citations are documented in include/kvs.h.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "kvs.h"
#include "kvs_common.cuh"
#include "kvs_kernels.h"

using namespace kvs;

namespace kvs {
static std::atomic<long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

namespace {
std::mutex g_attr_mutex;
// (device, kernel) -> the dynamic shared-memory limit set so far / the non-portable
// cluster attribute set
std::map<std::pair<int, const void*>, size_t> g_smem_attr;
std::map<std::pair<int, const void*>, bool> g_cluster_attr;
}  // namespace

bool ensure_smem_attr(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return true;   // the default limit
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(g_attr_mutex);
  size_t& done = g_smem_attr[std::make_pair(dev, fn)];
  if (bytes <= done) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
      cudaSuccess)
    return false;
  done = bytes;
  return true;
}

bool ensure_nonportable_cluster(const void* fn) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(g_attr_mutex);
  bool& done = g_cluster_attr[std::make_pair(dev, fn)];
  if (done) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
    return false;
  done = true;
  return true;
}
}  // namespace kvs

namespace {

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

kvs_status check_desc(const kvs_cache_desc* d) {
  if (!d) return KVS_ERR_INVALID_ARG;
  if (d->B <= 0 || d->H_kv <= 0 || d->H_q <= 0 || d->T_cap <= 0 || d->d <= 0)
    return KVS_ERR_INVALID_ARG;
  if (d->T_cap % 2 != 0 || d->H_q % d->H_kv != 0) return KVS_ERR_INVALID_ARG;
  const int G = d->H_q / d->H_kv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return KVS_ERR_UNSUPPORTED;
  if (d->d != 64 && d->d != 128) return KVS_ERR_UNSUPPORTED;
  if (d->dtype != KVS_F32 && d->dtype != KVS_BF16) return KVS_ERR_UNSUPPORTED;
  const unsigned long long rows = (unsigned long long)d->B * d->H_kv * (unsigned long long)d->T_cap;
  if (rows > (1ull << 40)) return KVS_ERR_INVALID_ARG;
  return KVS_OK;
}

size_t elem_bytes(const kvs_cache_desc* d) { return d->dtype == KVS_BF16 ? 2 : 4; }

size_t cache_bytes(const kvs_cache_desc* d, int T_cap) {
  return (size_t)d->B * d->H_kv * (size_t)T_cap * d->d * elem_bytes(d);
}

struct Range {
  const char* p;
  size_t n;
};
inline bool overlap(Range a, Range b) {
  if (!a.p || !b.p || a.n == 0 || b.n == 0) return false;
  return a.p < b.p + b.n && b.p < a.p + a.n;
}

// One scoring pass: the two fused tensor-core passes for bf16 caches, else the CUDA-core
// window statistics followed by the pair-scoring kernel.
cudaError_t score_pass(const kvs_cache_desc& d, const void* K, const void* V, const float* logn,
                       const int32_t* len, const int32_t* cand_begin, int n_recent,
                       const void* Q_win, int W, int form, const ScoreLayout& Ly, char* ws,
                       float* score, float* w_b, cudaStream_t st) {
  if (window_fused_supported(d, W))
    return launch_score_fused(d, K, V, logn, len, cand_begin, n_recent, Q_win, W,
                              form & KVS_FORM_DIAGONAL, form & KVS_FORM_PER_QUERY, Ly, ws, score,
                              w_b, st);
  cudaError_t e = launch_window_stats(d, K, V, logn, len, Q_win, W, Ly, ws, st);
  if (e != cudaSuccess) return e;
  return launch_pair_score(d, K, V, len, cand_begin, n_recent, form & KVS_FORM_DIAGONAL, Ly, ws,
                           score, w_b, st);
}

kvs_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws || !aligned(ws, kWsAlign)) return KVS_ERR_WORKSPACE;
  if (ws_bytes < need) return KVS_ERR_WORKSPACE;
  return KVS_OK;
}

kvs_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KVS_OK : KVS_ERR_CUDA; }

}  // namespace

extern "C" {

int32_t kvs_version(void) { return 1; }

int64_t kvs_launch_count(void) { return (int64_t)g_launches.load(std::memory_order_relaxed); }

const char* kvs_status_str(kvs_status s) {
  switch (s) {
    case KVS_OK: return "ok";
    case KVS_ERR_INVALID_ARG: return "invalid argument";
    case KVS_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case KVS_ERR_BUDGET: return "budget unreachable";
    case KVS_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case KVS_ERR_ALIAS: return "output overlaps an input";
    case KVS_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

size_t kvs_workspace_size(const kvs_cache_desc* desc, int32_t W, int32_t op) {
  if (check_desc(desc) != KVS_OK) return 0;
  switch (op) {
    case KVS_OP_SCORE:
      if (W < 1) return 0;
      return score_layout(*desc, W).total;
    case KVS_OP_MERGE:
      return merge_layout(*desc).total;
    case KVS_OP_DECODE:
      return decode_layout(*desc).total;
    case KVS_OP_PREFILL:
      if (W < 1) return 0;
      return prefill_layout(*desc, W).total;
    default:
      return 0;
  }
}

kvs_status kvs_score_pairs(const kvs_cache_desc* desc, const void* K, const void* V,
                           const float* logn, const int32_t* len, const int32_t* cand_begin,
                           int32_t n_recent, const void* Q_win, int32_t W, float* score,
                           float* w_b, void* ws, size_t ws_bytes, kvs_stream_t stream) {
  return kvs_score_pairs_form(desc, K, V, logn, len, cand_begin, n_recent, Q_win, W, score, w_b,
                              KVS_FORM_FULL, ws, ws_bytes, stream);
}

kvs_status kvs_score_pairs_form(const kvs_cache_desc* desc, const void* K, const void* V,
                                const float* logn, const int32_t* len, const int32_t* cand_begin,
                                int32_t n_recent, const void* Q_win, int32_t W, float* score,
                                float* w_b, int32_t form, void* ws, size_t ws_bytes,
                                kvs_stream_t stream) {
  if (form < 0 || form > (KVS_FORM_DIAGONAL | KVS_FORM_PER_QUERY)) return KVS_ERR_INVALID_ARG;
  kvs_status s = check_desc(desc);
  if (s != KVS_OK) return s;
  if (!K || !V || !len || !cand_begin || !Q_win || !score || !w_b) return KVS_ERR_INVALID_ARG;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(Q_win, 16) || !aligned(len, 4) ||
      !aligned(cand_begin, 4) || !aligned(score, 4) || !aligned(w_b, 4) ||
      (logn && !aligned(logn, 4)))
    return KVS_ERR_INVALID_ARG;
  if (W < 1 || n_recent < 0) return KVS_ERR_INVALID_ARG;
  const int G = desc->H_q / desc->H_kv;
  if (G * W > 128) return KVS_ERR_UNSUPPORTED;
  const size_t pairs_bytes = (size_t)desc->B * desc->H_kv * (desc->T_cap / 2) * sizeof(float);
  Range rs{(const char*)score, pairs_bytes}, rw{(const char*)w_b, pairs_bytes};
  Range rk{(const char*)K, cache_bytes(desc, desc->T_cap)}, rv{(const char*)V, cache_bytes(desc, desc->T_cap)};
  if (overlap(rs, rw) || overlap(rs, rk) || overlap(rs, rv) || overlap(rw, rk) || overlap(rw, rv))
    return KVS_ERR_ALIAS;
  const ScoreLayout Ly = score_layout(*desc, W);
  s = check_ws(ws, ws_bytes, Ly.total);
  if (s != KVS_OK) return s;
  const bool fused = window_fused_supported(*desc, W);
  if ((form & KVS_FORM_PER_QUERY) && !fused) return KVS_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  return from_cuda(score_pass(*desc, K, V, logn, len, cand_begin, n_recent, Q_win, W, form, Ly,
                              w, score, w_b, st));
}

kvs_status kvs_merge_compact(const kvs_cache_desc* desc, const void* K, const void* V,
                             const float* logn, const int32_t* len, const int32_t* cand_begin,
                             int32_t n_recent, const float* score, const float* w_b,
                             const int32_t* target, int32_t scope, int32_t T_cap_out,
                             void* K_out, void* V_out, float* logn_out, int32_t* len_out,
                             uint8_t* dbg_selected, int32_t* dbg_out_offset,
                             float* dbg_kmerged_f32, void* ws, size_t ws_bytes,
                             kvs_stream_t stream) {
  kvs_status s = check_desc(desc);
  if (s != KVS_OK) return s;
  if (!K || !V || !len || !cand_begin || !score || !w_b || !target || !K_out || !V_out ||
      !logn_out || !len_out)
    return KVS_ERR_INVALID_ARG;
  if (scope != KVS_SCOPE_HEAD && scope != KVS_SCOPE_POOLED) return KVS_ERR_INVALID_ARG;
  if (n_recent < 0 || T_cap_out <= 0) return KVS_ERR_INVALID_ARG;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(K_out, 16) || !aligned(V_out, 16) ||
      !aligned(len, 4) || !aligned(cand_begin, 4) || !aligned(score, 4) || !aligned(w_b, 4) ||
      !aligned(target, 4) || !aligned(logn_out, 4) || !aligned(len_out, 4) ||
      (logn && !aligned(logn, 4)) || (dbg_out_offset && !aligned(dbg_out_offset, 4)) ||
      (dbg_kmerged_f32 && !aligned(dbg_kmerged_f32, 16)))
    return KVS_ERR_INVALID_ARG;

  const bool inplace = (K_out == K);
  if (inplace) {
    if (V_out != V || logn_out != logn || len_out != len || T_cap_out != desc->T_cap)
      return KVS_ERR_ALIAS;
  }
  const size_t heads = (size_t)desc->B * desc->H_kv;
  const size_t pairs = heads * (desc->T_cap / 2);
  Range in[] = {{(const char*)K, cache_bytes(desc, desc->T_cap)},
                {(const char*)V, cache_bytes(desc, desc->T_cap)},
                {(const char*)logn, logn ? heads * desc->T_cap * sizeof(float) : 0},
                {(const char*)len, heads * sizeof(int32_t)},
                {(const char*)cand_begin, heads * sizeof(int32_t)},
                {(const char*)score, pairs * sizeof(float)},
                {(const char*)w_b, pairs * sizeof(float)},
                {(const char*)target, (scope == KVS_SCOPE_POOLED ? desc->B : heads) * sizeof(int32_t)}};
  Range outr[] = {{(const char*)K_out, cache_bytes(desc, T_cap_out)},
                  {(const char*)V_out, cache_bytes(desc, T_cap_out)},
                  {(const char*)logn_out, heads * (size_t)T_cap_out * sizeof(float)},
                  {(const char*)len_out, heads * sizeof(int32_t)},
                  {(const char*)dbg_selected, dbg_selected ? pairs : 0},
                  {(const char*)dbg_out_offset, dbg_out_offset ? pairs * sizeof(int32_t) : 0},
                  {(const char*)dbg_kmerged_f32, dbg_kmerged_f32 ? pairs * desc->d * sizeof(float) : 0}};
  const int n_in = sizeof(in) / sizeof(in[0]), n_out = sizeof(outr) / sizeof(outr[0]);
  for (int i = 0; i < n_out; ++i) {
    for (int j = 0; j < n_in; ++j) {
      // in-place mode rewrites K, V, logn and len through themselves
      if (inplace && i < 4 && j == i) continue;
      if (inplace && i < 4 && j < 4 && i != j && overlap(outr[i], in[j])) return KVS_ERR_ALIAS;
      if (!(inplace && i < 4 && j < 4) && overlap(outr[i], in[j])) return KVS_ERR_ALIAS;
    }
    for (int j = i + 1; j < n_out; ++j)
      if (overlap(outr[i], outr[j])) return KVS_ERR_ALIAS;
  }
  if (inplace && !logn) return KVS_ERR_INVALID_ARG;   // merged counts need somewhere to live

  const MergeLayout Ly = merge_layout(*desc);
  s = check_ws(ws, ws_bytes, Ly.total);
  if (s != KVS_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  cudaError_t e = launch_select(*desc, score, len, cand_begin, n_recent, target, scope, Ly, w, st);
  if (e != cudaSuccess) return KVS_ERR_CUDA;
  e = launch_merge(*desc, K, V, logn, score, w_b, scope, T_cap_out, inplace, K_out, V_out,
                   logn_out, len_out, dbg_selected, dbg_out_offset, dbg_kmerged_f32, Ly, w, st);
  return from_cuda(e);
}

kvs_status kvs_plan_rounds(int32_t len, int32_t target, int32_t cand_begin, int32_t n_recent,
                           int32_t* lens_out, int32_t max_lens, int32_t* n_rounds) {
  if (!lens_out || !n_rounds || len < 0 || target < 0 || cand_begin < 0 || n_recent < 0 ||
      max_lens < 1)
    return KVS_ERR_INVALID_ARG;
  int32_t L = len, k = 0;
  lens_out[0] = L;
  while (L > target) {
    const int32_t span = L - n_recent - cand_begin;
    const int32_t P = span > 0 ? span / 2 : 0;
    const int32_t R = P < L - target ? P : L - target;
    if (R <= 0) return KVS_ERR_BUDGET;
    if (k + 1 >= max_lens) return KVS_ERR_INVALID_ARG;
    L -= R;
    lens_out[++k] = L;
  }
  *n_rounds = k;
  return KVS_OK;
}

kvs_status kvs_prefill_chunk(const kvs_cache_desc* desc, void* K, void* V, float* logn,
                             int32_t* len, int32_t L, const void* k_chunk, const void* v_chunk,
                             int32_t n, const void* Q_win, int32_t W, int32_t budget,
                             int32_t sink, int32_t form, int32_t* L_out, void* ws,
                             size_t ws_bytes, kvs_stream_t stream) {
  kvs_status s = check_desc(desc);
  if (s != KVS_OK) return s;
  if (!K || !V || !logn || !len || !Q_win || !L_out || (n > 0 && (!k_chunk || !v_chunk)))
    return KVS_ERR_INVALID_ARG;
  if (form < 0 || form > (KVS_FORM_DIAGONAL | KVS_FORM_PER_QUERY)) return KVS_ERR_INVALID_ARG;
  if ((form & KVS_FORM_PER_QUERY) && !window_fused_supported(*desc, W)) return KVS_ERR_UNSUPPORTED;
  if (!aligned(K, 16) || !aligned(V, 16) || !aligned(Q_win, 16) || !aligned(logn, 4) ||
      !aligned(len, 4) || (n > 0 && (!aligned(k_chunk, 16) || !aligned(v_chunk, 16))))
    return KVS_ERR_INVALID_ARG;
  if (L < 0 || n < 0 || W < 1 || sink < 0 || budget < 0) return KVS_ERR_INVALID_ARG;
  if ((long long)L + n > desc->T_cap) return KVS_ERR_INVALID_ARG;
  const int G = desc->H_q / desc->H_kv;
  if (G * W > 128) return KVS_ERR_UNSUPPORTED;
  // the rounds rewrite each head in place from its candidate start on
  if ((long long)L + n - sink > kInplaceMaxSpan) return KVS_ERR_UNSUPPORTED;
  const size_t heads = (size_t)desc->B * desc->H_kv;
  const size_t chunk_bytes = heads * (size_t)n * desc->d * elem_bytes(desc);
  // the cache (written) must not overlap itself or the chunk and window (read);
  // inputs may share memory with each other
  const Range outs[] = {{(const char*)K, cache_bytes(desc, desc->T_cap)},
                        {(const char*)V, cache_bytes(desc, desc->T_cap)},
                        {(const char*)logn, heads * desc->T_cap * sizeof(float)},
                        {(const char*)len, heads * sizeof(int32_t)}};
  const Range ins[] = {{(const char*)k_chunk, chunk_bytes}, {(const char*)v_chunk, chunk_bytes},
                       {(const char*)Q_win, (size_t)desc->B * desc->H_q * W * desc->d * elem_bytes(desc)}};
  for (int i = 0; i < 4; ++i) {
    for (int j = i + 1; j < 4; ++j)
      if (overlap(outs[i], outs[j])) return KVS_ERR_ALIAS;
    for (int j = 0; j < 3; ++j)
      if (overlap(outs[i], ins[j])) return KVS_ERR_ALIAS;
  }
  // plan the rounds on the host (every head has length L): R = min(P, len - budget)
  int rounds = 0, Lc = L + n;
  while (Lc > budget) {
    const int span = Lc - W - sink;
    const int P = span > 0 ? span / 2 : 0;
    const int R = P < Lc - budget ? P : Lc - budget;
    if (R <= 0 || rounds == 64) return KVS_ERR_BUDGET;   // nothing launched
    ++rounds;
    Lc -= R;
  }
  const PrefillLayout Ly = prefill_layout(*desc, W);
  s = check_ws(ws, ws_bytes, Ly.total);
  if (s != KVS_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  float* score = reinterpret_cast<float*>(w + Ly.score_arr);
  float* w_b = reinterpret_cast<float*>(w + Ly.w_b_arr);
  int32_t* cand = reinterpret_cast<int32_t*>(w + Ly.cand);
  int32_t* target = reinterpret_cast<int32_t*>(w + Ly.target);
  cudaError_t e = launch_append_rows(*desc, K, V, logn, len, L, k_chunk, v_chunk, n, w, st);
  if (e != cudaSuccess) return KVS_ERR_CUDA;
  if (rounds > 0) {
    e = launch_fill2(cand, sink, target, budget, (int)heads, st);
    if (e != cudaSuccess) return KVS_ERR_CUDA;
  }
  for (int r = 0; r < rounds; ++r) {
    e = score_pass(*desc, K, V, logn, len, cand, W, Q_win, W, form, Ly.score, w, score, w_b, st);
    if (e != cudaSuccess) return KVS_ERR_CUDA;
    e = launch_select(*desc, score, len, cand, W, target, KVS_SCOPE_HEAD, Ly.merge, w, st);
    if (e != cudaSuccess) return KVS_ERR_CUDA;
    e = launch_merge(*desc, K, V, logn, score, w_b, KVS_SCOPE_HEAD, desc->T_cap, true, K, V, logn,
                     len, nullptr, nullptr, nullptr, Ly.merge, w, st);
    if (e != cudaSuccess) return KVS_ERR_CUDA;
  }
  *L_out = Lc;
  return KVS_OK;
}

kvs_status kvs_decode_attn(const kvs_cache_desc* desc, const void* q, void* K, void* V,
                           float* logn, int32_t* len, const void* k_new, const void* v_new,
                           void* out, void* ws, size_t ws_bytes, kvs_stream_t stream) {
  kvs_status s = check_desc(desc);
  if (s != KVS_OK) return s;
  if (!q || !K || !V || !len || !out) return KVS_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return KVS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 16) ||
      !aligned(len, 4) || (logn && !aligned(logn, 4)))
    return KVS_ERR_INVALID_ARG;
  const size_t qbytes = (size_t)desc->B * desc->H_q * desc->d * elem_bytes(desc);
  Range ro{(const char*)out, qbytes};
  if (overlap(ro, {(const char*)q, qbytes}) || overlap(ro, {(const char*)K, cache_bytes(desc, desc->T_cap)}) ||
      overlap(ro, {(const char*)V, cache_bytes(desc, desc->T_cap)}))
    return KVS_ERR_ALIAS;
  const DecodeLayout Ly = decode_layout(*desc);
  s = check_ws(ws, ws_bytes, Ly.total);
  if (s != KVS_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return from_cuda(launch_decode(*desc, q, K, V, logn, len, k_new, v_new, out, Ly,
                                 static_cast<char*>(ws), st));
}

kvs_status kvs_stream_read(const void* buf, int64_t rows, int32_t d, int32_t ctas, void* ws,
                           size_t ws_bytes, kvs_stream_t stream) {
  if (!buf || !aligned(buf, 16) || rows <= 0 || rows >= (1ll << 31) || ctas <= 0 ||
      ctas > 65535)
    return KVS_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return KVS_ERR_UNSUPPORTED;
  kvs_status s = check_ws(ws, ws_bytes, kWsAlign);
  if (s != KVS_OK) return s;
  if (!tensor_map_encoder()) return KVS_ERR_UNSUPPORTED;
  return from_cuda(launch_stream_probe(buf, rows, d, ctas, static_cast<char*>(ws),
                                       reinterpret_cast<cudaStream_t>(stream)));
}

kvs_status kvs_device_flags(void* ws, int32_t* flags, int32_t clear, kvs_stream_t stream) {
  if (!ws || !flags || !aligned(ws, kWsAlign)) return KVS_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return KVS_ERR_CUDA;
  if (clear && cudaMemsetAsync(ws, 0, sizeof(int32_t), st) != cudaSuccess) return KVS_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return KVS_ERR_CUDA;
  *flags = h;
  return KVS_OK;
}

}  // extern "C"
