// dspark_kv_commit: the kept verify rows of every request join its paged KV cache.
//
// "刚融完500亿…专治AI“嘴慢”" opening section (drafts the target confirms are adopted) and "DSpark 的
// 661% 提速…" §一 (verified tokens are kept): after acceptance, request r keeps verify tokens
// j = 0 .. a_r (the token at position kv_len[r] and its a_r accepted drafts); their K/V rows are
// written, for every layer, to the cache slots of positions kv_len[r] + j, and the cache length
// becomes kv_len[r] + a_r + 1.  Rejected drafts never reach the cache, so rollback writes nothing.
//
// One CTA per (request, layer); the request's rows are copied in 16-byte pieces.  Pure data
// movement: (a_r + 1) * Hkv * D * 2 (K and V) elements read and written per request and layer.
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kCommitThreads = 128;

struct CommitArgs {
  const char *k_new, *v_new;       // [layers][T_cap][Hkv][D] (bytes; layer stride below)
  char *kv;                        // `layers` caches [num_pages][2][Hkv][page][D]
  int64_t new_layer_bytes, cache_layer_bytes, num_pages;
  const int32_t *block_table, *kv_len, *q_offsets, *accepted_len;
  int32_t *kv_len_out;
  int max_pages, R, T_cap, Hkv, D, K, page_size, esz;
};

__global__ void __launch_bounds__(kCommitThreads) kv_commit_kernel(CommitArgs a) {
  const int r = blockIdx.x, layer = blockIdx.y, tid = threadIdx.x;
  const int t0 = __ldg(a.q_offsets + r), Q = __ldg(a.q_offsets + r + 1) - t0;
  const int n = __ldg(a.kv_len + r), acc = __ldg(a.accepted_len + r);
  const bool report = (layer == 0 && tid == 0);
  bool ok = Q >= 1 && Q <= a.K + 1 && t0 >= 0 && t0 <= a.T_cap - Q;
  if (!ok && report) raise_error(DSPARK_DERR_OFFSETS);
  if (ok && !(acc >= 0 && acc <= Q - 1)) {
    if (report) raise_error(DSPARK_DERR_ACCEPTED);
    ok = false;
  }
  if (ok && !(n >= 0 && (int64_t)(n + acc) / a.page_size < a.max_pages)) {
    if (report) raise_error(DSPARK_DERR_KV_LEN);
    ok = false;
  }
  // every page the kept rows land in must exist (checked before anything is written)
  __shared__ int s_bad;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  if (ok && tid <= acc) {
    const int pg = __ldg(a.block_table + (size_t)r * a.max_pages + (n + tid) / a.page_size);
    if (pg < 0 || pg >= a.num_pages) s_bad = 1;
  }
  __syncthreads();
  if (ok && s_bad) {
    if (report) raise_error(DSPARK_DERR_PAGE);
    ok = false;
  }
  if (!ok) {
    if (report) a.kv_len_out[r] = n;
    return;
  }
  const int row_chunks = a.D * a.esz / 16;           // 16-byte pieces per K or V row
  const int per_tok = a.Hkv * row_chunks;
  const int total = (acc + 1) * per_tok;
  const char *kn = a.k_new + layer * a.new_layer_bytes;
  const char *vn = a.v_new + layer * a.new_layer_bytes;
  char *kv = a.kv + layer * a.cache_layer_bytes;
  const size_t row_bytes = (size_t)a.D * a.esz;
  for (int i = tid; i < total; i += kCommitThreads) {
    const int j = i / per_tok, rem = i % per_tok, g = rem / row_chunks, c = rem % row_chunks;
    const int pos = n + j;
    const int pg = __ldg(a.block_table + (size_t)r * a.max_pages + pos / a.page_size);
    const size_t src = ((size_t)(t0 + j) * a.Hkv + g) * row_bytes + (size_t)c * 16;
    const size_t dk = ((((size_t)pg * 2) * a.Hkv + g) * a.page_size + pos % a.page_size) *
                          row_bytes + (size_t)c * 16;
    const size_t dv = dk + (size_t)a.Hkv * a.page_size * row_bytes;
    *reinterpret_cast<uint4 *>(kv + dk) = __ldg(reinterpret_cast<const uint4 *>(kn + src));
    *reinterpret_cast<uint4 *>(kv + dv) = __ldg(reinterpret_cast<const uint4 *>(vn + src));
  }
  if (report) a.kv_len_out[r] = n + acc + 1;
}

}  // namespace dspark
