// libdspark: C ABI entry points (include/dspark.h).  Host-side validation, launch shapes and
// dispatch; the kernels live in the included headers so that the whole library is one module
// with one device error word.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <cmath>
#include <cstdio>

#include "common.cuh"
#include "schedule.cuh"
#include "attn_common.cuh"
#include "attn_generic.cuh"
#include "accept.cuh"
#include "kv_commit.cuh"
#include "calibrate.cuh"
#include "draft.cuh"
#include "attn_tk.cuh"

#include <cudaTypedefs.h>

using namespace dspark;

namespace {

constexpr int kVersion = 100;  // 0.1.0

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DSPARK_OK : DSPARK_ECUDA;
}

int max_attn_ctas() {
  const int sms = sm_count();
  return sms > 0 ? sms * kMaxCtasPerSm : -1;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// The paged cache as whole-page boxes for the tensor-core kernel: a 4-D view
// {d 64, row-in-group 8, d-half 2, row group} with strides 256 B, 128 B and 2048 B over the rows
// of [rows][128] bf16 (rows = pages * 2 * Hkv * page_size, a multiple of 64), 128-byte swizzle,
// boxes of one page (8 groups): shared memory receives [group][d-half][8 rows][128 B].  Groups
// past the end read as 0.
bool encode_kv_page_map(CUtensorMap *map, const void *kv_pages, uint64_t rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {64, 8, 2, rows / 8};
  cuuint64_t strides[3] = {128 * 2, 64 * 2, 8 * 128 * 2};
  cuuint32_t box[4] = {64, 8, 2, 8};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(kv_pages), dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The verify tokens' own K or V rows [T_cap][Hkv][128] bf16 in the same shared-memory layout: a
// 4-D view {d 64, token, d-half 2, head} with strides Hkv * 256 B, 128 B and 256 B, 128-byte
// swizzle, boxes of 8 tokens x both d-halves of one head (one 2048-byte row group); tokens past
// T_cap read as 0.
bool encode_new_group_map(CUtensorMap *map, const void *ptr, int T_cap, int Hkv) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {64, (cuuint64_t)T_cap, 2, (cuuint64_t)Hkv};
  cuuint64_t strides[3] = {(cuuint64_t)Hkv * 128 * 2, 64 * 2, 128 * 2};
  cuuint32_t box[4] = {64, 8, 2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

const char *dspark_status_string(int status) {
  switch (status) {
    case DSPARK_OK: return "DSPARK_OK";
    case DSPARK_EINVAL: return "DSPARK_EINVAL: invalid argument";
    case DSPARK_ECUDA: return "DSPARK_ECUDA: CUDA runtime error";
    case DSPARK_EWORKSPACE: return "DSPARK_EWORKSPACE: workspace missing or too small";
    case DSPARK_EDEVICE_DATA: return "DSPARK_EDEVICE_DATA: invalid device-resident data";
    case DSPARK_ETIMEOUT: return "DSPARK_ETIMEOUT: bounded wait expired";
    case DSPARK_EUNSUPPORTED: return "DSPARK_EUNSUPPORTED: shape not supported by this build";
    default: return "DSPARK_UNKNOWN_STATUS";
  }
}

int dspark_version(void) { return kVersion; }

int dspark_schedule(const float *conf_ring, int ring_depth, int round_idx, int R, int K,
                    const int32_t *kv_len, const double *t_ms, int T_cap, int32_t *verify_len,
                    int32_t *q_offsets, int32_t *markers, int32_t *T_out, double *objective,
                    dspark_stream_t stream) {
  if (!conf_ring || !t_ms || !verify_len || !q_offsets || !T_out || !objective)
    return DSPARK_EINVAL;
  if ((kv_len == nullptr) != (markers == nullptr)) return DSPARK_EINVAL;  // both or neither
  if (R < 1 || K < 1 || K > DSPARK_MAX_K || ring_depth < DSPARK_CONF_LAG + 1 || round_idx < 0 ||
      T_cap < R)
    return DSPARK_EINVAL;
  if ((int64_t)R * K > DSPARK_MAX_CANDIDATES) return DSPARK_EUNSUPPORTED;
  const int N = R * K;
  int E = 1;
  while (kSchedThreads * E < N) E *= 2;
  const size_t smem = schedule_smem_bytes(E);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
#define DSPARK_SCHED_LAUNCH(EE)                                                                \
  do {                                                                                         \
    if (cudaFuncSetAttribute(schedule_kernel<EE>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             (int)smem) != cudaSuccess)                                        \
      return DSPARK_ECUDA;                                                                     \
    schedule_kernel<EE><<<1, kSchedThreads, smem, s>>>(conf_ring, ring_depth, round_idx, R, K, \
                                                       kv_len, t_ms, T_cap, verify_len,        \
                                                       q_offsets, markers, T_out, objective);  \
  } while (0)
  switch (E) {
    case 1: DSPARK_SCHED_LAUNCH(1); break;
    case 2: DSPARK_SCHED_LAUNCH(2); break;
    case 4: DSPARK_SCHED_LAUNCH(4); break;
    case 8: DSPARK_SCHED_LAUNCH(8); break;
    case 16: DSPARK_SCHED_LAUNCH(16); break;
    default: return DSPARK_EUNSUPPORTED;
  }
#undef DSPARK_SCHED_LAUNCH
  return launch_status();
}

int dspark_flatten_markers(const int32_t *kv_len, const int32_t *q_offsets, int R, int K,
                           int T_cap, int32_t *markers, dspark_stream_t stream) {
  if (!kv_len || !q_offsets || !markers || R < 1 || K < 1 || K > DSPARK_MAX_K || T_cap < R)
    return DSPARK_EINVAL;
  flatten_markers_kernel<<<(R + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      kv_len, q_offsets, R, K, T_cap, markers);
  return launch_status();
}

size_t dspark_verify_attn_workspace_bytes(int R, int Hq, int Hkv, int D, int K) {
  if (R < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || D < 1 || K < 1 || K > DSPARK_MAX_K)
    return 0;
  const int ctas = max_attn_ctas();
  if (ctas <= 0) return 0;
  return attn_ws_layout(R, Hkv, (Hq / Hkv) * (K + 1), D, ctas, nullptr, nullptr);
}

int dspark_verify_attn_plan(const int32_t *kv_len, const int32_t *q_offsets,
                            const int32_t *markers, int R, int T_cap, int Hq, int Hkv, int D,
                            int K, void *ws, size_t ws_bytes, dspark_stream_t stream) {
  if (!kv_len || !q_offsets || !markers || R < 1 || T_cap < R || Hkv < 1 || Hq < Hkv ||
      Hq % Hkv != 0 || D < 8 || D > 256 || D % 8 || K < 1 || K > DSPARK_MAX_K)
    return DSPARK_EINVAL;
  if (!ws || !aligned16(ws)) return DSPARK_EWORKSPACE;
  const int ctas = max_attn_ctas();
  if (ctas <= 0) return DSPARK_ECUDA;
  const int rows_max = (Hq / Hkv) * (K + 1);
  AttnWs w;
  if (ws_bytes < attn_ws_layout(R, Hkv, rows_max, D, ctas, &w, ws)) return DSPARK_EWORKSPACE;
  attn_plan_kernel<<<1, 1024, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      kv_len, q_offsets, markers, R, T_cap, K, Hkv, rows_max, D, sm_count(), w);
  return launch_status();
}

int dspark_verify_attn(const void *q, const void *k_new, const void *v_new, const void *kv_pages,
                       int64_t num_pages, const int32_t *block_table, int max_pages,
                       const int32_t *kv_len, const int32_t *markers, const int32_t *q_offsets,
                       int R, int T_cap, int Hq, int Hkv, int D, int K, int page_size, int dtype,
                       float scale, void *out, void *ws, size_t ws_bytes,
                       dspark_stream_t stream) {
  if (!q || !k_new || !v_new || !kv_pages || !block_table || !kv_len || !markers || !q_offsets ||
      !out)
    return DSPARK_EINVAL;
  if (R < 1 || T_cap < R || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || K < 1 || K > DSPARK_MAX_K ||
      page_size < 1 || max_pages < 1 || num_pages < 1 || !std::isfinite(scale))
    return DSPARK_EINVAL;
  if (D < 8 || D > 256 || D % 8 != 0) return DSPARK_EUNSUPPORTED;
  if (dtype != DSPARK_BF16 && dtype != DSPARK_F32) return DSPARK_EINVAL;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(kv_pages) ||
      !aligned16(out))
    return DSPARK_EINVAL;
  const int G = Hq / Hkv;
  const int rows_max = G * (K + 1);
  if (rows_max > 128) return DSPARK_EUNSUPPORTED;
  if (!ws || !aligned16(ws)) return DSPARK_EWORKSPACE;
  const int sms = sm_count();
  if (sms <= 0) return DSPARK_ECUDA;
  AttnWs w;
  if (ws_bytes < attn_ws_layout(R, Hkv, rows_max, D, sms * kMaxCtasPerSm, &w, ws))
    return DSPARK_EWORKSPACE;

  AttnArgs a;
  a.q = q; a.k_new = k_new; a.v_new = v_new; a.kv_pages = kv_pages; a.num_pages = num_pages;
  a.block_table = block_table; a.max_pages = max_pages; a.kv_len = kv_len; a.markers = markers;
  a.q_offsets = q_offsets; a.R = R; a.T_cap = T_cap; a.Hq = Hq; a.Hkv = Hkv; a.G = G; a.D = D;
  a.K = K; a.page_size = page_size; a.rows_max = rows_max;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = out; a.ws = w;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint64_t kv_rows = (uint64_t)num_pages * 2 * Hkv * page_size;
  if (dtype == DSPARK_BF16 && D == 128 && page_size % 64 == 0 && kv_rows < (1ull << 31) &&
      K + 1 <= tk::kNewRows && rows_max <= 64) {
    CUtensorMap map, map_kn, map_vn;
    if (!encode_kv_page_map(&map, kv_pages, kv_rows) ||
        !encode_new_group_map(&map_kn, k_new, T_cap, Hkv) ||
        !encode_new_group_map(&map_vn, v_new, T_cap, Hkv))
      return DSPARK_ECUDA;
    if (cudaFuncSetAttribute(tk::attn_tk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tk::kSmemBytes) != cudaSuccess)
      return DSPARK_ECUDA;
    // the kernel splits its register pool across warpgroups (setmaxnreg): the pool it is launched
    // with, the compiled registers per thread x threads, must hold the split, or the increase
    // would wait for registers that never come free
    {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, tk::attn_tk_kernel) != cudaSuccess) return DSPARK_ECUDA;
      if (fa.numRegs < tk::kRegsLaunch || fa.maxThreadsPerBlock < tk::kThreads)
        return DSPARK_EUNSUPPORTED;
    }
    // programmatic stream serialisation: the kernel's prologue may overlap the previous kernel
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(tk::kThreads);
    cfg.dynamicSmemBytes = tk::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, tk::attn_tk_kernel, map, map_kn, map_vn, a, (int)kv_rows) !=
        cudaSuccess)
      return DSPARK_ECUDA;
    return launch_status();
  }
  const size_t smem = attn_generic_smem_bytes(rows_max, D);
  if (smem > 227 * 1024) return DSPARK_EUNSUPPORTED;
  auto launch = [&](auto kernel) -> int {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DSPARK_ECUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kGenThreads, smem) !=
        cudaSuccess)
      return DSPARK_ECUDA;
    per_sm = std::max(1, std::min(per_sm, kMaxCtasPerSm));
    kernel<<<sms * per_sm, kGenThreads, smem, s>>>(a);
    return launch_status();
  };
  if (dtype == DSPARK_BF16) return launch(attn_generic_kernel<__nv_bfloat16>);
  return launch(attn_generic_kernel<float>);
}

size_t dspark_accept_workspace_bytes(int R, int K, int T_cap) {
  if (R < 1 || K < 1 || K > DSPARK_MAX_K || T_cap < R) return 0;
  return accept_ws_bytes(R, K, T_cap);
}

int dspark_accept(const void *target_logits, const void *draft_logits, int dtype, int V, int R,
                  int K, int T_cap, const int32_t *draft_tokens, const int32_t *verify_len,
                  const int32_t *q_offsets, const float *u_acc, const float *u_res,
                  float temperature, int32_t *accepted_len, int32_t *out_tokens, int32_t *n_out,
                  void *ws, size_t ws_bytes, dspark_stream_t stream) {
  const bool greedy = !(temperature > 0.f);
  if (!target_logits || !draft_tokens || !verify_len || !q_offsets || !accepted_len ||
      !out_tokens || !n_out)
    return DSPARK_EINVAL;
  if (!greedy && (!draft_logits || !u_acc || !u_res)) return DSPARK_EINVAL;
  if (std::isnan(temperature) || std::isinf(temperature)) return DSPARK_EINVAL;
  if (V < 1 || R < 1 || K < 1 || K > DSPARK_MAX_K || T_cap < R) return DSPARK_EINVAL;
  if (dtype != DSPARK_BF16 && dtype != DSPARK_F32) return DSPARK_EINVAL;
  if (!ws || ws_bytes < accept_ws_bytes(R, K, T_cap) || !aligned16(ws)) return DSPARK_EWORKSPACE;
  ExpScale c;
  c.d = greedy ? 0.0 : 1.4426950408889634 / (double)temperature;
  // hi rounded toward zero, so lo >= 0 (and > 0: a zero lo is replaced by the least normal
  // float), which lets d * hi + d * lo stay -inf for a -inf logit without a clamp
  c.hi = (float)c.d;
  if ((double)c.hi > c.d) c.hi = std::nextafter(c.hi, 0.f);  // c > 0: toward zero
  if (greedy) c.hi = 0.f;
  c.lo = greedy ? 0.f : fmaxf((float)(c.d - (double)c.hi), 1.17549435e-38f);
  RowStats *st = static_cast<RowStats *>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int nrows = T_cap + R * K;
  const size_t fin_smem = accept_finalize_smem(V);
  if (fin_smem > 227 * 1024) return DSPARK_EUNSUPPORTED;
  // CTAs per request for the draw: as many as keep the whole grid resident (kAccFinBlocks CTAs
  // per SM for bf16 rows, two for f32), at most 8 (the portable cluster size), never more than
  // the row has chunks
  int ncl = 1;
  if (!greedy) {
    const int sms = sm_count();
    if (sms <= 0) return DSPARK_ECUDA;
    const int nch = (V + kAccChunk - 1) / kAccChunk;
    const int per_sm = dtype == DSPARK_BF16 ? kAccFinBlocks : 2;
    ncl = std::max(1, std::min({8, nch, per_sm * sms / R}));
  }
  auto run = [&](auto tag) -> int {
    using T = decltype(tag);
    const T *tl = static_cast<const T *>(target_logits);
    const T *dl = static_cast<const T *>(draft_logits);
    auto launch = [&](auto stats_kernel, auto fin_kernel) -> int {
      stats_kernel<<<nrows, kAccThreads, 0, s>>>(tl, dl, V, R, K, T_cap, verify_len, q_offsets,
                                                 c, st);
      if (cudaGetLastError() != cudaSuccess) return DSPARK_ECUDA;
      if (fin_smem > 48 * 1024 &&
          cudaFuncSetAttribute(fin_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)fin_smem) != cudaSuccess)
        return DSPARK_ECUDA;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)(R * ncl));
      cfg.blockDim = dim3(kAccThreads);
      cfg.dynamicSmemBytes = fin_smem;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)ncl;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = ncl > 1 ? 1 : 0;
      if (cudaLaunchKernelEx(&cfg, fin_kernel, tl, dl, V, R, K, T_cap, draft_tokens, verify_len,
                             q_offsets, u_acc, u_res, c, (const RowStats *)st, accepted_len,
                             out_tokens, n_out, ncl) != cudaSuccess)
        return DSPARK_ECUDA;
      return launch_status();
    };
    if (greedy) return launch(accept_stats_kernel<T, true>, accept_finalize_kernel<T, true>);
    return launch(accept_stats_kernel<T, false>, accept_finalize_kernel<T, false>);
  };
  if (dtype == DSPARK_BF16) return run(__nv_bfloat16());
  return run(float());
}

int dspark_kv_commit(const void *k_new, const void *v_new, int64_t new_layer_stride,
                     void *kv_pages, int64_t num_pages, int64_t cache_layer_stride, int layers,
                     const int32_t *block_table, int max_pages, const int32_t *kv_len,
                     const int32_t *q_offsets, const int32_t *accepted_len, int R, int T_cap,
                     int Hkv, int D, int K, int page_size, int dtype, int32_t *kv_len_out,
                     dspark_stream_t stream) {
  if (!k_new || !v_new || !kv_pages || !block_table || !kv_len || !q_offsets || !accepted_len ||
      !kv_len_out || kv_len_out == kv_len)
    return DSPARK_EINVAL;
  if (dtype != DSPARK_BF16 && dtype != DSPARK_F32) return DSPARK_EINVAL;
  const int esz = dtype == DSPARK_BF16 ? 2 : 4;
  if (R < 1 || T_cap < R || Hkv < 1 || D < 1 || K < 1 || K > DSPARK_MAX_K || page_size < 1 ||
      max_pages < 1 || num_pages < 1 || layers < 1 || layers > 65535 || (D * esz) % 16 != 0)
    return DSPARK_EINVAL;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(kv_pages)) return DSPARK_EINVAL;
  const int64_t new_elems = (int64_t)T_cap * Hkv * D;
  const int64_t cache_elems = num_pages * 2 * Hkv * page_size * (int64_t)D;
  if (layers > 1 && (new_layer_stride < new_elems || cache_layer_stride < cache_elems ||
                     (new_layer_stride * esz) % 16 != 0 || (cache_layer_stride * esz) % 16 != 0))
    return DSPARK_EINVAL;
  CommitArgs a;
  a.k_new = static_cast<const char *>(k_new);
  a.v_new = static_cast<const char *>(v_new);
  a.kv = static_cast<char *>(kv_pages);
  a.new_layer_bytes = new_layer_stride * esz;
  a.cache_layer_bytes = cache_layer_stride * esz;
  a.num_pages = num_pages;
  a.block_table = block_table; a.kv_len = kv_len; a.q_offsets = q_offsets;
  a.accepted_len = accepted_len; a.kv_len_out = kv_len_out;
  a.max_pages = max_pages; a.R = R; a.T_cap = T_cap; a.Hkv = Hkv; a.D = D; a.K = K;
  a.page_size = page_size; a.esz = esz;
  kv_commit_kernel<<<dim3(R, layers), kCommitThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return launch_status();
}

int dspark_calibrate_confidence(const float *logits, const float *tau, int R, int K, float *conf,
                                dspark_stream_t stream) {
  if (!logits || !tau || !conf || R < 1 || K < 1 || K > DSPARK_MAX_K) return DSPARK_EINVAL;
  const int n = R * K;
  const int blocks = std::min((n + 255) / 256, 1024);
  calibrate_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(logits, tau, R, K,
                                                                                 conf);
  return launch_status();
}

int dspark_fit_temperature(const float *logits, const int32_t *verify_len,
                           const int32_t *accepted_len, int N, int K, float *tau,
                           dspark_stream_t stream) {
  if (!logits || !verify_len || !accepted_len || !tau || N < 1 || K < 1 || K > DSPARK_MAX_K)
    return DSPARK_EINVAL;
  fit_temperature_kernel<<<K, kFitThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      logits, verify_len, accepted_len, N, K, tau);
  return launch_status();
}

size_t dspark_markov_draft_workspace_bytes(int R, int V) {
  if (R < 1 || V < 4) return 0;
  return draft_ws_layout(R, V, nullptr, nullptr);
}

int dspark_markov_draft(const void *block_logits, const void *E, const void *U, int d,
                        const int32_t *x0, int R, int K, int V, float temperature,
                        uint32_t round_idx, uint32_t seed, void *draft_logits,
                        int32_t *draft_tokens, void *ws, size_t ws_bytes,
                        dspark_stream_t stream) {
  if (!block_logits || !E || !U || !x0 || !draft_logits || !draft_tokens) return DSPARK_EINVAL;
  if (R < 1 || K < 1 || K > DSPARK_MAX_K || V < 8 || V % 8 != 0 || d < 8 || d % 8 != 0 ||
      d > kDraftMaxRank || std::isnan(temperature) || std::isinf(temperature))
    return DSPARK_EINVAL;
  if (!aligned16(block_logits) || !aligned16(E) || !aligned16(U) || !aligned16(draft_logits))
    return DSPARK_EINVAL;
  if (!ws || !aligned16(ws) || ws_bytes < draft_ws_layout(R, V, nullptr, nullptr))
    return DSPARK_EWORKSPACE;
  DraftWs w;
  draft_ws_layout(R, V, &w, ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int nslices = (V + kDraftSlice - 1) / kDraftSlice;
  const bool sampled = temperature > 0.f;
  const float inv_tau = sampled ? 1.f / temperature : 1.f;
  const auto *b = static_cast<const __nv_bfloat16 *>(block_logits);
  const auto *e = static_cast<const __nv_bfloat16 *>(E);
  const auto *u = static_cast<const __nv_bfloat16 *>(U);
  auto *o = static_cast<__nv_bfloat16 *>(draft_logits);
  markov_init_kernel<<<(R + 255) / 256, 256, 0, s>>>(x0, R, V, w);
  for (int k = 1; k <= K; ++k) {
    markov_logits_kernel<<<nslices, kDraftThreads, 0, s>>>(b, e, u, d, w.xprev, R, K, V, k,
                                                           inv_tau, sampled ? 1 : 0, round_idx,
                                                           seed, o, w);
    markov_select_kernel<<<R, 128, 0, s>>>(nslices, R, K, k, w, draft_tokens);
  }
  return launch_status();
}

// One thread waits on an mbarrier that nothing arrives at, through the same bounded wait the
// attention kernel uses, with a short limit; it must give up, record DSPARK_DERR_TIMEOUT and
// return, leaving the context usable.
__global__ void wait_selftest_kernel(long long limit_cycles, int32_t *result) {
  __shared__ __align__(8) uint64_t mbar;
  __shared__ volatile int abort_flag;
  const uint32_t bar = ptx::smem_u32(&mbar);
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool completed = ptx::mbar_wait(bar, 0, &abort_flag, limit_cycles);
    result[0] = completed ? 1 : 0;
    result[1] = abort_flag;
  }
}

int dspark_selftest_wait_timeout(long long limit_cycles, int32_t *result, dspark_stream_t stream) {
  if (!result || limit_cycles < 1 || limit_cycles > ptx::kWaitLimitCycles) return DSPARK_EINVAL;
  wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_cycles, result);
  return launch_status();
}

int dspark_read_error(int32_t *host_code, dspark_stream_t stream) {
  if (!host_code) return DSPARK_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSPARK_ECUDA;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(int)) != cudaSuccess) return DSPARK_ECUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return DSPARK_ECUDA;
  *host_code = v;
  return DSPARK_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// No-allocation variant of dspark_accept.
//
// For callers that must not allocate device memory (their memory pool owns the GPU, their host
// runtime forbids allocation after start-up, or an allocation's implicit synchronisation is not
// acceptable).  The per-row statistics the acceptance kernels need live in this fixed array
// instead of a caller workspace.  In host code `g_accept_noalloc_scratch` only names the
// symbol; its device address is looked up once per device and context (with that device
// current) and that address is what the kernels receive.
static __device__ __align__(256) RowStats g_accept_noalloc_scratch[DSPARK_ACCEPT_NOALLOC_MAX_ROWS];

namespace {
constexpr int kNoAllocMaxDevices = 64;

// The array's device address belongs to the context that loaded this module.  A device reset
// (cudaDeviceReset, or the primary context released and created again) loads the module anew
// and may place the array elsewhere, so the cached address is kept together with the id of the
// context it was looked up in and looked up again when the current context's id differs.
struct NoAllocScratch {
  unsigned long long ctx_id = 0;  // 0: not looked up yet
  void *addr = nullptr;
};
NoAllocScratch g_noalloc_scratch[kNoAllocMaxDevices];
std::mutex g_noalloc_mutex;

// Unique id of the calling thread's current context (driver entry points through the runtime,
// no link-time libcuda); false if it cannot be read.
bool current_context_id(unsigned long long *id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}
}  // namespace

extern "C" int dspark_accept_noalloc(const void *target_logits, const void *draft_logits,
                                     int dtype, int V, int R, int K, int T_cap,
                                     const int32_t *draft_tokens, const int32_t *verify_len,
                                     const int32_t *q_offsets, const float *u_acc,
                                     const float *u_res, float temperature,
                                     int32_t *accepted_len, int32_t *out_tokens,
                                     int32_t *n_out, dspark_stream_t stream) {
  if (R < 1 || K < 1 || K > DSPARK_MAX_K || T_cap < R) return DSPARK_EINVAL;
  if ((int64_t)T_cap + (int64_t)R * K > DSPARK_ACCEPT_NOALLOC_MAX_ROWS) return DSPARK_EUNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSPARK_ECUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return DSPARK_EUNSUPPORTED;
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoAllocScratch &e = g_noalloc_scratch[dev];
    unsigned long long ctx_id = 0;
    // no current context yet: the symbol lookup below makes the runtime create it
    const bool have_ctx = current_context_id(&ctx_id);
    if (!have_ctx || e.ctx_id != ctx_id || e.addr == nullptr) {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_accept_noalloc_scratch) != cudaSuccess || !p)
        return DSPARK_ECUDA;
      if (!have_ctx && !current_context_id(&ctx_id)) return DSPARK_ECUDA;
      e.addr = p;
      e.ctx_id = ctx_id;
    }
    scratch = e.addr;
  }
  return dspark_accept(target_logits, draft_logits, dtype, V, R, K, T_cap, draft_tokens,
                       verify_len, q_offsets, u_acc, u_res, temperature, accepted_len,
                       out_tokens, n_out, scratch, sizeof(g_accept_noalloc_scratch), stream);
}
