// Generic verify attention on CUDA cores (any D % 8 == 0 up to 256, any page size, f32 or bf16).
//
// Each persistent CTA walks its contiguous range of (request, KV head, 64-key tile) units
// (attn_common.cuh).  Per segment piece it stages the G*Q_r query rows in shared memory
// (pre-scaled by scale*log2(e)), streams the cache keys/values of its tiles 32 keys at a time
// (page lookup per key through the block table), runs the online softmax per row in fp32 and
// accumulates P.V.  The piece that owns the segment's last tile also folds in the request's own
// verify tokens with the causal rule taken from the markers: new key i is visible to the query
// at position pos iff kv_len + i <= pos.
#pragma once

#include "attn_common.cuh"

namespace dspark {

constexpr int kGenThreads = 256;
constexpr int kGenKC = 32;  // keys per inner chunk (= warp width: one lane per key in softmax)

struct AttnArgs {
  const void *q, *k_new, *v_new, *kv_pages;
  int64_t num_pages;
  const int32_t *block_table;
  int max_pages;
  const int32_t *kv_len, *markers, *q_offsets;
  int R, T_cap, Hq, Hkv, G, D, K, page_size, rows_max;
  float scale_log2;  // softmax scale * log2(e)
  void *out;
  AttnWs ws;
};

inline size_t attn_generic_smem_bytes(int rows_max, int D) {
  return sizeof(float) * ((size_t)2 * rows_max * D + (size_t)kGenKC * (D + 1) +
                          (size_t)kGenKC * D + (size_t)rows_max * kGenKC + 3 * (size_t)rows_max);
}

// Validate a segment's offsets, cache length and markers; fills pos[] (absolute positions).
__device__ __forceinline__ bool validate_segment(const AttnArgs &a, int r, int &t0, int &Q,
                                                 int &n, int *pos, int *s_bad) {
  t0 = __ldg(a.q_offsets + r);
  Q = __ldg(a.q_offsets + r + 1) - t0;
  n = __ldg(a.kv_len + r);
  if (threadIdx.x == 0) *s_bad = 0;
  __syncthreads();
  bool ok = (Q >= 1 && Q <= a.K + 1 && t0 >= 0 && t0 + Q <= a.T_cap);
  if (!ok && threadIdx.x == 0) raise_error(DSPARK_DERR_OFFSETS);
  const bool okn = (n >= 0 && (int64_t)(n + a.page_size - 1) / a.page_size <= a.max_pages);
  if (ok && !okn && threadIdx.x == 0) raise_error(DSPARK_DERR_KV_LEN);
  ok = ok && okn;
  if (ok && (int)threadIdx.x < Q) {
    const int j = threadIdx.x;
    const int mr = __ldg(a.markers + 2 * (t0 + j));
    const int mp = __ldg(a.markers + 2 * (t0 + j) + 1);
    pos[j] = mp;
    if (mr != r || mp != n + j) {
      raise_error(DSPARK_DERR_MARKER);
      atomicOr(s_bad, 1);
    }
  }
  __syncthreads();
  return ok && (*s_bad == 0);
}

template <typename T>
__device__ __forceinline__ void load_row8(float *dst, const T *src) {
  float v[8];
  load8(src, v);
#pragma unroll
  for (int e = 0; e < 8; ++e) dst[e] = v[e];
}

template <typename T>
__global__ void __launch_bounds__(kGenThreads)
attn_generic_kernel(AttnArgs a) {
  extern __shared__ __align__(16) float gsm[];
  const int D = a.D, rows_max = a.rows_max, G = a.G;
  float *qs = gsm;                              // [rows_max][D]
  float *acc = qs + (size_t)rows_max * D;       // [rows_max][D]
  float *ks = acc + (size_t)rows_max * D;       // [KC][D+1]
  float *vs = ks + (size_t)kGenKC * (D + 1);    // [KC][D]
  float *sc = vs + (size_t)kGenKC * D;          // [rows_max][KC]
  float *m_s = sc + (size_t)rows_max * kGenKC;
  float *l_s = m_s + rows_max;
  float *al_s = l_s + rows_max;
  __shared__ int s_pos[DSPARK_MAX_K + 1];
  __shared__ int s_bad, s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = kGenThreads / 32;
  const T *qg = static_cast<const T *>(a.q);
  const T *kn = static_cast<const T *>(a.k_new);
  const T *vn = static_cast<const T *>(a.v_new);
  const T *kv = static_cast<const T *>(a.kv_pages);
  T *og = static_cast<T *>(a.out);

  const int total = __ldg(a.ws.tile_prefix + a.R);
  const int W = (total + gridDim.x - 1) / gridDim.x;
  const int c = blockIdx.x;
  const int u0 = c * W, u1 = min(u0 + W, total);
  if (u0 >= u1) return;

  int u = u0;
  bool first = true;
  while (u < u1) {
    int r, g, tiles, s0;
    find_segment(a.ws.tile_prefix, a.R, a.Hkv, u, r, g, tiles, s0);
    const int ta = u - s0;
    const int tb = min(tiles, ta + (u1 - u));
    int t0, Q, n;
    const bool valid = validate_segment(a, r, t0, Q, n, s_pos, &s_bad);
    const int rows = valid ? G * Q : 0;

    // stage queries (row rho = j*G + i <-> token t0+j, head g*G+i), reset the softmax state
    for (int idx = tid; idx < rows * (D / 8); idx += kGenThreads) {
      const int rho = idx / (D / 8), d8 = idx % (D / 8);
      const int j = rho / G, i = rho % G;
      float v[8];
      load8(qg + ((size_t)(t0 + j) * a.Hq + g * G + i) * D + d8 * 8, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) qs[rho * D + d8 * 8 + e] = v[e] * a.scale_log2;
    }
    for (int idx = tid; idx < rows * D; idx += kGenThreads) acc[idx] = 0.f;
    for (int rho = tid; rho < rows; rho += kGenThreads) { m_s[rho] = -INFINITY; l_s[rho] = 0.f; }
    __syncthreads();

    auto chunk_update = [&](int nk, bool causal) {
      for (int idx = tid; idx < rows * kGenKC; idx += kGenThreads) {
        const int rho = idx / kGenKC, kk = idx % kGenKC;
        float s = -INFINITY;
        if (kk < nk && (!causal || n + kk <= s_pos[rho / G])) {
          const float *qr = qs + rho * D;
          const float *kr = ks + kk * (D + 1);
          float d0 = 0.f, d1 = 0.f;
          for (int d = 0; d < D; d += 2) { d0 = fmaf(qr[d], kr[d], d0); d1 = fmaf(qr[d + 1], kr[d + 1], d1); }
          s = d0 + d1;
        }
        sc[idx] = s;
      }
      __syncthreads();
      for (int rho = warp; rho < rows; rho += NW) {
        const float s = sc[rho * kGenKC + lane];
        const float m_old = m_s[rho];
        const float m_new = fmaxf(m_old, warp_max(s));
        float p = 0.f, alpha = 1.f;
        if (m_new != -INFINITY) { p = exp2f(s - m_new); alpha = exp2f(m_old - m_new); }
        sc[rho * kGenKC + lane] = p;
        const float psum = warp_sum(p);
        if (lane == 0) { l_s[rho] = l_s[rho] * alpha + psum; m_s[rho] = m_new; al_s[rho] = alpha; }
      }
      __syncthreads();
      for (int idx = tid; idx < rows * D; idx += kGenThreads) {
        const int rho = idx / D, d = idx % D;
        float o = acc[idx] * al_s[rho];
        const float *pr = sc + rho * kGenKC;
        for (int kk = 0; kk < nk; ++kk) o = fmaf(pr[kk], vs[kk * D + d], o);
        acc[idx] = o;
      }
      __syncthreads();
    };

    if (rows > 0) {
      for (int tile = ta; tile < min(tb, segment_cache_tiles(tiles)); ++tile) {  // cache tiles
        const int k0 = tile * kTileKeys, k1 = min(k0 + kTileKeys, n);
        for (int c0 = k0; c0 < k1; c0 += kGenKC) {
          const int nk = min(kGenKC, k1 - c0);
          for (int idx = tid; idx < kGenKC * (D / 8); idx += kGenThreads) {
            const int kk = idx / (D / 8), d8 = idx % (D / 8);
            float kvv[8], vvv[8];
            bool have = false;
            if (kk < nk) {
              const int p = c0 + kk;
              const int page = __ldg(a.block_table + (size_t)r * a.max_pages + p / a.page_size);
              if (page >= 0 && page < a.num_pages) {
                const size_t base = ((((size_t)page * 2) * a.Hkv + g) * a.page_size +
                                     p % a.page_size) * D + d8 * 8;
                const size_t vofs = (size_t)a.Hkv * a.page_size * D;
                load8(kv + base, kvv);
                load8(kv + base + vofs, vvv);
                have = true;
              } else if (d8 == 0) {
                raise_error(DSPARK_DERR_PAGE);
              }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              ks[kk * (D + 1) + d8 * 8 + e] = have ? kvv[e] : 0.f;
              vs[kk * D + d8 * 8 + e] = have ? vvv[e] : 0.f;
            }
          }
          __syncthreads();
          chunk_update(nk, false);
        }
      }
      if (tb == tiles) {  // the segment's last unit: the request's own verify tokens, causal
        for (int idx = tid; idx < kGenKC * (D / 8); idx += kGenThreads) {
          const int kk = idx / (D / 8), d8 = idx % (D / 8);
          float kvv[8] = {0, 0, 0, 0, 0, 0, 0, 0}, vvv[8] = {0, 0, 0, 0, 0, 0, 0, 0};
          if (kk < Q) {
            load8(kn + ((size_t)(t0 + kk) * a.Hkv + g) * D + d8 * 8, kvv);
            load8(vn + ((size_t)(t0 + kk) * a.Hkv + g) * D + d8 * 8, vvv);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            ks[kk * (D + 1) + d8 * 8 + e] = kvv[e];
            vs[kk * D + d8 * 8 + e] = vvv[e];
          }
        }
        __syncthreads();
        chunk_update(Q, true);
      }
    }

    if (ta == 0 && tb == tiles) {
      for (int idx = tid; idx < rows * D; idx += kGenThreads) {
        const int rho = idx / D, d = idx % D, j = rho / G, i = rho % G;
        og[((size_t)(t0 + j) * a.Hq + g * G + i) * D + d] = from_f32<T>(acc[idx] / l_s[rho]);
      }
    } else {
      float *P = a.ws.partials + (size_t)partial_slot(c, s0, W) * rows_max * part_stride(D);
      for (int idx = tid; idx < rows_max * part_stride(D); idx += kGenThreads) {
        const int rho = idx / part_stride(D), d = idx % part_stride(D);
        float val;
        if (rho < rows) val = (d < D) ? acc[rho * D + d] : (d == D ? m_s[rho] : l_s[rho]);
        else val = (d == D) ? -INFINITY : 0.f;
        P[idx] = val;
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) {
        const int pieces = (s0 + tiles - 1) / W - s0 / W + 1;
        const int prev = atomicAdd(a.ws.counters + r * a.Hkv + g, 1);
        s_last = (prev == pieces - 1);
      }
      __syncthreads();
      if (s_last) {
        __threadfence();
        const int c_first = s0 / W, c_last = (s0 + tiles - 1) / W;
        for (int rho = warp; rho < rows; rho += NW) {
          float M = -INFINITY;
          for (int cc = c_first; cc <= c_last; ++cc) {
            const float *Pp = a.ws.partials + (size_t)partial_slot(cc, s0, W) * rows_max * part_stride(D);
            M = fmaxf(M, __ldcg(Pp + rho * part_stride(D) + D));
          }
          float Lsum = 0.f;
          for (int cc = c_first; cc <= c_last; ++cc) {
            const float *Pp = a.ws.partials + (size_t)partial_slot(cc, s0, W) * rows_max * part_stride(D);
            const float mp = __ldcg(Pp + rho * part_stride(D) + D);
            if (mp != -INFINITY) Lsum += __ldcg(Pp + rho * part_stride(D) + D + 1) * exp2f(mp - M);
          }
          const int j = rho / G, i = rho % G;
          for (int d = lane; d < D; d += 32) {
            float o = 0.f;
            for (int cc = c_first; cc <= c_last; ++cc) {
              const float *Pp = a.ws.partials + (size_t)partial_slot(cc, s0, W) * rows_max * part_stride(D);
              const float mp = __ldcg(Pp + rho * part_stride(D) + D);
              if (mp != -INFINITY) o += __ldcg(Pp + rho * part_stride(D) + d) * exp2f(mp - M);
            }
            og[((size_t)(t0 + j) * a.Hq + g * G + i) * D + d] = from_f32<T>(o / Lsum);
          }
        }
        if (tid == 0) a.ws.counters[r * a.Hkv + g] = 0;  // ready for the next call
      }
    }
    __syncthreads();
    u += tb - ta;
    first = false;
  }
  (void)first;
}

}  // namespace dspark
