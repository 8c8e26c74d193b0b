// dspark_accept: exact acceptance rule, longest accepted prefix, residual / bonus draw.
//
// Method (DSpark write-ups): "DSpark 的 661% 提速，是真突破还是数字游戏？" §一 (verify all draft
// tokens in one pass, keep the verified ones, resample after the first divergence, output
// distribution equal to the target's); "DeepSeek服务器不再卡顿！…", sections "DSpark的神奇之处"
// (from the first wrong guess the large model writes a correct token itself) and
// "成本与质量的考量" (the acceptance rule preserves the target distribution exactly).
//
// Two kernels:
//   accept_stats_kernel    one CTA per scheduled logit row (target rows t < T, and draft rows
//                          (r, k) with k < verify_len[r] unless greedy).  One streaming pass:
//                          per-thread running max with float32 exp2 terms accumulated into
//                          float64 sums (rescaled when the running max rises), then a block
//                          merge -> (m, Z = sum exp((z - m)/tau), argmax with lowest index).
//   accept_finalize_kernel one CTA per request: the accept chain (thread 0), then the
//                          correction / bonus draw by inverse CDF over one row pair: pass 1
//                          sums the weights per 2048-element chunk (float64), the threshold
//                          u * Z picks the chunk, pass 2 re-reads that chunk and scans it.
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kAccThreads = 256;
constexpr int kAccChunk = kAccThreads * 8;

struct RowStats {
  float m;      // row maximum
  int argmax;   // lowest index attaining m
  double Z;     // sum_v exp2((z_v - m) * c), c = log2(e) / tau
};

__host__ __device__ inline size_t accept_ws_bytes(int R, int K, int T_cap) {
  return ((size_t)T_cap + (size_t)R * K) * sizeof(RowStats);
}

template <typename T>
__device__ __forceinline__ float ld1(const T *p) { return to_f32(__ldg(p)); }

template <typename T>
__global__ void __launch_bounds__(kAccThreads)
accept_stats_kernel(const T *__restrict__ target, const T *__restrict__ draft, int V, int R, int K,
                    int T_cap, const int32_t *__restrict__ verify_len,
                    const int32_t *__restrict__ q_offsets, float c, int greedy,
                    RowStats *__restrict__ stats) {
  const int b = blockIdx.x;
  const T *row;
  if (b < T_cap) {
    const int Tn = min(__ldg(q_offsets + R), T_cap);
    if (b >= Tn) return;
    row = target + (size_t)b * V;
  } else {
    if (greedy) return;
    const int i = b - T_cap, r = i / K, k = i % K;
    const int L = __ldg(verify_len + r);
    if (k >= L) return;
    row = draft + (size_t)i * V;
  }
  const int tid = threadIdx.x;
  float m = -INFINITY;
  double Z = 0.0;
  int amax = 0x7fffffff;
  const bool vec = ((reinterpret_cast<uintptr_t>(row) & 15) == 0) && (V % 8 == 0) &&
                   (sizeof(T) == 2 || (reinterpret_cast<uintptr_t>(row) & 31) == 0);
  auto consume = [&](const float (&x)[8], int base, int cnt) {
    float mx = -INFINITY;
    int ix = 0x7fffffff;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (e < cnt && x[e] > mx) { mx = x[e]; ix = base + e; }
    }
    if (mx > m) {
      if (!greedy && m != -INFINITY) Z *= exp2((double)(m - mx) * (double)c);
      m = mx;
      amax = ix;
    }
    if (!greedy && m != -INFINITY) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (e < cnt) s += exp2f((x[e] - m) * c);
      Z += (double)s;
    }
  };
  if (vec) {
    const int nv = V / 8;
    int v8 = tid;
    for (; v8 + 3 * kAccThreads < nv; v8 += 4 * kAccThreads) {
      float x[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u) load8(row + (size_t)(v8 + u * kAccThreads) * 8, x[u]);
#pragma unroll
      for (int u = 0; u < 4; ++u) consume(x[u], (v8 + u * kAccThreads) * 8, 8);
    }
    for (; v8 < nv; v8 += kAccThreads) {
      float x[8];
      load8(row + (size_t)v8 * 8, x);
      consume(x, v8 * 8, 8);
    }
  } else {
    for (int base = tid * 8; base < V; base += kAccThreads * 8) {
      float x[8];
      const int cnt = min(8, V - base);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = (e < cnt) ? ld1(row + base + e) : -INFINITY;
      consume(x, base, cnt);
    }
  }
  // block merge
  __shared__ float sm_m[kAccThreads / 32];
  __shared__ int sm_i[kAccThreads / 32];
  __shared__ double sm_z[kAccThreads / 32];
  const int lane = tid & 31, warp = tid >> 5;
  float wm = warp_max(m);
  int wi = (m == wm) ? amax : 0x7fffffff;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wi = min(wi, __shfl_xor_sync(0xffffffffu, wi, o));
  if (lane == 0) { sm_m[warp] = wm; sm_i[warp] = wi; }
  __syncthreads();
  float M = sm_m[0];
  for (int w = 1; w < kAccThreads / 32; ++w) M = fmaxf(M, sm_m[w]);
  int I = 0x7fffffff;
  for (int w = 0; w < kAccThreads / 32; ++w)
    if (sm_m[w] == M) I = min(I, sm_i[w]);
  double z = (!greedy && m != -INFINITY && M != -INFINITY) ? Z * exp2((double)(m - M) * (double)c)
                                                          : 0.0;
  z = warp_sum(z);
  if (lane == 0) sm_z[warp] = z;
  __syncthreads();
  if (tid == 0) {
    double Zt = 0.0;
    for (int w = 0; w < kAccThreads / 32; ++w) Zt += sm_z[w];
    if (!(M > -INFINITY && M < INFINITY)) raise_error(DSPARK_DERR_LOGITS);
    RowStats st;
    st.m = M;
    st.argmax = I;
    st.Z = Zt;
    stats[b] = st;
  }
}

template <typename T>
struct RowPair {
  const T *t;  // target row
  const T *d;  // draft row (residual only)
  float mt, md;
  double invZt, invZd;
  float c;
  bool residual;
  __device__ __forceinline__ double weight(float zt, float zd) const {
    const double pt = (double)exp2f((zt - mt) * c) * invZt;
    if (!residual) return pt;
    const double qd = (double)exp2f((zd - md) * c) * invZd;
    return fmax(0.0, pt - qd);
  }
};

// Sum of the weights of elements [base, base + 8) of the row pair (float64, in index order).
template <typename T>
__device__ __forceinline__ double weights8(const RowPair<T> &rp, int base, int V, double (&w)[8]) {
  double s = 0.0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int v = base + e;
    double x = 0.0;
    if (v < V) x = rp.weight(ld1(rp.t + v), rp.residual ? ld1(rp.d + v) : 0.f);
    w[e] = x;
    s += x;
  }
  return s;
}

__device__ __forceinline__ double block_sum_f64(double x, double *sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  x = warp_sum(x);
  if (lane == 0) sm[warp] = x;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < kAccThreads / 32; ++w) t += sm[w];
  __syncthreads();
  return t;
}

__device__ __forceinline__ double block_excl_scan_f64_acc(double x, double *sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sm[warp] = incl;
  __syncthreads();
  double off = 0.0;
  for (int w = 0; w < warp; ++w) off += sm[w];
  __syncthreads();
  return off + incl - x;
}

// Inverse-CDF draw over a row pair: smallest v with C(v) > u * C(V-1).
template <typename T>
__device__ int draw_inverse_cdf(const RowPair<T> &rp, int V, float u, double *chunk_sum,
                                double *sm) {
  __shared__ int s_pick;
  const int tid = threadIdx.x;
  const int nch = (V + kAccChunk - 1) / kAccChunk;
  for (int ch = 0; ch < nch; ++ch) {
    double w[8];
    const double s = weights8(rp, ch * kAccChunk + tid * 8, V, w);
    const double tot = block_sum_f64(s, sm);
    if (tid == 0) chunk_sum[ch] = tot;
  }
  __syncthreads();
  if (tid == 0) {
    double Z = 0.0;
    for (int ch = 0; ch < nch; ++ch) Z += chunk_sum[ch];
    const double thr = (double)u * Z;
    double cum = 0.0;
    int pick = -1;
    double base = 0.0;
    for (int ch = 0; ch < nch; ++ch) {
      if (chunk_sum[ch] > 0.0 && cum + chunk_sum[ch] > thr) { pick = ch; base = cum; break; }
      cum += chunk_sum[ch];
    }
    if (pick < 0) {  // rounding put the threshold past the end: last chunk with mass
      for (int ch = nch - 1; ch >= 0; --ch)
        if (chunk_sum[ch] > 0.0) { pick = ch; break; }
      base = -1.0;   // marker: take the last positive element of that chunk
    }
    chunk_sum[nch] = thr;
    chunk_sum[nch + 1] = base;
    s_pick = pick;
  }
  __syncthreads();
  const int pick = s_pick;
  if (pick < 0) return -1;  // no mass anywhere
  const double thr = chunk_sum[nch], base = chunk_sum[nch + 1];
  double w[8];
  const int b0 = pick * kAccChunk + tid * 8;
  const double s = weights8(rp, b0, V, w);
  const double ex = block_excl_scan_f64_acc(s, sm);
  __shared__ int s_found, s_lastpos;
  if (tid == 0) { s_found = 0x7fffffff; s_lastpos = -1; }
  __syncthreads();
  int found = 0x7fffffff, lastpos = -1;
  double C = base + ex;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    C += w[e];
    if (w[e] > 0.0) {
      lastpos = b0 + e;
      if (base >= 0.0 && C > thr && found == 0x7fffffff) found = b0 + e;
    }
  }
  if (found != 0x7fffffff) atomicMin(&s_found, found);
  if (lastpos >= 0) atomicMax(&s_lastpos, lastpos);
  __syncthreads();
  return (s_found != 0x7fffffff) ? s_found : s_lastpos;
}

template <typename T>
__global__ void __launch_bounds__(kAccThreads)
accept_finalize_kernel(const T *__restrict__ target, const T *__restrict__ draft, int V, int R,
                       int K, int T_cap, const int32_t *__restrict__ draft_tokens,
                       const int32_t *__restrict__ verify_len,
                       const int32_t *__restrict__ q_offsets, const float *__restrict__ u_acc,
                       const float *__restrict__ u_res, float c, int greedy,
                       const RowStats *__restrict__ stats, int32_t *__restrict__ accepted_len,
                       int32_t *__restrict__ out_tokens, int32_t *__restrict__ n_out) {
  extern __shared__ double chunk_sum[];  // [nch + 2]
  __shared__ double sm[kAccThreads / 32];
  __shared__ int s_a, s_ok;
  const int r = blockIdx.x, tid = threadIdx.x;
  const int L = __ldg(verify_len + r);
  const int t0 = __ldg(q_offsets + r), t1 = __ldg(q_offsets + r + 1);
  if (tid == 0) {
    int ok = 1;
    if (L < 0 || L > K) { raise_error(DSPARK_DERR_VERIFY_LEN); ok = 0; }
    else if (t1 - t0 != L + 1 || t0 < 0 || t1 > T_cap) { raise_error(DSPARK_DERR_OFFSETS); ok = 0; }
    int a = 0;
    if (ok) {
      for (; a < L; ++a) {
        const int x = __ldg(draft_tokens + (size_t)r * K + a);
        if (x < 0 || x >= V) { raise_error(DSPARK_DERR_TOKEN); break; }
        const RowStats st = stats[t0 + a];
        if (greedy) {
          if (x != st.argmax) break;
        } else {
          const RowStats sd = stats[T_cap + r * K + a];
          const float zt = ld1(target + (size_t)(t0 + a) * V + x);
          const float zd = ld1(draft + ((size_t)r * K + a) * V + x);
          const double p = (double)exp2f((zt - st.m) * c) / st.Z;
          const double q = (double)exp2f((zd - sd.m) * c) / sd.Z;
          const double ratio = (q > 0.0) ? p / q : (p > 0.0 ? INFINITY : 0.0);
          const double thr = fmin(1.0, ratio);
          if (!((double)__ldg(u_acc + (size_t)r * K + a) < thr)) break;
        }
      }
    }
    s_a = a;
    s_ok = ok;
  }
  __syncthreads();
  const int a = s_a;
  if (!s_ok) {
    for (int j = tid; j <= K; j += kAccThreads) out_tokens[(size_t)r * (K + 1) + j] = -1;
    if (tid == 0) { accepted_len[r] = 0; n_out[r] = 0; }
    return;
  }
  int corr;
  if (greedy) {
    corr = stats[t0 + a].argmax;
  } else {
    RowPair<T> rp;
    const RowStats st = stats[t0 + a];
    rp.t = target + (size_t)(t0 + a) * V;
    rp.mt = st.m;
    rp.invZt = 1.0 / st.Z;
    rp.c = c;
    rp.residual = a < L;
    if (rp.residual) {
      const RowStats sd = stats[T_cap + r * K + a];
      rp.d = draft + ((size_t)r * K + a) * V;
      rp.md = sd.m;
      rp.invZd = 1.0 / sd.Z;
    } else {
      rp.d = nullptr;
      rp.md = 0.f;
      rp.invZd = 0.0;
    }
    const float u = __ldg(u_res + (size_t)r * (K + 1) + a);
    corr = draw_inverse_cdf(rp, V, u, chunk_sum, sm);
    if (corr < 0 && rp.residual) {  // residual empty in floating point: draw from p instead
      rp.residual = false;
      __syncthreads();
      corr = draw_inverse_cdf(rp, V, u, chunk_sum, sm);
    }
  }
  for (int j = tid; j <= K; j += kAccThreads) {
    int v = -1;
    if (j < a) v = __ldg(draft_tokens + (size_t)r * K + j);
    else if (j == a) v = corr;
    out_tokens[(size_t)r * (K + 1) + j] = v;
  }
  if (tid == 0) { accepted_len[r] = a; n_out[r] = a + 1; }
}

}  // namespace dspark
