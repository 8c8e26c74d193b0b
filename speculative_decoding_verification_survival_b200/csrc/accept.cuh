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
//                          merge -> (m, Z = sum exp((z - m)/tau); greedy: argmax, lowest index).
//                          The exponent (z - m) log2(e) / tau is formed with log2(e) / tau split
//                          into two floats, so that the rounding of that constant (the same in
//                          every term, hence not averaged out) does not bias Z.
//   accept_finalize_kernel one cluster of `ncl` CTAs per request: all draft positions tested at
//                          once, the accepted prefix ends at the first failure; then the
//                          correction / bonus draw by inverse CDF over one row pair: pass 1
//                          sums the weights per 2048-element chunk (float64), each CTA of the
//                          cluster over its own run of chunks; the chunk sums are gathered
//                          through distributed shared memory and the threshold u * Z picks the
//                          chunk; pass 2 re-reads that chunk and scans it, in the CTA owning it.
//                          For bf16 rows pass 1 forms the exponent arguments two at a time in
//                          packed floats straight from the raw 16-byte groups (the same bits as
//                          the scalar weights), in few enough registers for four CTAs per SM.
#pragma once

#include "common.cuh"
#include "ptx_sm100.cuh"

namespace dspark {

constexpr int kAccThreads = 256;
constexpr int kAccWarps = kAccThreads / 32;
constexpr int kAccChunk = kAccThreads * 8;  // elements per chunk of the inverse-CDF scan
// CTAs of the bf16 sampled draw resident per SM (its registers are bounded for that): the host
// sizes the draw's clusters so that the whole grid fits at once where it can
constexpr int kAccFinBlocks = 4;

struct RowStats {
  float m;      // row maximum
  int argmax;   // lowest index attaining m (greedy verification only)
  double Z;     // sum_v exp2((z_v - m) * c), c = log2(e) / tau
};

__host__ __device__ inline size_t accept_ws_bytes(int R, int K, int T_cap) {
  return ((size_t)T_cap + (size_t)R * K) * sizeof(RowStats);
}

// Dynamic shared memory of the finalize kernel: per-warp partial sums of every chunk, this
// CTA's chunk sums, the gathered chunk sums of the whole row and two scalars.
__host__ __device__ inline size_t accept_finalize_smem(int V) {
  const size_t nch = ((size_t)V + kAccChunk - 1) / kAccChunk;
  return ((size_t)kAccWarps * nch + 2 * nch + 2) * sizeof(double);
}

// The run of chunks [chunk_lo(k), chunk_lo(k + 1)) that CTA k of a cluster of ncl sums.
__host__ __device__ inline int chunk_lo(int nch, int k, int ncl) {
  return (int)((long long)nch * k / ncl);
}
__device__ __forceinline__ int chunk_owner(int nch, int ch, int ncl) {
  int k = 0;
  while (k + 1 < ncl && chunk_lo(nch, k + 1, ncl) <= ch) ++k;
  return k;
}

template <typename T>
__device__ __forceinline__ float ld1(const T *p) { return to_f32(__ldg(p)); }

// 2^x with the SFU (relative error about 2^-22; results below 2^-126 flush to zero).
__device__ __forceinline__ float exp2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The scale c = log2(e) / tau as an unevaluated float sum hi + lo (lo = c - hi rounded), and in
// float64 for the few per-request evaluations done at that precision.
struct ExpScale {
  float hi, lo;  // hi = c rounded toward zero, lo = c - hi rounded (> 0 for sampled rows)
  double d;
  // d * c in float32 without the systematic error of a rounded c.  d = -inf (a masked logit,
  // or padding) is first clamped to a large finite negative number, whose 2^x is still 0:
  // -inf * lo would give NaN when lo is 0 or has the opposite sign of hi.
  __device__ __forceinline__ float mul(float d_) const {
    d_ = fmaxf(d_, -1e30f);
    return fmaf(d_, lo, d_ * hi);
  }
};

// Eight consecutive logits as raw bits (one 16-byte load for bf16, two for f32), so that a
// step's loads are all issued before any of them is converted.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> { uint4 a; };
template <> struct Raw8<float> { float4 a, b; };
__device__ __forceinline__ void load_raw8(const __nv_bfloat16 *p, Raw8<__nv_bfloat16> &r) {
  r.a = __ldg(reinterpret_cast<const uint4 *>(p));
}
__device__ __forceinline__ void load_raw8(const float *p, Raw8<float> &r) {
  r.a = __ldg(reinterpret_cast<const float4 *>(p));
  r.b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
}
__device__ __forceinline__ void cvt8(const Raw8<__nv_bfloat16> &r, float (&v)[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r.a);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void cvt8(const Raw8<float> &r, float (&v)[8]) {
  v[0] = r.a.x; v[1] = r.a.y; v[2] = r.a.z; v[3] = r.a.w;
  v[4] = r.b.x; v[5] = r.b.y; v[6] = r.b.z; v[7] = r.b.w;
}

// bf16 logits, sampled verification: this thread's share of one row (16-byte groups g = tid,
// tid + 256, ...) as a running maximum m and Z = sum 2^((z - m) c), with as few instructions per
// element as the arithmetic allows (the pass is issue-bound before it is memory-bound on this
// part).  A pair of groups' maximum comes from packed bf16 pairs and Z is rescaled only when it
// rises; per pair of elements the bf16 -> float conversion is a shift and a mask, then
// d = z - m (exact), d hi + d lo and the running sums run as packed float pairs, and ex2 per
// element: the even and the odd elements of a pair of groups each go to one float partial (8
// terms each), the partials summed in float64.  Loads run one step of four groups ahead (64
// bytes per thread in flight; four CTAs per SM, so 64 KB per SM), in two register sets used in
// turn.
using ptx::f2_add;
using ptx::f2_fma;
using ptx::f2_mul;
using ptx::f2_pack;
using ptx::f2_unpack;
__device__ __forceinline__ uint64_t f2_pack_dup(float x) { return ptx::f2_pack(x, x); }
__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  const __nv_bfloat162 r = __hmax2(*reinterpret_cast<const __nv_bfloat162 *>(&a),
                                   *reinterpret_cast<const __nv_bfloat162 *>(&b));
  return *reinterpret_cast<const uint32_t *>(&r);
}
__device__ __forceinline__ void stats_bf16_sampled(const uint4 *__restrict__ rowv, int nv,
                                                   const ExpScale &c, float &m, double &Z) {
  const int tid = threadIdx.x;
  const uint64_t hi2 = f2_pack_dup(c.hi), lo2 = f2_pack_dup(c.lo);
  // a pair of groups: its maximum, the rescale if it rises, its 16 terms
  auto step = [&](const uint4 &a, const uint4 &b) {
    const uint32_t p = bmax2(bmax2(bmax2(a.x, a.y), bmax2(a.z, a.w)),
                             bmax2(bmax2(b.x, b.y), bmax2(b.z, b.w)));
    const float gm = fmaxf(bf16_lo_f(p), bf16_hi_f(p));
    if (gm > m) {
      if (m != -INFINITY) Z *= exp2(((double)m - (double)gm) * c.d);
      m = gm;
    }
    if (m == -INFINITY) return;  // every value so far is -inf
    const uint64_t nm2 = f2_pack_dup(-m);
    uint64_t s2 = 0;  // (even, odd) partial sums: two float zeros
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint64_t d2 = f2_add(f2_pack(bf16_lo_f(w[i]), bf16_hi_f(w[i])), nm2);
      const uint64_t e2 = f2_fma(d2, lo2, f2_mul(d2, hi2));
      float e0, e1;
      f2_unpack(e2, e0, e1);
      s2 = f2_add(s2, f2_pack(exp2_sfu(e0), exp2_sfu(e1)));
    }
    float s0, s1;
    f2_unpack(s2, s0, s1);
    Z += (double)(s0 + s1);
  };
  // a step is two pairs of groups per thread (four 16-byte loads); the next step's loads are
  // issued before this step's values are used, in two register sets used in turn
  constexpr int kStep = 4 * kAccThreads;  // groups per step of the whole CTA
  const int steps = nv / kStep;           // steps in which every thread has all four groups
  uint4 x0[4], x1[4];
  auto load = [&](uint4 (&x)[4], int st) {
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = __ldg(rowv + st * kStep + u * kAccThreads + tid);
  };
  if (steps > 0) load(x0, 0);
  int s = 0;
  for (; s + 1 < steps; s += 2) {
    load(x1, s + 1);
    step(x0[0], x0[1]);
    step(x0[2], x0[3]);
    if (s + 2 < steps) load(x0, s + 2);
    step(x1[0], x1[1]);
    step(x1[2], x1[3]);
  }
  if (s < steps) {
    step(x0[0], x0[1]);
    step(x0[2], x0[3]);
  }
  const int done_groups = steps * kStep;
  // the rest: single groups (the other of a pair is all -inf)
  const uint4 ninf = make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
  for (int g = done_groups + tid; g < nv; g += kAccThreads) step(__ldg(rowv + g), ninf);
}

// One CTA per scheduled logit row: one streaming pass with 16-byte loads, 32 elements per thread
// and step; the running maximum rescales the float64 sum only when it rises.  GREEDY rows only
// need the maximum and its lowest index.  Five CTAs per SM (registers capped to fit), so that a
// 64-request step's 704 rows run as one wave of 740 rather than 1.2 waves of 592.
template <typename T, bool GREEDY>
__global__ void __launch_bounds__(kAccThreads, (sizeof(T) == 2 && !GREEDY) ? 4 : 5)
accept_stats_kernel(const T *__restrict__ target, const T *__restrict__ draft, int V, int R, int K,
                    int T_cap, const int32_t *__restrict__ verify_len,
                    const int32_t *__restrict__ q_offsets, ExpScale c,
                    RowStats *__restrict__ stats) {
  const int b = blockIdx.x;
  const T *row;
  if (b < T_cap) {
    const int Tn = min(__ldg(q_offsets + R), T_cap);
    if (b >= Tn) return;
    row = target + (size_t)b * V;
  } else {
    if (GREEDY) return;
    const int i = b - T_cap, r = i / K, k = i % K;
    const int L = __ldg(verify_len + r);
    if (k >= L) return;
    row = draft + (size_t)i * V;
  }
  const int tid = threadIdx.x;
  float m = -INFINITY;
  double Z = 0.0;
  int amax = 0x7fffffff;
  // x[u][e] is element base[u] + e; groups are visited in index order
  auto consume = [&](const auto &x, const auto &base) {
    constexpr int NU = sizeof(base) / sizeof(base[0]);
    if (GREEDY) {
#pragma unroll
      for (int u = 0; u < NU; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (x[u][e] > m) { m = x[u][e]; amax = base[u] + e; }
    } else {
      float lm = -INFINITY;
#pragma unroll
      for (int u = 0; u < NU; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e) lm = fmaxf(lm, x[u][e]);
      if (lm > m) {
        if (m != -INFINITY) Z *= exp2(((double)m - (double)lm) * c.d);
        m = lm;
      }
      if (m != -INFINITY) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int u = 0; u < NU; ++u)
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            s0 += exp2_sfu(c.mul(x[u][e] - m));
            s1 += exp2_sfu(c.mul(x[u][e + 1] - m));
          }
        Z += (double)(s0 + s1);
      }
    }
  };
  const bool vec = ((reinterpret_cast<uintptr_t>(row) & 15) == 0) && (V % 8 == 0) &&
                   (sizeof(T) == 2 || (reinterpret_cast<uintptr_t>(row) & 31) == 0);
  bool done = false;
  if constexpr (sizeof(T) == 2 && !GREEDY) {
    if (vec) {
      stats_bf16_sampled(reinterpret_cast<const uint4 *>(row), V / 8, c, m, Z);
      done = true;
    }
  }
  if (done) {
  } else if (vec) {
    // the next step's loads are issued before this step's values are used, so every thread
    // keeps loads in flight while it computes
    constexpr int kU = 2;
    const int nv = V / 8;
    constexpr int kStep = kU * kAccThreads;
    Raw8<T> cur[kU], nxt[kU];
    auto issue = [&](Raw8<T>(&r)[kU], int v8) {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int g = v8 + u * kAccThreads;
        load_raw8(row + (size_t)(g < nv ? g : 0) * 8, r[u]);  // in bounds; masked below
      }
    };
    if (tid < nv) issue(cur, tid);
    for (int v8 = tid; v8 < nv; v8 += kStep) {
      if (v8 + kStep < nv) issue(nxt, v8 + kStep);
      float x[kU][8];
      int base[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int g = v8 + u * kAccThreads;
        base[u] = g * 8;
        if (g < nv) {
          cvt8(cur[u], x[u]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) x[u][e] = -INFINITY;
        }
      }
      consume(x, base);
#pragma unroll
      for (int u = 0; u < kU; ++u) cur[u] = nxt[u];
    }
  } else {
    for (int b0 = tid * 8; b0 < V; b0 += 4 * kAccThreads * 8) {
      float x[4][8];
      int base[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        base[u] = b0 + u * kAccThreads * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          x[u][e] = (base[u] + e < V) ? ld1(row + base[u] + e) : -INFINITY;
      }
      consume(x, base);
    }
  }
  // block merge
  __shared__ float sm_m[kAccWarps];
  __shared__ int sm_i[kAccWarps];
  __shared__ double sm_z[kAccWarps];
  const int lane = tid & 31, warp = tid >> 5;
  const float wm = warp_max(m);
  int wi = (m == wm) ? amax : 0x7fffffff;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wi = min(wi, __shfl_xor_sync(0xffffffffu, wi, o));
  if (lane == 0) { sm_m[warp] = wm; sm_i[warp] = wi; }
  __syncthreads();
  float M = sm_m[0];
  for (int w = 1; w < kAccWarps; ++w) M = fmaxf(M, sm_m[w]);
  int I = 0x7fffffff;
  for (int w = 0; w < kAccWarps; ++w)
    if (sm_m[w] == M) I = min(I, sm_i[w]);
  double z = (!GREEDY && m != -INFINITY && M != -INFINITY)
                 ? Z * exp2(((double)m - (double)M) * c.d)
                 : 0.0;
  z = warp_sum(z);
  if (lane == 0) sm_z[warp] = z;
  __syncthreads();
  if (tid == 0) {
    double Zt = 0.0;
    for (int w = 0; w < kAccWarps; ++w) Zt += sm_z[w];
    if (!(M > -INFINITY && M < INFINITY)) raise_error(DSPARK_DERR_LOGITS);
    RowStats st;
    st.m = M;
    st.argmax = I;
    st.Z = Zt;
    stats[b] = st;
  }
}

// Per-element weights are float32 (their exp2 is float32 anyway, relative error ~2^-22); the
// sums over the vocabulary are float64 (groups of 8 summed in float32 first).  Float64 is a slow
// pipe on this part, so it is kept out of the per-element work.
template <typename T>
struct RowPair {
  const T *t;  // target row
  const T *d;  // draft row (residual only)
  float mt, md;
  float invZt, invZd;
  ExpScale c;
  bool residual, vec;
  // Both probabilities are rounded before the difference (no fused multiply-add): equal rows
  // with equal statistics then give exactly 0, so an empty residual is seen as empty.
  __device__ __forceinline__ float weight(float zt, float zd) const {
    const float pt = __fmul_rn(exp2_sfu(c.mul(zt - mt)), invZt);
    if (!residual) return pt;
    return fmaxf(0.f, pt - __fmul_rn(exp2_sfu(c.mul(zd - md)), invZd));
  }
};

// Logits [base, base + 8) of the row pair, element by element (any alignment; -inf past V).
template <typename T>
__device__ __forceinline__ void load_pair8_scalar(const RowPair<T> &rp, int base, int V,
                                                  float (&xt)[8], float (&xd)[8]) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const bool in = base + e < V;
    xt[e] = in ? ld1(rp.t + base + e) : -INFINITY;
    xd[e] = (in && rp.residual) ? ld1(rp.d + base + e) : 0.f;
  }
}

// Weights of elements [base, base + 8) (0 past the end) and their sum in index order.
template <typename T>
__device__ __forceinline__ double weights8(const RowPair<T> &rp, int base, int V,
                                           const float (&xt)[8], const float (&xd)[8],
                                           float (&w)[8]) {
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    w[e] = (base + e < V) ? rp.weight(xt[e], xd[e]) : 0.f;
    s += w[e];
  }
  return (double)s;
}

// The same sum for eight bf16 logits of a row pair taken straight from their raw 16-byte groups,
// the exponent arguments two elements per packed-float operation.  Bit for bit what weights8
// gives: the packed add, multiply and fused multiply-add round each lane as the scalar
// operations do, x - y is x + (-y), and a -inf logit gives weight 0 without the clamp of
// ExpScale::mul (c's low part is > 0 for sampled rows).  The products by 1/Z and the difference
// p - q stay scalar with explicit rounding, so that nothing fuses them into one rounding (an
// empty residual must stay exactly empty); the eight weights are added in index order.
struct PackedPairConsts {
  uint64_t hi2, lo2, nmt2, nmd2;
};
template <typename T>
__device__ __forceinline__ PackedPairConsts packed_consts(const RowPair<T> &rp) {
  PackedPairConsts k;
  k.hi2 = ptx::f2_pack(rp.c.hi, rp.c.hi);
  k.lo2 = ptx::f2_pack(rp.c.lo, rp.c.lo);
  k.nmt2 = ptx::f2_pack(-rp.mt, -rp.mt);
  k.nmd2 = ptx::f2_pack(-rp.md, -rp.md);
  return k;
}
template <typename T>
__device__ __forceinline__ float weights8_bf16_packed(const RowPair<T> &rp,
                                                      const PackedPairConsts &k,
                                                      const uint4 &rt, const uint4 &rd) {
  const uint32_t wt[4] = {rt.x, rt.y, rt.z, rt.w};
  const uint32_t wd[4] = {rd.x, rd.y, rd.z, rd.w};
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint64_t dt = ptx::f2_add(ptx::f2_pack(__uint_as_float(wt[i] << 16),
                                                 __uint_as_float(wt[i] & 0xffff0000u)), k.nmt2);
    float e0, e1;
    ptx::f2_unpack(ptx::f2_fma(dt, k.lo2, ptx::f2_mul(dt, k.hi2)), e0, e1);
    float w0 = __fmul_rn(exp2_sfu(e0), rp.invZt), w1 = __fmul_rn(exp2_sfu(e1), rp.invZt);
    if (rp.residual) {
      const uint64_t dd = ptx::f2_add(ptx::f2_pack(__uint_as_float(wd[i] << 16),
                                                   __uint_as_float(wd[i] & 0xffff0000u)), k.nmd2);
      float g0, g1;
      ptx::f2_unpack(ptx::f2_fma(dd, k.lo2, ptx::f2_mul(dd, k.hi2)), g0, g1);
      w0 = fmaxf(0.f, __fsub_rn(w0, __fmul_rn(exp2_sfu(g0), rp.invZd)));
      w1 = fmaxf(0.f, __fsub_rn(w1, __fmul_rn(exp2_sfu(g1), rp.invZd)));
    }
    s += w0;
    s += w1;
  }
  return s;
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

// Inverse-CDF draw over a row pair: smallest v with C(v) > u * C(V-1).  Pass 1 streams this
// CTA's chunks of the row (four chunks per step with every load of the step issued before any
// is used, per-warp partial sums in shared memory, no barrier inside the loop); the chunk sums of
// all `ncl` CTAs of the cluster are gathered in index order, the threshold picks a chunk; pass 2
// re-reads that chunk and scans it in index order, in the CTA that owns it.  Returns the token,
// -1 in every CTA when the row has no mass, -2 in the CTAs that do not own the picked chunk.
// Every CTA of the cluster calls it with the same row pair and u.
template <typename T>
__device__ int draw_inverse_cdf(const RowPair<T> &rp, int V, float u, double *fsm, double *sm,
                                int rank, int ncl) {
  __shared__ int s_pick;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nch = (V + kAccChunk - 1) / kAccChunk;
  double *part = fsm;                         // [kAccWarps][nch]
  double *chunk_sum = fsm + kAccWarps * nch;  // [nch], this CTA's chunks
  double *all_sum = chunk_sum + nch;          // [nch + 2], every chunk, then thr and base
  const int lo = chunk_lo(nch, rank, ncl), hi = chunk_lo(nch, rank + 1, ncl);
  constexpr int kU = 4;
  if constexpr (sizeof(T) == 2) {
    if (rp.vec) {  // bf16, V % 8 == 0, rows aligned: packed weights from the raw groups
      const PackedPairConsts kc = packed_consts(rp);
      for (int ch0 = lo; ch0 < hi; ch0 += kU) {
        uint4 rt[kU], rd[kU];
#pragma unroll
        for (int k = 0; k < kU; ++k) {
          const int base = (ch0 + k) * kAccChunk + tid * 8;
          const int b = base < V ? base : 0;  // in-bounds address; a group past V weighs 0
          rt[k] = __ldg(reinterpret_cast<const uint4 *>(rp.t + b));
          rd[k] = rp.residual ? __ldg(reinterpret_cast<const uint4 *>(rp.d + b)) : rt[k];
        }
#pragma unroll
        for (int k = 0; k < kU; ++k) {
          if (ch0 + k < hi) {
            const int base = (ch0 + k) * kAccChunk + tid * 8;
            const float sf = base < V ? weights8_bf16_packed(rp, kc, rt[k], rd[k]) : 0.f;
            const double sd = warp_sum((double)sf);
            if (lane == 0) part[warp * nch + ch0 + k] = sd;
          }
        }
      }
    }
  }
  for (int ch0 = lo; ch0 < hi && !(sizeof(T) == 2 && rp.vec); ch0 += kU) {
    float xt[kU][8], xd[kU][8];
    if (rp.vec) {  // V % 8 == 0, rows aligned: a group is either wholly inside or past the end
      Raw8<T> rt[kU], rd[kU];
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        const int base = (ch0 + k) * kAccChunk + tid * 8;
        const int b = base < V ? base : 0;  // in-bounds address; values past V are masked below
        load_raw8(rp.t + b, rt[k]);
        if (rp.residual) load_raw8(rp.d + b, rd[k]);
      }
#pragma unroll
      for (int k = 0; k < kU; ++k) {
        cvt8(rt[k], xt[k]);
        if (rp.residual) {
          cvt8(rd[k], xd[k]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) xd[k][e] = 0.f;
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < kU; ++k)
        load_pair8_scalar(rp, (ch0 + k) * kAccChunk + tid * 8, V, xt[k], xd[k]);
    }
#pragma unroll
    for (int k = 0; k < kU; ++k) {
      if (ch0 + k < hi) {
        float w[8];
        const double s = warp_sum(weights8(rp, (ch0 + k) * kAccChunk + tid * 8, V, xt[k], xd[k], w));
        if (lane == 0) part[warp * nch + ch0 + k] = s;
      }
    }
  }
  __syncthreads();
  for (int ch = lo + tid; ch < hi; ch += kAccThreads) {
    double t = 0.0;
    for (int w = 0; w < kAccWarps; ++w) t += part[w * nch + ch];
    chunk_sum[ch] = t;
  }
  if (ncl > 1) {
    ptx::cluster_sync();  // every CTA's chunk sums are written
    for (int ch = tid; ch < nch; ch += kAccThreads)
      all_sum[ch] = ptx::ld_dsmem_f64(chunk_sum + ch, (uint32_t)chunk_owner(nch, ch, ncl));
    ptx::cluster_sync();  // every CTA has read them: shared memory may be rewritten, CTAs exit
  } else {
    __syncthreads();
    for (int ch = tid; ch < nch; ch += kAccThreads) all_sum[ch] = chunk_sum[ch];
  }
  __syncthreads();
  if (tid == 0) {
    double Z = 0.0;
    for (int ch = 0; ch < nch; ++ch) Z += all_sum[ch];
    const double thr = (double)u * Z;
    double cum = 0.0;
    int pick = -1;
    double base = 0.0;
    for (int ch = 0; ch < nch; ++ch) {
      if (all_sum[ch] > 0.0 && cum + all_sum[ch] > thr) { pick = ch; base = cum; break; }
      cum += all_sum[ch];
    }
    if (pick < 0) {  // rounding put the threshold past the end: last chunk with mass
      for (int ch = nch - 1; ch >= 0; --ch)
        if (all_sum[ch] > 0.0) { pick = ch; break; }
      base = -1.0;   // marker: take the last positive element of that chunk
    }
    all_sum[nch] = thr;
    all_sum[nch + 1] = base;
    s_pick = pick;
  }
  __syncthreads();
  const int pick = s_pick;
  if (pick < 0) return -1;  // no mass anywhere
  if (chunk_owner(nch, pick, ncl) != rank) return -2;
  const double thr = all_sum[nch], base = all_sum[nch + 1];
  const int b0 = pick * kAccChunk + tid * 8;
  float xt[8], xd[8];
  load_pair8_scalar(rp, b0, V, xt, xd);
  float w[8];
  const double s = weights8(rp, b0, V, xt, xd, w);
  const double ex = block_excl_scan_f64_acc(s, sm);
  __shared__ int s_found, s_lastpos;
  if (tid == 0) { s_found = 0x7fffffff; s_lastpos = -1; }
  __syncthreads();
  int found = 0x7fffffff, lastpos = -1;
  double C = base + ex;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    C += (double)w[e];
    if (w[e] > 0.f) {
      lastpos = b0 + e;
      if (base >= 0.0 && C > thr && found == 0x7fffffff) found = b0 + e;
    }
  }
  if (found != 0x7fffffff) atomicMin(&s_found, found);
  if (lastpos >= 0) atomicMax(&s_lastpos, lastpos);
  __syncthreads();
  // the chunk had mass in pass 1 and pass 2 recomputes the same weights, so a position exists;
  // were it missing, -3 keeps the retry decision (-1) the same in every CTA of the cluster
  return (s_found != 0x7fffffff) ? s_found : (s_lastpos >= 0 ? s_lastpos : -3);
}

// One cluster of ncl CTAs per request (launched with cluster dimension ncl; ncl = 1 without
// clusters, always so for GREEDY): every CTA takes every draft position's test at once (one
// thread each) and finds the accepted prefix ending at the first failure; the CTAs then share
// the correction / bonus draw.  CTA 0 writes the outputs except a drawn token, which the CTA
// owning its chunk writes.
template <typename T, bool GREEDY>
__global__ void __launch_bounds__(kAccThreads, (sizeof(T) == 2 && !GREEDY) ? kAccFinBlocks : 2)
accept_finalize_kernel(const T *__restrict__ target, const T *__restrict__ draft, int V, int R,
                       int K, int T_cap, const int32_t *__restrict__ draft_tokens,
                       const int32_t *__restrict__ verify_len,
                       const int32_t *__restrict__ q_offsets, const float *__restrict__ u_acc,
                       const float *__restrict__ u_res, ExpScale c,
                       const RowStats *__restrict__ stats, int32_t *__restrict__ accepted_len,
                       int32_t *__restrict__ out_tokens, int32_t *__restrict__ n_out, int ncl) {
  extern __shared__ double fsm[];
  __shared__ double sm[kAccWarps];
  __shared__ int s_fail;
  const int r = blockIdx.x / ncl, tid = threadIdx.x;
  const int rank = ncl > 1 ? (int)ptx::cluster_ctarank() : 0;
  const bool lead = rank == 0;
  const int L = __ldg(verify_len + r);
  const int t0 = __ldg(q_offsets + r), t1 = __ldg(q_offsets + r + 1);
  const bool len_ok = L >= 0 && L <= K;
  const bool ok = len_ok && t1 - t0 == L + 1 && t0 >= 0 && t1 <= T_cap;
  if (tid == 0) {
    if (lead && !len_ok) raise_error(DSPARK_DERR_VERIFY_LEN);
    else if (lead && !ok) raise_error(DSPARK_DERR_OFFSETS);
    s_fail = ok ? L : 0;
  }
  __syncthreads();
  if (!ok) {  // the same in every CTA of the cluster: none reaches a cluster barrier
    if (lead) {
      for (int j = tid; j <= K; j += kAccThreads) out_tokens[(size_t)r * (K + 1) + j] = -1;
      if (tid == 0) { accepted_len[r] = 0; n_out[r] = 0; }
    }
    return;
  }
  bool bad = false;
  if (tid < L) {
    const int x = __ldg(draft_tokens + (size_t)r * K + tid);
    bad = x < 0 || x >= V;
    bool fail = bad;
    if (!bad) {
      const RowStats st = stats[t0 + tid];
      if (GREEDY) {
        fail = x != st.argmax;
      } else {
        const RowStats sd = stats[T_cap + r * K + tid];
        const float zt = ld1(target + (size_t)(t0 + tid) * V + x);
        const float zd = ld1(draft + ((size_t)r * K + tid) * V + x);
        // p(x) and q(x) in float64: a draft token far below its row's maximum has an exponent
        // of 30-40 whose float32 evaluation would be off by more than the 1e-6 decision window
        const double p = exp2(((double)zt - (double)st.m) * c.d) / st.Z;
        const double q = exp2(((double)zd - (double)sd.m) * c.d) / sd.Z;
        const double ratio = (q > 0.0) ? p / q : (p > 0.0 ? INFINITY : 0.0);
        fail = !((double)__ldg(u_acc + (size_t)r * K + tid) < fmin(1.0, ratio));
      }
    }
    if (fail) atomicMin(&s_fail, tid);
  }
  __syncthreads();
  const int a = s_fail;
  if (lead && tid == a && bad) raise_error(DSPARK_DERR_TOKEN);  // the token the chain stopped at
  int corr;
  if (GREEDY) {
    corr = stats[t0 + a].argmax;
  } else {
    RowPair<T> rp;
    const RowStats st = stats[t0 + a];
    rp.t = target + (size_t)(t0 + a) * V;
    rp.mt = st.m;
    rp.invZt = (float)(1.0 / st.Z);
    rp.c = c;
    rp.residual = a < L;
    if (rp.residual) {
      const RowStats sd = stats[T_cap + r * K + a];
      rp.d = draft + ((size_t)r * K + a) * V;
      rp.md = sd.m;
      rp.invZd = (float)(1.0 / sd.Z);
    } else {
      rp.d = nullptr;
      rp.md = 0.f;
      rp.invZd = 0.f;
    }
    const size_t align = sizeof(T) == 2 ? 15 : 31;
    rp.vec = (V % 8 == 0) && ((reinterpret_cast<uintptr_t>(rp.t) & align) == 0) &&
             (!rp.residual || (reinterpret_cast<uintptr_t>(rp.d) & align) == 0);
    const float u = __ldg(u_res + (size_t)r * (K + 1) + a);
    corr = draw_inverse_cdf(rp, V, u, fsm, sm, rank, ncl);
    if (corr == -1 && rp.residual) {  // residual empty in floating point: draw from p instead
      rp.residual = false;
      __syncthreads();
      corr = draw_inverse_cdf(rp, V, u, fsm, sm, rank, ncl);
    }
  }
  // corr: the token in the CTA that drew it, -1 in every CTA when nothing could be drawn,
  // -2 in the other CTAs
  if ((corr >= 0 || corr == -3) && tid == 0) out_tokens[(size_t)r * (K + 1) + a] = max(corr, -1);
  if (lead) {
    for (int j = tid; j <= K; j += kAccThreads) {
      if (j < a) out_tokens[(size_t)r * (K + 1) + j] = __ldg(draft_tokens + (size_t)r * K + j);
      else if (j > a || corr == -1) out_tokens[(size_t)r * (K + 1) + j] = -1;
    }
    if (tid == 0) { accepted_len[r] = a; n_out[r] = a + 1; }
  }
}

}  // namespace dspark
