// Synthetic Markov-head draft step (cost measurement of the sequential part of the drafter).
//
// "刚融完500亿…专治AI“嘴慢”" section "1. 半自回归生成": a parallel backbone produces the whole draft
// block; a light sequential module injects the prefix token by token, one form being a Markov
// head that depends only on the previous token.  Reading: block position k of request r has
// logits z_k = bf16(B[r][k] + E[x_{k-1}] . U) (backbone block logits plus a rank-d transition
// term of the previous token), and x_k is drawn by the Gumbel-max trick over Philox4x32-10
// noise (counter (round, r, v / 4, 3 + 256 (k - 1)), key (seed, 0), u = ((word >> 8) + 1/2)
// 2^-24), or greedily (lowest index of the maximum) at temperature <= 0.
//
// Per position two kernels: markov_logits_kernel (one CTA per 256-token slice of the
// vocabulary: the transition terms of 64 requests at a time as a bf16 tensor-core GEMM of rank
// d <= 64, then the block logits, bf16 rounding, draft-logit store, Gumbel noise and the slice's
// best token per request) and markov_select_kernel (one CTA per request: best over the slices).
#pragma once

#include "common.cuh"
#include "ptx_sm100.cuh"

namespace dspark {

constexpr int kDraftThreads = 256;
constexpr int kDraftSlice = 256;                // tokens per CTA of markov_logits_kernel
constexpr int kDraftMaxRank = 64;
constexpr int kDraftGroup = 64;                 // requests whose E rows sit in shared memory

struct DraftWs {
  float *best_s;  // [nslices][R]
  int *best_i;    // [nslices][R]
  int *xprev;     // [R]
};

__host__ __device__ inline size_t draft_ws_layout(int R, int V, DraftWs *ws, void *base) {
  const size_t ns = ((size_t)V + kDraftSlice - 1) / kDraftSlice;
  size_t off = 0;
  const size_t o_s = off; off += align256(ns * R * sizeof(float));
  const size_t o_i = off; off += align256(ns * R * sizeof(int));
  const size_t o_x = off; off += align256((size_t)R * sizeof(int));
  if (ws) {
    char *b = static_cast<char *>(base);
    ws->best_s = reinterpret_cast<float *>(b + o_s);
    ws->best_i = reinterpret_cast<int *>(b + o_i);
    ws->xprev = reinterpret_cast<int *>(b + o_x);
  }
  return off;
}

// Philox4x32-10 ("Parallel Random Numbers: As Easy as 1, 2, 3", SC'11, section 3).
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
  for (int rnd = 0; rnd < 10; ++rnd) {
    if (rnd > 0) {
      k.x += 0x9E3779B9u;
      k.y += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
  }
  return c;
}

// Gumbel noise -log(-log(u)) with the SFU logarithm (absolute error ~1e-6 here; a token whose
// score is that close to the runner-up is a near-tie in any precision).
__device__ __forceinline__ float gumbel_from_word(uint32_t w) {
  const float u = ((float)(w >> 8) + 0.5f) * 5.9604644775390625e-8f;  // 2^-24
  return -__logf(-__logf(u));
}

// Better of two (score, index) candidates: higher score, then lower index.
__device__ __forceinline__ bool draft_better(float s, int i, float s2, int i2) {
  return s > s2 || (s == s2 && i < i2);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &a, uint32_t &b, uint32_t &c,
                                        uint32_t &d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &a, uint32_t &b,
                                              uint32_t &c, uint32_t &d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One CTA per kDraftSlice-token slice of the vocabulary.  The transition terms of up to 64
// requests at once are a small GEMM, E_prev [64 x 64] . U_slice [64 x 256], on the tensor cores
// (warp w owns 32 tokens of the slice, all 64 request rows); the epilogue adds the block
// logits, rounds to bf16, writes the draft logits, adds the Gumbel noise and keeps each
// request's best token of the slice.
__global__ void __launch_bounds__(kDraftThreads, 2)
markov_logits_kernel(const __nv_bfloat16 *__restrict__ B, const __nv_bfloat16 *__restrict__ E,
                     const __nv_bfloat16 *__restrict__ U, int d, const int32_t *__restrict__ xprev,
                     int R, int K, int V, int k, float inv_tau, int sampled, uint32_t round_idx,
                     uint32_t seed, __nv_bfloat16 *__restrict__ out, DraftWs ws) {
  constexpr int kUS = kDraftSlice + 8;         // padded row (elements): ldmatrix without conflicts
  constexpr int kES = kDraftMaxRank + 8;
  __shared__ __align__(16) __nv_bfloat16 Us[kDraftMaxRank][kUS];
  __shared__ __align__(16) __nv_bfloat16 Es[kDraftGroup][kES];
  __shared__ float bs[kDraftThreads / 32][kDraftGroup];
  __shared__ int bi[kDraftThreads / 32][kDraftGroup];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int vs = blockIdx.x * kDraftSlice;
  // U slice (rows j < d; tokens past V and rows past d are zero)
  for (int idx = tid; idx < kDraftMaxRank * (kDraftSlice / 8); idx += kDraftThreads) {
    const int j = idx / (kDraftSlice / 8), c = idx % (kDraftSlice / 8);
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (j < d && vs + c * 8 < V) w = __ldg(reinterpret_cast<const uint4 *>(U + (size_t)j * V + vs + c * 8));
    *reinterpret_cast<uint4 *>(&Us[j][c * 8]) = w;
  }
  const uint32_t us_base = ptx::smem_u32(&Us[0][0]), es_base = ptx::smem_u32(&Es[0][0]);
  const int n0 = warp * 32;  // this warp's tokens within the slice
  for (int r0 = 0; r0 < R; r0 += kDraftGroup) {
    const int nr = min(kDraftGroup, R - r0);
    __syncthreads();
    for (int idx = tid; idx < kDraftGroup * (kDraftMaxRank / 8); idx += kDraftThreads) {
      const int rr = idx / (kDraftMaxRank / 8), c = idx % (kDraftMaxRank / 8);
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (rr < nr && c * 8 < d) {
        int x = __ldg(xprev + r0 + rr);
        if (x < 0 || x >= V) x = 0;
        w = __ldg(reinterpret_cast<const uint4 *>(E + (size_t)x * d + c * 8));
      }
      *reinterpret_cast<uint4 *>(&Es[rr][c * 8]) = w;
    }
    __syncthreads();
    // this thread's block logits (independent of the GEMM): all loads in flight before the MMAs
    uint32_t braw[4][2][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          const int rr = mt * 16 + (lane >> 2) + h * 8;
          const int v = vs + n0 + nt * 8 + 2 * (lane & 3);
          braw[mt][h][nt] = (rr < nr && v < V)
              ? __ldg(reinterpret_cast<const uint32_t *>(B + ((size_t)(r0 + rr) * K + (k - 1)) * V + v))
              : 0u;
        }
    float acc[4][4][4];  // [m tile][n tile][fragment]
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < kDraftMaxRank / 16; ++ks) {
      uint32_t a[4][4], b[4][2];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const int row = mt * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int col = ks * 16 + (lane >> 4) * 8;
        ldsm_x4(es_base + (row * kES + col) * 2, a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
      }
#pragma unroll
      for (int np = 0; np < 2; ++np) {  // two n8 tiles per x4 load
        const int krow = ks * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int ncol = n0 + np * 16 + (lane >> 4) * 8;
        ldsm_x4_trans(us_base + (krow * kUS + ncol) * 2, b[2 * np][0], b[2 * np][1],
                      b[2 * np + 1][0], b[2 * np + 1][1]);
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_16816(acc[mt][nt], a[mt], b[nt][0], b[nt][1]);
    }
    // epilogue: this thread holds rows 16 mt + lane / 4 (+ 8), tokens n0 + 8 nt + 2 (lane % 4) (+ 1)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int rr = mt * 16 + (lane >> 2) + h * 8;
        const int r = r0 + rr;
        float best = -INFINITY;
        int bidx = 0x7fffffff;
        if (rr < nr) {
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            const int v = vs + n0 + nt * 8 + 2 * (lane & 3);
            if (v < V) {
              const size_t off = ((size_t)r * K + (k - 1)) * V + v;
              const float2 bl =
                  __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&braw[mt][h][nt]));
              const __nv_bfloat162 z = __floats2bfloat162_rn(bl.x + acc[mt][nt][2 * h],
                                                             bl.y + acc[mt][nt][2 * h + 1]);
              *reinterpret_cast<__nv_bfloat162 *>(out + off) = z;
              const float2 zf = __bfloat1622float2(z);
              float s0 = zf.x, s1 = zf.y;
              if (sampled) {
                const uint4 w = philox4x32_10(
                    make_uint4(round_idx, (uint32_t)r, (uint32_t)(v >> 2),
                               3u + 256u * (uint32_t)(k - 1)),
                    make_uint2(seed, 0u));
                const bool hi = (v & 2) != 0;
                s0 = s0 * inv_tau + gumbel_from_word(hi ? w.z : w.x);
                s1 = s1 * inv_tau + gumbel_from_word(hi ? w.w : w.y);
              }
              if (s0 > best) { best = s0; bidx = v; }
              if (s1 > best) { best = s1; bidx = v + 1; }
            }
          }
        }
        // the four lanes holding this row
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          const float s2 = __shfl_xor_sync(0xffffffffu, best, o);
          const int i2 = __shfl_xor_sync(0xffffffffu, bidx, o);
          if (draft_better(s2, i2, best, bidx)) { best = s2; bidx = i2; }
        }
        if ((lane & 3) == 0) { bs[warp][rr] = best; bi[warp][rr] = bidx; }
      }
    }
    __syncthreads();
    for (int rr = tid; rr < nr; rr += kDraftThreads) {
      float best = bs[0][rr];
      int bidx = bi[0][rr];
      for (int w = 1; w < kDraftThreads / 32; ++w)
        if (draft_better(bs[w][rr], bi[w][rr], best, bidx)) { best = bs[w][rr]; bidx = bi[w][rr]; }
      ws.best_s[(size_t)blockIdx.x * R + r0 + rr] = best;
      ws.best_i[(size_t)blockIdx.x * R + r0 + rr] = bidx;
    }
  }
}

__global__ void __launch_bounds__(128)
markov_select_kernel(int nslices, int R, int K, int k, DraftWs ws,
                     int32_t *__restrict__ tokens) {
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float best = -INFINITY;
  int bidx = 0x7fffffff;
  for (int c = tid; c < nslices; c += 128) {
    const float s = ws.best_s[(size_t)c * R + r];
    const int i = ws.best_i[(size_t)c * R + r];
    if (draft_better(s, i, best, bidx)) { best = s; bidx = i; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float s2 = __shfl_xor_sync(0xffffffffu, best, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, bidx, o);
    if (draft_better(s2, i2, best, bidx)) { best = s2; bidx = i2; }
  }
  __shared__ float ss[4];
  __shared__ int si[4];
  if (lane == 0) { ss[warp] = best; si[warp] = bidx; }
  __syncthreads();
  if (tid == 0) {
    best = ss[0];
    bidx = si[0];
    for (int w = 1; w < 4; ++w)
      if (draft_better(ss[w], si[w], best, bidx)) { best = ss[w]; bidx = si[w]; }
    tokens[(size_t)r * K + (k - 1)] = bidx;
    ws.xprev[r] = bidx;
  }
}

// x_prev <- x_0 (validated: a token outside [0, V) raises DSPARK_DERR_TOKEN and counts as 0).
__global__ void markov_init_kernel(const int32_t *__restrict__ x0, int R, int V, DraftWs ws) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < R; r += gridDim.x * blockDim.x) {
    int x = x0[r];
    if (x < 0 || x >= V) { raise_error(DSPARK_DERR_TOKEN); x = 0; }
    ws.xprev[r] = x;
  }
}

}  // namespace dspark
