// dspark_schedule: survival scan + greedy marginal-gain prefix scheduler + flattening.
//
// Method (DSpark write-ups): "DSpark 的 661% 提速，是真突破还是数字游戏？" §3.2 (confidence =
// acceptance probability given the accepted prefix; scheduler inputs: load, confidences, the
// engine's throughput curve); "DeepSeek服务器不再卡顿！…", section "DSpark的神奇之处" (queue the
// draft tokens of all requests by score, keep adding while the extra correct tokens pay for the
// extra time); the mooersco.com engineering table (asynchronous scheduler fed by confidences two
// rounds old; flattened verify tokens tagged with markers).
//
// One CTA of 1024 threads does the whole step on-chip:
//   1. S[r][k] = c[r][0] * ... * c[r][k] in float64 (explicit round-to-nearest multiplies, left
//      to right).  Candidate i = k*R + r gets key ~bits(S): for non-negative doubles the bit
//      pattern orders like the value, so ascending keys = descending S.
//   2. Stable LSD radix sort (8-bit digits) of the keys with the candidate index as payload.
//      Ranks within a warp come from __match_any_sync; per-(digit, warp) counts are scanned in
//      digit-major order, so equal keys keep their initial (k, r) order — the tie rule.
//      Passes whose digit is the same for every key are skipped.
//   3. Prefix sums of the sorted S (float64; sequential per thread, tree across threads),
//      f(n) = (R + P(n)) / t_ms[R + n], n* = first n with f(n+1) <= f(n).
//   4. verify_len by counting the first n* payloads, exclusive scan into q_offsets, markers
//      (or, for a lengths-only call, no markers: flatten_markers_kernel writes them later from
//      the cache lengths current then).
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kSchedThreads = 1024;
constexpr int kSchedWarps = kSchedThreads / 32;

__device__ __forceinline__ uint32_t block_excl_scan_u32(uint32_t x, uint32_t *sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sm[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t v = (lane < kSchedWarps) ? sm[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    sm[lane] = v;
  }
  __syncthreads();
  uint32_t res = (warp ? sm[warp - 1] : 0u) + incl - x;
  __syncthreads();
  return res;
}

__device__ __forceinline__ double block_excl_scan_f64(double x, double *sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl = __dadd_rn(incl, y);
  }
  if (lane == 31) sm[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    double v = (lane < kSchedWarps) ? sm[lane] : 0.0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      double y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v = __dadd_rn(v, y);
    }
    sm[lane] = v;
  }
  __syncthreads();
  // exclusive prefix of this thread = sum of earlier warps + exclusive within warp
  double excl_warp = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl_warp = 0.0;
  double res = warp ? __dadd_rn(sm[warp - 1], excl_warp) : excl_warp;
  __syncthreads();
  return res;
}

__device__ __forceinline__ uint64_t block_or_and(uint64_t v, bool is_and, uint64_t *sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    uint64_t y = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_and ? (v & y) : (v | y);
  }
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  uint64_t r = sm[0];
  for (int w = 1; w < kSchedWarps; ++w) r = is_and ? (r & sm[w]) : (r | sm[w]);
  __syncthreads();
  return r;
}

// Dynamic shared memory: keys u64[NPAD] | vals u16[NPAD] | hist u32[256*32] | scratch.
template <int E>
__global__ void __launch_bounds__(kSchedThreads, 1)
schedule_kernel(const float *__restrict__ conf_ring, int ring_depth, int round_idx, int R, int K,
                const int32_t *__restrict__ kv_len, const double *__restrict__ t_ms, int T_cap,
                int32_t *__restrict__ verify_len, int32_t *__restrict__ q_offsets,
                int32_t *__restrict__ markers, int32_t *__restrict__ T_out,
                double *__restrict__ objective) {
  constexpr int NPAD = kSchedThreads * E;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);
  uint16_t *vals = reinterpret_cast<uint16_t *>(keys + NPAD);
  uint32_t *hist = reinterpret_cast<uint32_t *>(vals + NPAD);
  __shared__ uint64_t red64[kSchedWarps];
  __shared__ uint32_t red32[kSchedWarps];
  __shared__ double redf[kSchedWarps];
  __shared__ int s_fail;
  __shared__ double s_f0;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = R * K;
  const int slot = max(round_idx - DSPARK_CONF_LAG, 0) % ring_depth;
  const float *conf = conf_ring + (size_t)slot * R * K;

  // 1. survival products and sort keys
  for (int r = tid; r < R; r += kSchedThreads) {
    double acc = 1.0;
    bool bad = false;
    for (int k = 0; k < K; ++k) {
      float c = conf[(size_t)r * K + k];
      if (!(c >= 0.f && c <= 1.f)) { bad = true; c = 0.f; }
      if (c == 0.f) c = 0.f;  // canonical +0 so that -0 cannot sort ahead of positive values
      acc = __dmul_rn(acc, (double)c);
      keys[k * R + r] = ~(uint64_t)__double_as_longlong(acc);
      vals[k * R + r] = (uint16_t)(k * R + r);
    }
    if (bad) raise_error(DSPARK_DERR_CONF);
  }
  for (int i = N + tid; i < NPAD; i += kSchedThreads) {
    keys[i] = ~0ull;  // padding sorts last (stable: after any S == 0 candidate)
    vals[i] = (uint16_t)i;
  }
  __syncthreads();

  // 2. stable LSD radix sort, warp-striped registers
  uint64_t k[E];
  uint16_t v[E];
  uint64_t kor = 0, kand = ~0ull;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int idx = warp * 32 * E + e * 32 + lane;
    k[e] = keys[idx];
    v[e] = vals[idx];
    kor |= k[e];
    kand &= k[e];
  }
  kor = block_or_and(kor, false, red64);
  kand = block_or_and(kand, true, red64);
  const uint64_t varying = kor ^ kand;

  for (int pass = 0; pass < 8; ++pass) {
    const int shift = pass * 8;
    if (((varying >> shift) & 0xFFull) == 0) continue;  // uniform across the block
    for (int i = tid; i < 256 * kSchedWarps; i += kSchedThreads) hist[i] = 0;
    __syncthreads();
    uint32_t rank[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const unsigned d = (unsigned)((k[e] >> shift) & 0xFF);
      const unsigned peers = __match_any_sync(0xffffffffu, d);
      const unsigned before = __popc(peers & lanemask_lt());
      const uint32_t base = hist[d * kSchedWarps + warp];
      __syncwarp();
      if (before == 0) hist[d * kSchedWarps + warp] = base + __popc(peers);
      __syncwarp();
      rank[e] = base + before;
    }
    __syncthreads();
    {  // exclusive scan over (digit, warp), digit-major: 8 counters per thread
      uint32_t loc[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { loc[i] = hist[tid * 8 + i]; s += loc[i]; }
      uint32_t ex = block_excl_scan_u32(s, red32);
#pragma unroll
      for (int i = 0; i < 8; ++i) { hist[tid * 8 + i] = ex; ex += loc[i]; }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const unsigned d = (unsigned)((k[e] >> shift) & 0xFF);
      const uint32_t dst = hist[d * kSchedWarps + warp] + rank[e];
      keys[dst] = k[e];
      vals[dst] = v[e];
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = warp * 32 * E + e * 32 + lane;
      k[e] = keys[idx];
      v[e] = vals[idx];
    }
    __syncthreads();
  }

  // 3. prefix sums in sorted order (blocked: thread owns positions tid*E .. tid*E+E-1)
  const int n_max = min(N, T_cap - R);
  double pre[E];
  uint16_t cand[E];
  double run = 0.0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = tid * E + e;
    const double s = (i < N) ? __longlong_as_double((long long)~keys[i]) : 0.0;
    cand[e] = vals[i];
    run = __dadd_rn(run, s);
    pre[e] = run;
  }
  const double excl = block_excl_scan_f64(run, redf);  // contains __syncthreads
  double *fbuf = reinterpret_cast<double *>(keys);      // fbuf[i] = f(i + 1)
  const double Rd = (double)R;
  bool bad_table = false;
  if (tid == 0) {
    const double t0 = t_ms[R];
    if (!(t0 > 0.0)) bad_table = true;
    s_f0 = (t0 > 0.0) ? __ddiv_rn(Rd, t0) : 0.0;
    s_fail = n_max;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = tid * E + e;
    if (i < n_max) {
      const double P = __dadd_rn(excl, pre[e]);
      const double t = t_ms[R + i + 1];
      if (!(t > 0.0)) bad_table = true;
      fbuf[i] = (t > 0.0) ? __ddiv_rn(__dadd_rn(Rd, P), t) : 0.0;
    }
  }
  if (bad_table) raise_error(DSPARK_DERR_TABLE);
  __syncthreads();
  {
    int fail = n_max;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int n = tid * E + e;  // compare f(n + 1) with f(n)
      if (n < n_max) {
        const double fn = (n == 0) ? s_f0 : fbuf[n - 1];
        if (!(fbuf[n] > fn)) { fail = min(fail, n); }
      }
    }
    if (fail < n_max) atomicMin(&s_fail, fail);
  }
  __syncthreads();
  const int n_star = s_fail;
  if (tid == 0) *objective = (n_star == 0) ? s_f0 : fbuf[n_star - 1];
  __syncthreads();

  // 4. verify lengths (counts reuse the key buffer), offsets, markers
  int *Lcnt = reinterpret_cast<int *>(keys);
  for (int r = tid; r < R; r += kSchedThreads) Lcnt[r] = 0;
  __syncthreads();
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if (tid * E + e < n_star) atomicAdd(&Lcnt[cand[e] % R], 1);
  }
  __syncthreads();
  const int per = (R + kSchedThreads - 1) / kSchedThreads;  // blocked over requests
  uint32_t qsum = 0;
  for (int i = 0; i < per; ++i) {
    const int r = tid * per + i;
    if (r < R) qsum += 1u + (uint32_t)Lcnt[r];
  }
  uint32_t off = block_excl_scan_u32(qsum, red32);
  for (int i = 0; i < per; ++i) {
    const int r = tid * per + i;
    if (r < R) {
      const int L = Lcnt[r];
      verify_len[r] = L;
      q_offsets[r] = (int32_t)off;
      if (markers != nullptr) {  // lengths-only calls leave the markers to flatten_markers_kernel
        int n = kv_len[r];
        if (n < 0) { raise_error(DSPARK_DERR_KV_LEN); n = 0; }
        for (int j = 0; j <= L; ++j) {
          markers[2 * (off + j)] = r;
          markers[2 * (off + j) + 1] = n + j;
        }
      }
      off += 1u + (uint32_t)L;
      if (r == R - 1) {
        q_offsets[R] = (int32_t)off;
        *T_out = (int32_t)off;
      }
    }
  }
}

// The flattening step alone: markers[q_offsets[r] + j] = (r, kv_len[r] + j), j < Q_r, from
// offsets a lengths-only schedule wrote earlier and the cache lengths current now.  One thread
// per request; offsets that are not a valid flattening within T_cap raise DSPARK_DERR_OFFSETS
// and that request's markers are not written.
__global__ void flatten_markers_kernel(const int32_t *__restrict__ kv_len,
                                       const int32_t *__restrict__ q_offsets, int R, int K,
                                       int T_cap, int32_t *__restrict__ markers) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= R) return;
  const int t0 = q_offsets[r], Q = q_offsets[r + 1] - t0;
  if (Q < 1 || Q > K + 1 || t0 < 0 || t0 > T_cap - Q) {
    raise_error(DSPARK_DERR_OFFSETS);
    return;
  }
  int n = kv_len[r];
  if (n < 0) { raise_error(DSPARK_DERR_KV_LEN); n = 0; }
  for (int j = 0; j < Q; ++j) {
    markers[2 * (t0 + j)] = r;
    markers[2 * (t0 + j) + 1] = n + j;
  }
}

inline size_t schedule_smem_bytes(int E) {
  const size_t npad = (size_t)kSchedThreads * E;
  return npad * 8 + npad * 2 + 256 * kSchedWarps * 4;
}

}  // namespace dspark
