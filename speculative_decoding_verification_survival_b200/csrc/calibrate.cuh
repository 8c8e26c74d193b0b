// Temporal temperature scaling of the confidence head and its maximum-likelihood fit.
//
// "刚融完500亿…专治AI“嘴慢”" section "2. 置信度调度验证": after training, a post-hoc calibration
// ("temporal temperature scaling") corrects the raw confidence head's over-confidence;
// "DSpark 的 661% 提速…" §3.2: the confidence of block position k is the probability that the
// token is accepted given that its prefix was.  Reading: one temperature per block position,
// c_k = sigmoid(l_k / tau_k), tau_k fitted by maximum likelihood on observed accept outcomes
// (position k is observed iff the prefix before it survived verification), beta = 1 / tau_k
// kept in [1/64, 64].
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kFitThreads = 256;
constexpr double kBetaLo = 1.0 / 64.0, kBetaHi = 64.0;

// c[r][k] = sigmoid(l[r][k] / tau[k]), evaluated in float64 and rounded once.  A temperature
// that is not a positive finite number, or a NaN logit, gives c = 0 and sets DSPARK_DERR_CONF.
__global__ void calibrate_kernel(const float *__restrict__ logits, const float *__restrict__ tau,
                                 int R, int K, float *__restrict__ conf) {
  const int n = R * K;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int k = i % K;
    const float t = __ldg(tau + k), l = __ldg(logits + i);
    float c = 0.f;
    if (!(t > 0.f && t < INFINITY) || l != l) {
      raise_error(DSPARK_DERR_CONF);
    } else {
      const double x = (double)l / (double)t;
      c = (float)(1.0 / (1.0 + exp(-x)));
    }
    conf[i] = c;
  }
}

// Block sum of two float64 values (all threads receive the totals).
__device__ __forceinline__ double2 block_sum2(double a, double b, double2 *sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  a = warp_sum(a);
  b = warp_sum(b);
  if (lane == 0) sm[warp] = make_double2(a, b);
  __syncthreads();
  double2 t = make_double2(0.0, 0.0);
  for (int w = 0; w < kFitThreads / 32; ++w) { t.x += sm[w].x; t.y += sm[w].y; }
  __syncthreads();
  return t;
}

// One CTA per block position k.  Outcome of sample i at position k (1-based k + 1): observed iff
// k + 1 <= min(a_i + 1, L_i); accepted iff k + 1 <= a_i.  The negative log-likelihood
// sum log(1 + exp(-s beta l)) (s = +1 accepted, -1 rejected) is convex in beta; its root of the
// derivative is bracketed in [kBetaLo, kBetaHi] and found by Newton steps that fall back to a
// geometric bisection whenever a step leaves the bracket.
__global__ void __launch_bounds__(kFitThreads)
fit_temperature_kernel(const float *__restrict__ logits, const int32_t *__restrict__ verify_len,
                       const int32_t *__restrict__ accepted_len, int N, int K,
                       float *__restrict__ tau) {
  __shared__ double2 sm[kFitThreads / 32];
  const int k = blockIdx.x, tid = threadIdx.x;
  // derivative and second derivative of the NLL at beta; .x also counts usable samples at beta 0
  auto eval = [&](double beta, bool count) -> double2 {
    double g = 0.0, h = 0.0;
    for (int i = tid; i < N; i += kFitThreads) {
      const int L = __ldg(verify_len + i), a = __ldg(accepted_len + i);
      if (L < 0 || L > K || a < 0 || a > L) {
        if (count) raise_error(DSPARK_DERR_ACCEPTED);
        continue;
      }
      if (k + 1 > min(a + 1, L)) continue;  // not observed
      const float l = __ldg(logits + (size_t)i * K + k);
      if (l != l) continue;
      if (count) {
        g += 1.0;
        h += (l != 0.f) ? 1.0 : 0.0;
        continue;
      }
      const float s = (k + 1 <= a) ? 1.f : -1.f;
      const float z = -s * (float)beta * l;
      const float sig = 1.f / (1.f + expf(-z));  // sigmoid(z)
      g += -(double)(s * l * sig);
      h += (double)(l * l * sig * (1.f - sig));
    }
    return block_sum2(g, h, sm);
  };
  const double2 cnt = eval(0.0, true);
  double beta = 1.0;
  if (cnt.y > 0.0) {
    double lo = kBetaLo, hi = kBetaHi;
    if (eval(lo, false).x >= 0.0) {
      beta = lo;
    } else if (eval(hi, false).x <= 0.0) {
      beta = hi;
    } else {
      beta = 1.0;
      for (int it = 0; it < 100; ++it) {
        const double2 gh = eval(beta, false);
        if (gh.x < 0.0) lo = beta; else hi = beta;
        double nb = (gh.y > 0.0) ? beta - gh.x / gh.y : -1.0;
        if (!(nb > lo && nb < hi)) nb = sqrt(lo * hi);
        const bool done = fabs(nb - beta) <= 1e-12 * beta || hi - lo <= 1e-12 * hi;
        beta = nb;
        if (done) break;
      }
    }
  }
  if (tid == 0) tau[k] = (float)(1.0 / beta);
}

}  // namespace dspark
