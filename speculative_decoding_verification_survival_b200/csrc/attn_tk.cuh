// Tensor-core verify attention with the keys on the tensor-memory lanes (sm_100a; bf16, D = 128,
// page size a multiple of 64, K + 1 <= 16, G * (K + 1) <= 64).
//
// A persistent CTA per SM walks a contiguous range of (request, KV head, unit) work as the plan
// cut it (attn_common.cuh): the units of a segment are its 64-key cache pages, then the request's
// own verify tokens; every KV byte is read once for all G * Q_r query rows of its (request, KV
// head) — the flattened, unpadded verify batch of "刚融完500亿…专治AI“嘴慢”" (engineering table,
// row "内核利用率暴跌").  A 128-key tile (two pages) meets the rows through two MMA chains:
//
//   S^T = K . Q^T       M = 128 keys (the tensor-memory lanes), N = 32 query rows, K = D:
//                       8 tcgen05.mma (kind::f16), the K tile as the TMA wrote it and the
//                       rows staged by cp.async, both in shared memory
//   O^T += V^T . P^T    M = 128 (D on the lanes), N = 32 rows, K = 128 keys: 8 MMAs, V as the
//                       TMA wrote it (MN-major), P^T written by the softmax warps
//
// N is the query-row count: with the rows on the M side (128 lanes) three quarters of every MMA
// would be padding for <= 32 rows, and the tensor core's time and power set the pace.  A
// segment with 33..64 rows is taken in two passes of 32 rows over the same keys (each pass
// reads its keys again; the schedules of the benchmark workloads give at most 32 rows).
//
// Per CTA (512 threads, 16 warps): warps 8 and 12 load K (TMA, one 128-byte-swizzled 4-D box per
// page, page 0 and page 1 of every tile, a ring of 3 tiles with one barrier each), warps 10 and
// 14 load V (the same, its own ring): one warp issues about one box per 850 cycles, and two per
// ring keep up with HBM also at a power-capped clock.  One thread of warp 9 issues the S^T MMAs
// and one of warp 11 the P.V MMAs; warps 13 and 15 idle.  Warpgroups 2 and 3 hand registers to
// warpgroups 0 and 1 (setmaxnreg: 88 and 168 per thread, from 128 at launch), which do the
// softmax and the epilogue: warp w reads the lanes of its
// quadrant q = w % 4 (keys 32q .. 32q + 31 of the tile, and d = 32q .. 32q + 31 of O^T) and the
// columns of its half hf = w / 4 of the rows, so every thread holds one key's scores for 16
// rows.  A row's reference maximum comes from the pass's first tile and is raised only when a
// score exceeds it by more than 2^8 (log2 domain): the 128 threads of a half vote every tile and
// a tile that exceeds takes the slow path (row maxima by warp shuffles and a shared-memory
// exchange, tensor-memory rescale of O^T).  Row sums stay per thread (per key) until the pass's
// epilogue.  Every mbarrier wait is bounded (ptx::mbar_wait, its polling loop out of line in the
// MMA issuers, inlined elsewhere); on timeout the CTA records DSPARK_DERR_TIMEOUT, skips the
// remaining work and still releases its TMEM.
#pragma once

#include "attn_generic.cuh"
#include "ptx_sm100.cuh"

namespace dspark {
namespace tk {

constexpr int kPage = 64;
constexpr int kTK = 128;                             // keys per tile (two page slots)
constexpr int kPairsK = 3, kPairsV = 3;              // tile slots per ring (two pages each)
constexpr int kMaxPairs = 4;
static_assert(kPairsK <= kMaxPairs && kPairsV <= kMaxPairs && 8 * kMaxPairs <= 48, "slot counts");
constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
// warpgroup 2: K producer (page 0 of each tile), S^T issuer, V producer (page 0), P.V issuer;
// warpgroup 3: K producer (page 1), idle, V producer (page 1), idle
constexpr int kWarpK = kSoftmaxWarps, kWarpMma = kSoftmaxWarps + 1, kWarpV = kSoftmaxWarps + 2,
              kWarpPV = kSoftmaxWarps + 3, kWarpK2 = kSoftmaxWarps + 4, kWarpV2 = kSoftmaxWarps + 6;
constexpr int kThreads = kSoftmaxThreads + 256;
// registers per thread: at launch (the pool: 65536 / 512), then the softmax warpgroups and the
// others after the split; the shares add up to the pool
constexpr int kRegsLaunch = 128, kRegsSoftmax = 168, kRegsOther = 88;
static_assert(kRegsSoftmax * kSoftmaxThreads + kRegsOther * (kThreads - kSoftmaxThreads) <=
                  kRegsLaunch * kThreads, "register split");
constexpr int kD = 128;
constexpr int kNewRows = 16;                         // verify tokens per tile (K + 1 <= 16)
constexpr int kN = 32;                               // query rows per pass (the MMAs' N)
constexpr int kRH = kN / 2;                          // rows per softmax thread
// A page slot holds one page of K or V (64 rows x 128 d, bf16) as eight 2048-byte row groups,
// each the two d-halves of its 8 rows as 1024-byte 128-byte-swizzled atoms:
//   byte (r / 8) * 2048 + h * 1024 + (r % 8) * 128 + swizzled 16-byte chunk   (h = d / 64)
// so the 128 rows of a tile's two consecutive page slots are 16 atoms 2048 bytes apart for
// either d-half: one K-major operand (K, SBO 2048) or one MN-major operand (V, LBO 1024 between
// the d-halves, SBO 2048 between groups of 8 keys), and one TMA box brings a whole page.
constexpr uint32_t kPageBytes = 64 * 256;
constexpr uint32_t kGroupBytes = 2048;
constexpr uint32_t kTileBytes = 2 * kPageBytes;
constexpr uint32_t kRingBytesK = kPairsK * kTileBytes;
constexpr uint32_t kRingBytesV = kPairsV * kTileBytes;
constexpr uint32_t kNewBytes = kNewRows * 256;        // the verify tokens' 16 rows
constexpr uint32_t kQHalfBytes = kN * 128;           // one d-half of a query buffer
constexpr uint32_t kQBufBytes = 2 * kQHalfBytes;
constexpr uint32_t kPBytes = kTK * kN * 2;           // P^T: 128 keys x 32 rows, bf16
constexpr uint32_t kOffQ = kRingBytesK + kRingBytesV;
constexpr uint32_t kOffP = kOffQ + 2 * kQBufBytes;
constexpr uint32_t kOffAux = kOffP + kPBytes;
constexpr uint32_t kAuxBytes = 2048;
constexpr uint32_t kSmemBytes = kOffAux + kAuxBytes + 1024;  // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
constexpr int kPS = part_stride(kD);

// aux region (bytes)
constexpr uint32_t kBarKFull = 0, kBarSFree = 48, kBarVFull = 64, kBarKEmpty = 128, kBarVEmpty = 192,
                   kBarSFull = 256, kBarPFull = 272, kBarODone = 280, kBarQFull = 288,
                   kBarQEmpty = 304, kBarOFree = 320, kBarDrain = 328;  // [2]: S^T, P.V issuer
constexpr uint32_t kAuxTmem = 344, kAuxAbort = 348, kAuxLast = 352, kAuxSplit = 356,
                   kAuxFlags = 384,   // int [2 tile parity][2 halves][4 quadrants]
                   kAuxRmax = 512,    // float [2 tile parity][2 halves][4 quadrants][16 rows]
                   kAuxLsum = 1536;   // float [2 halves][4 quadrants][16 rows]  (to 2048)

constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kColS = 0;      // + 32 * buffer
constexpr uint32_t kColO = 64;
constexpr float kRescaleLog2 = 8.f;
// named barriers: 1 + hf for the 128 threads of one half of the rows, 3 for all softmax warps
constexpr int kBarAllSoftmax = 3;

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, kN, 0, 0);   // K (K-major) x Q^T (K-major)
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, kN, 1, 1);  // V^T (MN) x P^T (MN)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// 128-byte swizzle: 16-byte chunk c of row r in 8-row atoms of 1024 bytes
__device__ __forceinline__ uint32_t sw128(uint32_t base, int r, int c) {
  return base + (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u +
         ((uint32_t)(c ^ (r & 7)) << 4);
}
// 64-byte swizzle: 16-byte chunk c (0..3) of row r in 8-row atoms of 512 bytes
__device__ __forceinline__ uint32_t sw64(uint32_t base, int r, int c) {
  return base + (uint32_t)(r >> 3) * 512u + (uint32_t)(r & 7) * 64u +
         ((uint32_t)(c ^ ((r >> 1) & 3)) << 4);
}

// A piece of a segment: the plan's per-request record (one 16-byte load) and the piece's share
// of the segment's units; every role derives it identically.
struct Meta {
  int t0, Q, n, rows, npages, ncache, ntiles, npass;  // npages: cache pages of the piece
  bool valid, last, newtile;                          // ncache: their 128-key tiles
};
__device__ __forceinline__ Meta piece_meta(const AttnArgs &a, const int4 &rec, int ta, int tb,
                                           int tiles, bool raise) {
  Meta m;
  m.t0 = rec.x;
  m.Q = rec.y;
  m.n = rec.z;
  bool ok = rec.w != 0;
  const bool okn = (int64_t)(m.n + a.page_size - 1) / a.page_size <= a.max_pages;
  if (ok && !okn && raise) raise_error(DSPARK_DERR_KV_LEN);
  ok = ok && okn;
  m.valid = ok;
  m.rows = ok ? a.G * m.Q : 0;
  m.npass = m.rows > kN ? 2 : 1;
  m.npages = ok ? max(0, min(tb, segment_cache_tiles(tiles)) - ta) : 0;
  m.ncache = (m.npages + 1) / 2;
  m.last = (tb == tiles);
  m.newtile = ok && m.last;
  m.ntiles = m.ncache + (m.newtile ? 1 : 0);
  return m;
}

// This CTA's contiguous range of units [u, u1) as pieces (one per segment it touches), walking
// the segments in order from the CTA's start record written by the plan.
struct PieceIter {
  int u, u1;
  Ranges rg;
  int r, g, tiles, s0;  // current segment
  int4 first_rec;       // the first segment's request record, from the plan's start records
  bool have_first;
  __device__ __forceinline__ void init(const AttnArgs &a) {
    // every load of the start issued at once (all in bounds for any grid up to the plan's
    // maximum), so the first piece is one round trip away
    const int total = __ldg(&a.ws.hdr->total);
    const int ctas = __ldg(&a.ws.hdr->tc_ctas);
    const int4 st = __ldg(a.ws.cta_start + blockIdx.x);
    const int b0 = __ldg(a.ws.cta_begin + blockIdx.x), b1 = __ldg(a.ws.cta_begin + blockIdx.x + 1);
    first_rec = __ldg(a.ws.cta_req + blockIdx.x);
    have_first = false;
    if (ctas == (int)gridDim.x) {  // the plan's cost-balanced ranges
      rg.begin = a.ws.cta_begin;
      rg.W = 0;
      rg.ctas = ctas;
      rg.total = total;
      r = st.x; g = st.y; s0 = st.z; tiles = st.w;
      u = b0;
      u1 = (r < 0) ? u : min(b1, total);
      have_first = true;
      return;
    } else {  // a grid the plan did not prepare for: equal ranges, search the first segment
      rg.begin = nullptr;
      rg.W = (total + gridDim.x - 1) / gridDim.x;
      rg.ctas = gridDim.x;
      rg.total = total;
      r = -1;
      if ((int64_t)blockIdx.x * rg.W < total)
        find_segment(a.ws.tile_prefix, a.R, a.Hkv, blockIdx.x * rg.W, r, g, tiles, s0);
    }
    u = rg.start(blockIdx.x);
    u1 = (r < 0) ? u : min(rg.start(blockIdx.x + 1), total);
  }
  __device__ __forceinline__ bool next(const AttnArgs &a, int &r_, int &g_, int &ta, int &tb,
                                       int &tiles_, int &s0_) {
    if (u >= u1) return false;
    r_ = r; g_ = g; tiles_ = tiles; s0_ = s0;
    ta = u - s0;
    tb = min(tiles, u1 - s0);
    u = s0 + tb;
    if (tb == tiles && u < u1) {  // on to the next segment: (r, g + 1) or (r + 1, 0)
      s0 += tiles;
      if (++g == a.Hkv) {
        g = 0;
        ++r;
        tiles = (__ldg(a.ws.tile_prefix + r + 1) - __ldg(a.ws.tile_prefix + r)) / a.Hkv;
      }
    }
    return true;
  }
};

// A pass: a piece and one of its (at most two) groups of 32 query rows.
struct Pass {
  int r, g, ta, tb, tiles, s0, h;
  Meta m;
};

// Walks the passes of this CTA's pieces in order.
struct PassIter {
  PieceIter it;
  __device__ __forceinline__ void init(const AttnArgs &a) { it.init(a); }
  __device__ __forceinline__ bool first(const AttnArgs &a, Pass &p, bool raise) {
    if (!it.next(a, p.r, p.g, p.ta, p.tb, p.tiles, p.s0)) return false;
    p.h = 0;
    const int4 rec = it.have_first ? it.first_rec : __ldg(a.ws.req + p.r);
    it.have_first = false;
    p.m = piece_meta(a, rec, p.ta, p.tb, p.tiles, raise);
    return true;
  }
  __device__ __forceinline__ bool next(const AttnArgs &a, const Pass &cur, Pass &p, bool raise) {
    if (cur.h + 1 < cur.m.npass) {
      p = cur;
      ++p.h;
      return true;
    }
    return first(a, p, raise);
  }
};

// Walks the tiles of this CTA's passes in order (passes without tiles are skipped).  gt =
// global tile index of the CTA, pq = index of the current pass among the passes with tiles.
struct TileCursor {
  PassIter pi;
  Pass p;
  int j;
  uint32_t gt, pq;
  bool ok;
  __device__ __forceinline__ bool settle(const AttnArgs &a, bool have) {
    while (have) {
      if (p.m.ntiles > 0) {
        j = 0;
        return true;
      }
      Pass nx;
      have = pi.next(a, p, nx, false);
      p = nx;
    }
    return false;
  }
  __device__ __forceinline__ void init(const AttnArgs &a) {
    pi.init(a);
    gt = 0;
    pq = 0;
    ok = settle(a, pi.first(a, p, false));
  }
  __device__ __forceinline__ void advance(const AttnArgs &a) {
    ++gt;
    if (++j == p.m.ntiles) {
      ++pq;
      Pass nx;
      const bool have = pi.next(a, p, nx, false);
      p = nx;
      ok = settle(a, have);
    }
  }
};

// One tile for this thread's key (kk) and half of the pass's rows: scores from TMEM, masking,
// the vote on the reference maxima (slow path: row maxima over the tile's keys, rescale of the
// row sums and of O^T), P^T of its key into shared memory.
__device__ __forceinline__ void softmax_tile(const AttnArgs &a, float (&mref)[kRH],
                                             float (&lpart)[kRH], uint32_t tmem,
                                             uint32_t lane_base, unsigned char *gaux, uint32_t aux,
                                             volatile int *abort_flag, uint32_t gt, int vk,
                                             bool cache_tile, int kk, int q, int hf, int lane,
                                             int nr, int rcausal, uint32_t pbase, bool first_tile) {
  const uint32_t b = gt & 1;
  float x[kRH];
  ptx::tmem_ld16(tmem + lane_base + kColS + b * kN + hf * kRH, x);
  ptx::tmem_wait_ld();
  // S^T(gt) is in registers: S^T(gt + 2) may overwrite its buffer
  ptx::tc_fence_before();
  ptx::mbar_arrive(aux + kBarSFree + 8u * b);
  // local row i (of the pass) sees this key if the key is valid and, in the verify-token tile,
  // the key's token is not after the row's (i >= rcausal = kk * G - first row of the pass)
  const int rmin = cache_tile ? 0 : rcausal;
  const int rlim = kk < vk ? nr : 0;
  bool exceed = false;
#pragma unroll
  for (int i = 0; i < kRH; ++i) {
    const int rl = hf * kRH + i;
    x[i] = (rl < rlim && rl >= rmin) ? x[i] * a.scale_log2 : -INFINITY;
    exceed |= x[i] > mref[i] + kRescaleLog2;
  }
  int *flags = reinterpret_cast<int *>(gaux + kAuxFlags) + b * 8 + hf * 4;
  const bool wexceed = __any_sync(0xffffffffu, exceed);
  if (lane == 0) flags[q] = wexceed ? 1 : 0;
  ptx::named_bar_sync(1 + hf, 128);
  const bool slow = (flags[0] | flags[1] | flags[2] | flags[3]) != 0;
  if (slow) {
    // row maxima over the tile's 128 keys: within the warp by shuffles, across the quadrants
    // through shared memory
    float *rmax = reinterpret_cast<float *>(gaux + kAuxRmax) + (b * 2 + hf) * 4 * kRH;
#pragma unroll
    for (int i = 0; i < kRH; ++i) {
      const float w = warp_max(x[i]);
      if (lane == i) rmax[q * kRH + i] = w;
    }
    ptx::named_bar_sync(1 + hf, 128);
    // raise the reference maxima; the row sums so far and O^T's row columns of this thread's
    // lane (d = kk), which hold the earlier tiles, are rescaled by 2^(old - new) — O^T once the
    // previous tile's P.V has completed
    const bool rescale_o = !first_tile;
    if (rescale_o) {
      ptx::mbar_wait_inl(aux + kBarODone, (gt - 1) & 1, abort_flag);
      ptx::tc_fence_after();
    }
    const uint32_t o_taddr = tmem + lane_base + kColO + hf * kRH;
#pragma unroll
    for (int c8 = 0; c8 < kRH / 8; ++c8) {
      float o8[8];
      if (rescale_o) {
        ptx::tmem_ld8(o_taddr + c8 * 8, o8);
        ptx::tmem_wait_ld();
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = c8 * 8 + e;
        const float t = fmaxf(fmaxf(rmax[i], rmax[kRH + i]), fmaxf(rmax[2 * kRH + i], rmax[3 * kRH + i]));
        const float mnew = fmaxf(mref[i], t);
        float alpha = 1.f;
        if (mnew > mref[i]) {
          alpha = (mref[i] == -INFINITY) ? 0.f : ex2(mref[i] - mnew);
          mref[i] = mnew;
        }
        lpart[i] *= alpha;
        o8[e] *= alpha;
      }
      if (rescale_o) {
        uint32_t ow[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ow[e] = __float_as_uint(o8[e]);
        ptx::tmem_st<8>(o_taddr + c8 * 8, ow);
      }
    }
    if (rescale_o) ptx::tmem_wait_st();
  }
  // P for this key (bf16, what the tensor core multiplies), row sums of the rounded values
  uint32_t w[kRH / 2];
#pragma unroll
  for (int h = 0; h < kRH / 2; ++h) {
    const float m0 = mref[2 * h] == -INFINITY ? 0.f : mref[2 * h];
    const float m1 = mref[2 * h + 1] == -INFINITY ? 0.f : mref[2 * h + 1];
    const __nv_bfloat162 hb = __floats2bfloat162_rn(ex2(x[2 * h] - m0), ex2(x[2 * h + 1] - m1));
    const float2 back = __bfloat1622float2(hb);
    lpart[2 * h] += back.x;
    lpart[2 * h + 1] += back.y;
    w[h] = *reinterpret_cast<const uint32_t *>(&hb);
  }
  // the single P^T buffer was last read by the P.V of tile gt - 1
  if (gt >= 1) {
    ptx::mbar_wait_inl(aux + kBarODone, (gt - 1) & 1, abort_flag);
    ptx::tc_fence_after();
  }
  // P^T row of key kk (MN-major, 64-byte swizzle): rows hf*16 .. hf*16 + 15 = chunks 2hf, 2hf+1
  st_shared_v4(sw64(pbase, kk, 2 * hf), w[0], w[1], w[2], w[3]);
  st_shared_v4(sw64(pbase, kk, 2 * hf + 1), w[4], w[5], w[6], w[7]);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tk_kernel(const __grid_constant__ CUtensorMap tmap_kv, const __grid_constant__ CUtensorMap tmap_kn,
               const __grid_constant__ CUtensorMap tmap_vn, AttnArgs a, int oob_row) {
  extern __shared__ __align__(1024) unsigned char tk_smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  const uint32_t raw_u32 = ptx::smem_u32(tk_smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  unsigned char *gbase = tk_smem_raw + (base - raw_u32);
  const uint32_t aux = base + kOffAux;
  unsigned char *gaux = gbase + kOffAux;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gaux + kAuxAbort);
  volatile int *s_last = reinterpret_cast<volatile int *>(gaux + kAuxLast);
  volatile int *s_split = reinterpret_cast<volatile int *>(gaux + kAuxSplit);  // [3]
  float *lsum_buf = reinterpret_cast<float *>(gaux + kAuxLsum);
  const uint32_t pbase = base + kOffP;
  // tile slot t of the K ring (v = 0) or of the V ring (v = 1): two page slots
  auto ring = [&](int v, uint32_t t) { return base + (uint32_t)v * kRingBytesK + t * kTileBytes; };
  auto qbuf = [&](int qb, int h) {
    return base + kOffQ + (uint32_t)qb * kQBufBytes + (uint32_t)h * kQHalfBytes;
  };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto bar = [&](uint32_t off, int i) { return aux + off + 8u * (uint32_t)i; };

  if (tid == 0) {
    // a tile's full barrier: one arrival (with its transaction bytes) per page producer
    for (int i = 0; i < kPairsK; ++i) {
      ptx::mbar_init(bar(kBarKFull, i), 2);
      ptx::mbar_init(bar(kBarKEmpty, i), 1);
    }
    for (int i = 0; i < kPairsV; ++i) {
      ptx::mbar_init(bar(kBarVFull, i), 2);
      ptx::mbar_init(bar(kBarVEmpty, i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(kBarSFree, i), kSoftmaxThreads);
      ptx::mbar_init(bar(kBarSFull, i), 1);
      ptx::mbar_init(bar(kBarQFull, i), 1);
      ptx::mbar_init(bar(kBarQEmpty, i), 1);
    }
    ptx::mbar_init(bar(kBarPFull, 0), kSoftmaxThreads);
    ptx::mbar_init(bar(kBarODone, 0), 1);
    ptx::mbar_init(bar(kBarOFree, 0), kSoftmaxThreads);
    ptx::mbar_init(bar(kBarDrain, 0), 1);
    ptx::mbar_init(bar(kBarDrain, 1), 1);
    *abort_flag = 0;
    *s_last = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kWarpK && lane == 0) {
    ptx::prefetch_tmap(&tmap_kv);
    ptx::prefetch_tmap(&tmap_kn);
    ptx::prefetch_tmap(&tmap_vn);
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(aux + kAuxTmem, kTmemCols);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(gaux + kAuxTmem);
  // Launched with programmatic stream serialisation: the prologue above overlaps the previous
  // kernel's tail; nothing written by an earlier kernel is read before this wait.  The next
  // launch may then start its own prologue as soon as SMs free up.
  ptx::grid_dependency_wait();
  ptx::grid_launch_dependents();
  if (warp >= kSoftmaxWarps) {
    // producers and issuers (warpgroups 2 and 3) hand registers to the softmax warpgroups
    ptx::setmaxnreg_dec<kRegsOther>();
    if (warp == kWarpK || warp == kWarpV || warp == kWarpK2 || warp == kWarpV2) {
      // ------------------------------------------------------------------ TMA producers
      // Two warps load K and two V, a tile (two pages) per ring slot and one barrier per tile:
      // producer hp of a ring loads page hp of every tile as one 4-D box (a warp issues about one
      // box per 850 cycles, so two per ring keep up with HBM at a power-capped clock) and arrives
      // with its bytes.  The whole warp walks the tiles; lane 0 waits on the barriers and issues
      // the copies.  The block-table entries come 32 at a time,
      // lane i holding entry base + i, and the chunk after the current one is loaded ahead, so a
      // page's lookup is a register shuffle and no copy waits on a dependent global load.  Tile gt
      // uses tile slot gt mod 3 of its ring.
      const bool is_k = (warp == kWarpK || warp == kWarpK2);
      const int hp = (warp == kWarpK2 || warp == kWarpV2) ? 1 : 0;  // the page of the tile
      const uint32_t full0 = is_k ? kBarKFull : kBarVFull, empty0 = is_k ? kBarKEmpty : kBarVEmpty;
      const int v = is_k ? 0 : 1;
      const CUtensorMap *nmap = is_k ? &tmap_kn : &tmap_vn;
      const int npairs = is_k ? kPairsK : kPairsV;
      // every cached page is read once per pass by one CTA: let it leave L2 first, so that the
      // split-KV partials written early in the kernel are still there when they are merged
      const uint64_t stream_policy = ptx::l2_policy_evict_first();
      int last_use[kMaxPairs];  // latest slot use that was armed, -1 if none
#pragma unroll
      for (int k = 0; k < kMaxPairs; ++k) last_use[k] = -1;
      auto bt_chunk = [&](int rr, int b0) -> int {
        const int i = b0 + lane;
        return (i < a.max_pages) ? __ldg(a.block_table + (size_t)rr * a.max_pages + i) : -1;
      };
      int creq = -1, cbase = 0, cval = -1, nbase = 0, nval = -1;
      // the page behind block-table index bi of request rr (a warp-wide call)
      auto page_of = [&](int rr, int bi) -> int {
        if (rr != creq || bi < cbase || bi >= cbase + 32) {
          if (rr == creq && bi >= nbase && bi < nbase + 32) {
            cbase = nbase;
            cval = nval;
          } else {
            cbase = bi;
            cval = bt_chunk(rr, cbase);
          }
          creq = rr;
          nbase = cbase + 32;
          nval = bt_chunk(rr, nbase);  // the next chunk, ahead of its use
        }
        return __shfl_sync(0xffffffffu, cval, bi - cbase);
      };
      TileCursor tc;
      tc.init(a);
      while (__shfl_sync(0xffffffffu, (tc.ok && !*abort_flag) ? 1 : 0, 0)) {
        const Meta &m = tc.p.m;
        const uint32_t slot = tc.gt % npairs;
        if (lane == 0) ptx::mbar_wait_inl(bar(empty0, slot), ((tc.gt / npairs) & 1) ^ 1, abort_flag);
        if (__shfl_sync(0xffffffffu, *abort_flag, 0) != 0) break;
        const uint32_t fb = bar(full0, slot), dst = ring(v, slot);
        if (tc.j < m.ncache) {
          const bool has = hp < min(2, m.npages - 2 * tc.j);  // the piece has this page
          const int key0 = (tc.p.ta + 2 * tc.j + hp) * kPage;
          const int page = has ? page_of(tc.p.r, key0 / a.page_size) : -1;
          if (lane == 0) {
            if (has) {
              ptx::mbar_arrive_expect_tx(fb, kPageBytes);
              int row = oob_row;
              if (page >= 0 && page < a.num_pages) {
                row = ((page * 2 + v) * a.Hkv + tc.p.g) * a.page_size + key0 % a.page_size;
              } else if (is_k) {
                raise_error(DSPARK_DERR_PAGE);
              }
              ptx::tma_load_4d_hint(dst + hp * kPageBytes, &tmap_kv, fb, 0, 0, 0, row >> 3,
                                    stream_policy);
            } else {
              ptx::mbar_arrive(fb);
            }
          }
        } else {  // the verify tokens: 16 rows of KV head g, a box of 8 tokens per producer
          if (lane == 0) {
            ptx::mbar_arrive_expect_tx(fb, kNewBytes / 2);
            ptx::tma_load_4d(dst + hp * kGroupBytes, nmap, fb, 0, m.t0 + 8 * hp, 0, tc.p.g);
          }
        }
        last_use[slot] = (int)tc.gt;
        tc.advance(a);
      }
      // never leave the CTA with a bulk copy in flight: wait for the latest armed use of every
      // slot (its phase is the newest one the slot's barrier can complete)
      if (lane == 0) {
        volatile int no_abort = 0;
        for (int k = 0; k < npairs; ++k)
          if (last_use[k] >= 0)
            ptx::mbar_wait_inl(bar(full0, k), ((uint32_t)last_use[k] / npairs) & 1, &no_abort);
      }
    } else if (warp == kWarpMma || warp == kWarpPV) {
      // ------------------------------------------------------------------ MMA issuers
      // One thread issues the S^T MMAs (warp 9), another the P.V MMAs (warp 11): each walks the
      // tiles in order and waits (bounded) on its own barriers, and the two overlap the per-issue
      // work that surrounds the MMAs.  They touch disjoint tensor memory (S^T buffers, O^T) and
      // shared memory (K ring and query rows, V ring and P^T); P.V(j) needs P^T(j), which the
      // softmax warps publish only after loading S^T(j).  S^T(j) overwrites the buffer of
      // S^T(j - 2), which the softmax warps release as soon as they have loaded it, so S^T(j + 2)
      // can go out while the softmax of tile j runs.
      if (lane == 0) {
        const bool is_s = (warp == kWarpMma);
        TileCursor c;
        c.init(a);
        // P^T as B: MN-major with 64-byte swizzle, 8 keys per 512-byte atom
        const uint64_t bd_p = ptx::smem_desc_sw64(pbase, 16, 512);
        uint32_t issued = 0;
        for (; c.ok; c.advance(a)) {
          if (is_s) {
            const uint32_t pair = c.gt % kPairsK, ph = (c.gt / kPairsK) & 1;
            const int qb = c.pq & 1;
            if (c.gt >= 2) ptx::mbar_wait(bar(kBarSFree, c.gt & 1), ((c.gt - 2) >> 1) & 1, abort_flag);
            if (c.j == 0) ptx::mbar_wait(bar(kBarQFull, qb), (c.pq >> 1) & 1, abort_flag);
            ptx::mbar_wait(bar(kBarKFull, pair), ph, abort_flag);
            if (*abort_flag) break;
            ptx::tc_fence_after();
            const uint32_t d_tmem = tmem + kColS + (c.gt & 1) * kN;
            // K tile as A (K-major: the keys on the lanes, groups of 8 keys 2048 bytes apart),
            // the rows as B (K-major); 16 d per k-step: 32 bytes within the 128-byte atom rows,
            // the d-halves 1024 bytes apart
            const uint64_t a0 = ptx::smem_desc_sw128(ring(0, pair), 16, kGroupBytes);
            const uint64_t a1 = ptx::smem_desc_sw128(ring(0, pair) + 1024, 16, kGroupBytes);
            const uint64_t b0 = ptx::smem_desc_sw128(qbuf(qb, 0), 16, 1024);
            const uint64_t b1 = ptx::smem_desc_sw128(qbuf(qb, 1), 16, 1024);
#pragma unroll
            for (int k = 0; k < kD / 16; ++k) {
              const uint64_t off = (uint64_t)((k & 3) * 2);
              ptx::mma_bf16_ss(d_tmem, (k < 4 ? a0 : a1) + off, (k < 4 ? b0 : b1) + off, kIdescS,
                               k > 0 ? 1u : 0u);
            }
            ptx::mma_commit(bar(kBarSFull, c.gt & 1));
            ptx::mma_commit(bar(kBarKEmpty, pair));
            // the pass's last S^T read of its rows: the buffer may be refilled
            if (c.j == c.p.m.ntiles - 1) ptx::mma_commit(bar(kBarQEmpty, qb));
          } else {
            const uint32_t pair = c.gt % kPairsV, ph = (c.gt / kPairsV) & 1;
            if (c.j == 0) ptx::mbar_wait(bar(kBarOFree, 0), (c.pq & 1) ^ 1, abort_flag);
            ptx::mbar_wait(bar(kBarPFull, 0), c.gt & 1, abort_flag);
            ptx::mbar_wait(bar(kBarVFull, pair), ph, abort_flag);
            if (*abort_flag) break;
            ptx::tc_fence_after();
            const Meta &m = c.p.m;
            const int jj = c.j;
            const int ksteps = (jj < m.ncache) ? (min(kTK, m.npages * kPage - jj * kTK) / 16)
                                               : kNewRows / 16;
            // V^T as A: MN-major (D on the lanes, d-halves 1024 bytes apart, groups of 8 keys
            // 2048 apart); fully unrolled k-steps with compile-time descriptor offsets (16 keys:
            // 4096 bytes of V, 1024 of P^T)
            const uint64_t ad0 = ptx::smem_desc_sw128(ring(1, pair), 1024, kGroupBytes);
            const uint32_t acc0 = jj > 0 ? 1u : 0u;
            if (ksteps == kTK / 16) {
#pragma unroll
              for (int k = 0; k < kTK / 16; ++k)
                ptx::mma_bf16_ss(tmem + kColO, ad0 + (uint64_t)(k * 256), bd_p + (uint64_t)(k * 64),
                                 kIdescPV, k > 0 ? 1u : acc0);
            } else if (ksteps == kPage / 16) {
#pragma unroll
              for (int k = 0; k < kPage / 16; ++k)
                ptx::mma_bf16_ss(tmem + kColO, ad0 + (uint64_t)(k * 256), bd_p + (uint64_t)(k * 64),
                                 kIdescPV, k > 0 ? 1u : acc0);
            } else {
              ptx::mma_bf16_ss(tmem + kColO, ad0, bd_p, kIdescPV, acc0);
            }
            ptx::mma_commit(bar(kBarODone, 0));
            ptx::mma_commit(bar(kBarVEmpty, pair));
          }
          ++issued;
        }
        // every MMA this thread issued has completed before the CTA releases shared memory and
        // TMEM, also after an abort (each issuer drains through its own barrier)
        if (issued > 0) {
          const uint32_t drain = bar(kBarDrain, is_s ? 0 : 1);
          ptx::mma_commit(drain);
          volatile int no_abort = 0;
          ptx::mbar_wait(drain, 0, &no_abort);
        }
      }
    }
  } else {
    ptx::setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax + epilogue
    const int q = warp & 3, hf = warp >> 2;
    const int kk = q * 32 + lane;  // key of the tile on this thread's TMEM lane (and d of O^T)
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q);
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.out);
    const int G = a.G;
    uint32_t gt = 0;
    int pidx = 0;  // index of the current pass among those with tiles

    // A pass's query rows (local row rl = segment row 32h + rl: token (32h + rl) / G, query
    // head g * G + (32h + rl) % G) into query buffer qb, K-major with 128-byte swizzle; rows
    // past the pass's are zeroed.
    auto q_prefetch = [&](const Pass &p, int qb) {
      const int r0 = p.h * kN, nr = min(kN, p.m.rows - r0);
      for (int idx = tid; idx < kN * 16; idx += kSoftmaxThreads) {
        const int rl = idx >> 4, h = (idx >> 3) & 1, c = idx & 7;
        const uint32_t dst = sw128(qbuf(qb, h), rl, c);
        if (rl < nr) {
          const int rr = r0 + rl, j = rr / G, i = rr % G;
          ptx::cp_async16(dst, qg + ((size_t)(p.m.t0 + j) * a.Hq + p.g * G + i) * kD + h * 64 + c * 8);
        } else {
          st_shared_v4(dst, 0u, 0u, 0u, 0u);
        }
      }
      ptx::cp_async_commit();
    };
    // every thread's copies have landed and are visible to the tensor core: the buffer is full
    auto q_publish = [&](int qb) {
      ptx::cp_async_wait_all();
      ptx::fence_proxy_async_smem();
      ptx::named_bar_sync(kBarAllSoftmax, kSoftmaxThreads);
      if (tid == 0) ptx::mbar_arrive(bar(kBarQFull, qb));
    };
    // before refilling the buffer of the pass with index p: the S^T MMAs of pass p - 2, its
    // previous user, are done
    auto q_wait_empty = [&](int p) {
      if (p >= 2) ptx::mbar_wait_inl(bar(kBarQEmpty, p & 1), ((p >> 1) - 1) & 1, abort_flag);
    };

    PassIter pit;
    pit.init(a);
    Pass cur;
    bool have = pit.first(a, cur, tid == 0);
    if (have && cur.m.ntiles > 0) {
      q_prefetch(cur, 0);
      q_publish(0);
    }
    while (have) {
      const Meta &m = cur.m;
      // look one pass ahead: its metadata now, its rows on their way into the other buffer
      Pass nxt;
      const bool have2 = pit.next(a, cur, nxt, tid == 0);
      const int pnext = pidx + (m.ntiles > 0 ? 1 : 0);
      if (have2 && nxt.m.ntiles > 0) {
        q_wait_empty(pnext);
        q_prefetch(nxt, pnext & 1);
      }
      const int r = cur.r, g = cur.g, ta = cur.ta, tb = cur.tb, tiles = cur.tiles, s0 = cur.s0;
      const bool whole = (ta == 0 && tb == tiles);
      const bool last_pass = cur.h + 1 == m.npass;
      const int r0 = cur.h * kN, nr = max(0, min(kN, m.rows - r0));
      // A split piece whose other pieces have all published by the time its last pass starts
      // merges without publishing its own partial; this early read keeps the counter's latency
      // off the epilogue.  tid 0 also finds the CTAs holding the segment's pieces.
      int pre_count = -1;
      if (tid == 0 && !whole && last_pass) {
        pre_count = ptx::ld_acquire_gpu(a.ws.counters + r * a.Hkv + g);
        const int c_first = ta == 0 ? (int)blockIdx.x : pit.it.rg.cta_of(s0);
        const int c_last = tb == tiles ? (int)blockIdx.x : pit.it.rg.cta_of(s0 + tiles - 1);
        s_split[0] = c_first;
        s_split[1] = c_last;
        s_split[2] = 2 * c_first + (s0 != pit.it.rg.start(c_first) ? 1 : 0);
      }

      float mref[kRH], lpart[kRH];
#pragma unroll
      for (int i = 0; i < kRH; ++i) {
        mref[i] = -INFINITY;
        lpart[i] = 0.f;
      }
      for (int j = 0; j < m.ntiles; ++j) {
        const uint32_t gt_ = gt + j;
        const bool cache_tile = j < m.ncache;
        // valid keys: the tile's pages that belong to this piece, cut at the cache length
        const int vk = cache_tile ? min(min(2, m.npages - 2 * j) * kPage, m.n - (ta + 2 * j) * kPage)
                                  : m.Q;
        ptx::mbar_wait_inl(bar(kBarSFull, gt_ & 1), (gt_ >> 1) & 1, abort_flag);
        ptx::tc_fence_after();
        softmax_tile(a, mref, lpart, tmem, lane_base, gaux, aux, abort_flag, gt_, vk, cache_tile,
                     kk, q, hf, lane, nr, kk * G - r0, pbase, j == 0);
        // V rows the P.V MMA reads past the valid keys may hold anything: zero them so that
        // P = 0 times V stays 0 (the MMA reads whole 16-key steps of valid pages)
        const int vrows = cache_tile ? min(kTK, (vk + kPage - 1) / kPage * kPage) : kNewRows;
        if (vk < vrows) {
          const uint32_t pair = gt_ % kPairsV;
          ptx::mbar_wait_inl(bar(kBarVFull, pair), (gt_ / kPairsV) & 1, abort_flag);
          for (int idx = tid; idx < (vrows - vk) * 16; idx += kSoftmaxThreads) {
            const uint32_t row = vk + idx / 16, half = (idx % 16) / 8, c = idx % 8;
            st_shared_v4(ring(1, pair) + (row >> 3) * kGroupBytes + half * 1024 + (row & 7) * 128 +
                             c * 16,
                         0u, 0u, 0u, 0u);
          }
        }
        ptx::fence_proxy_async_smem();  // P^T (and zeroed V rows) to the tensor core
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kBarPFull, 0));
        // the next pass's rows (prefetched at this pass's start) are published after its first
        // tile, so the S^T MMAs of the next pass run ahead of this pass's last tiles
        if (j == 0 && have2 && nxt.m.ntiles > 0) q_publish(pnext & 1);
      }
      if (m.ntiles == 0 && have2 && nxt.m.ntiles > 0) q_publish(pnext & 1);

      // ---------------------------------------------------------------- epilogue
      // Row sums: per row, the sum over the warp's keys by shuffles, over the four quadrants
      // through shared memory.  O^T: this thread's lane is d = kk, its columns its rows.
      float *ls = lsum_buf + hf * 4 * kRH;
      if (m.ntiles > 0) {
        // the 16 sums over the warp's lanes by halving exchanges (16 shuffles, not 80): at each
        // level a lane keeps one half of its values and adds the partner's copy of that half;
        // every sum takes the same pairs as a butterfly warp sum.  Row i ends in lanes 2i, 2i + 1.
#pragma unroll
        for (int w = kRH / 2, bit = 16; w >= 1; w >>= 1, bit >>= 1) {
          const bool up = (lane & bit) != 0;
#pragma unroll
          for (int k = 0; k < w; ++k) {
            const float send = up ? lpart[k] : lpart[k + w];
            const float keep = up ? lpart[k + w] : lpart[k];
            lpart[k] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
          }
        }
        lpart[0] += __shfl_xor_sync(0xffffffffu, lpart[0], 1);
        if ((lane & 1) == 0) ls[q * kRH + (lane >> 1)] = lpart[0];
        ptx::mbar_wait_inl(bar(kBarODone, 0), (gt + m.ntiles - 1) & 1, abort_flag);
        ptx::tc_fence_after();
      }
      if (tid == 0 && !whole && last_pass) {  // 2: merge at once (read after the next barrier)
        const int pieces = s_split[1] - s_split[0] + 1;
        *s_last = (pre_count == pieces - 1) ? 2 : 0;
      }
      ptx::named_bar_sync(kBarAllSoftmax, kSoftmaxThreads);
      // this CTA's partial slot for the segment: 2c for its first segment, 2c + 1 for one that
      // starts inside its range and continues past it
      float *part = a.ws.partials;
      if (!whole) {
        const bool inner = (ta == 0 && s0 != pit.it.rg.start(blockIdx.x));
        part += (size_t)(2 * (int)blockIdx.x + (inner ? 1 : 0)) * a.rows_max * kPS;
      }
      if (m.ntiles > 0) {
        float o[kRH];
        ptx::tmem_ld16(tmem + lane_base + kColO + hf * kRH, o);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kBarOFree, 0));  // O^T read: the next pass's P.V may overwrite it
        if (whole) {
          // the pass's output rows as bf16 [32 rows][128 d] in the P^T buffer (free: the last
          // P.V has completed, the next pass's first P^T comes after two barriers), then 16-byte
          // stores of whole rows: row rl is token (r0 + rl) / G, head (r0 + rl) % G of the group
#pragma unroll
          for (int i = 0; i < kRH; ++i) {
            const int rl = hf * kRH + i;
            const float l = ls[i] + ls[kRH + i] + ls[2 * kRH + i] + ls[3 * kRH + i];
            // l >= 1 (a visible row): its reference maximum is one of its own scores
            const __nv_bfloat16 v = __float2bfloat16_rn(rl < nr ? __fdividef(o[i], l) : 0.f);
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(pbase + (uint32_t)(rl * kD + kk) * 2u),
                         "h"(*reinterpret_cast<const unsigned short *>(&v))
                         : "memory");
          }
          ptx::named_bar_sync(kBarAllSoftmax, kSoftmaxThreads);
#pragma unroll
          for (int c = tid; c < kN * (kD / 8); c += kSoftmaxThreads) {
            const int rl = c / (kD / 8), ch = c % (kD / 8);
            if (rl < nr) {
              const uint4 w = ptx::ld_shared_v4(pbase + (uint32_t)(rl * kD + ch * 8) * 2u);
              const int rr = r0 + rl, jt = rr / G, ih = rr % G;
              *reinterpret_cast<uint4 *>(og + ((size_t)(m.t0 + jt) * a.Hq + g * G + ih) * kD +
                                         ch * 8) = w;
            }
          }
          ptx::named_bar_sync(kBarAllSoftmax, kSoftmaxThreads);
        } else {
#pragma unroll
          for (int i = 0; i < kRH; ++i) {
            const int rl = hf * kRH + i;
            if (rl < nr) {
              const float l = ls[i] + ls[kRH + i] + ls[2 * kRH + i] + ls[3 * kRH + i];
              const int rr = r0 + rl;
              part[(size_t)rr * kPS + kk] = o[i];
              if (kk == 0) {
                part[(size_t)rr * kPS + kD] = mref[i];
                part[(size_t)rr * kPS + kD + 1] = l;
              }
            }
          }
        }
        gt += m.ntiles;
      } else if (!whole) {
        // a piece holding only tail units of its segment: a partial without keys
        for (int idx = tid; idx < m.rows * kPS; idx += kSoftmaxThreads)
          part[idx] = (idx % kPS == kD) ? -INFINITY : 0.f;
      }

      if (!whole && last_pass) {  // split segment: publish the partial, the last piece merges
        const int c_first = s_split[0], c_last = s_split[1], slot_first = s_split[2];
        if (*s_last != 2) {
          __threadfence();
          ptx::named_bar_sync(kBarAllSoftmax, kSoftmaxThreads);
          if (tid == 0) {
            const int pieces = c_last - c_first + 1;
            const int prev = atomicAdd(a.ws.counters + r * a.Hkv + g, 1);
            *s_last = (prev == pieces - 1);
          }
        } else {
          // every other piece published before this one's last pass started (tid 0's acquire
          // read of the counter, ordered for the CTA by the barriers): no publish, no count; the
          // merge below reads this CTA's own partial after the barrier and resets the counter
        }
        ptx::named_bar_sync(kBarAllSoftmax, kSoftmaxThreads);
        if (*s_last) {
          __threadfence();
          const size_t pstride = (size_t)a.rows_max * kPS;
          const float *P0 = a.ws.partials;
          // items (row, float4 column), four per thread: each item merges the pieces online,
          // (m, l, values) of two pieces for all four items in flight at once, so that the usual
          // split (this piece and one other) costs a single round trip
          const int nitems = m.rows * (kD / 4);
          for (int it0 = tid; it0 < nitems; it0 += 4 * kSoftmaxThreads) {
            float4 acc[4];
            float Mi[4], Lsum[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
              Mi[k] = -INFINITY;
              Lsum[k] = 0.f;
            }
            for (int c2 = c_first; c2 <= c_last; c2 += 2) {
              float mp[2][4], lp[2][4];
              float4 v[2][4];
#pragma unroll
              for (int pc = 0; pc < 2; ++pc) {
                const int cc = min(c2 + pc, c_last);
                const float *Pp = P0 + (size_t)(cc == c_first ? slot_first : 2 * cc) * pstride;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const int item = min(it0 + k * kSoftmaxThreads, nitems - 1);
                  const int row = item / (kD / 4), d4 = item % (kD / 4);
                  mp[pc][k] = __ldcg(Pp + (size_t)row * kPS + kD);
                  lp[pc][k] = __ldcg(Pp + (size_t)row * kPS + kD + 1);
                  v[pc][k] = __ldcg(reinterpret_cast<const float4 *>(Pp + (size_t)row * kPS) + d4);
                }
              }
#pragma unroll
              for (int pc = 0; pc < 2; ++pc) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  if (c2 + pc <= c_last && mp[pc][k] != -INFINITY) {
                    const float Mn = fmaxf(Mi[k], mp[pc][k]);
                    const float so = ex2(Mi[k] - Mn), sp = ex2(mp[pc][k] - Mn);
                    Lsum[k] = Lsum[k] * so + lp[pc][k] * sp;
                    acc[k].x = acc[k].x * so + v[pc][k].x * sp;
                    acc[k].y = acc[k].y * so + v[pc][k].y * sp;
                    acc[k].z = acc[k].z * so + v[pc][k].z * sp;
                    acc[k].w = acc[k].w * so + v[pc][k].w * sp;
                    Mi[k] = Mn;
                  }
                }
              }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int item = it0 + k * kSoftmaxThreads;
              if (item < nitems) {
                const int row = item / (kD / 4), d4 = item % (kD / 4);
                const int jj = row / G, ii = row % G;
                const float li = 1.f / Lsum[k];
                uint2 w2;
                w2.x = ptx::pack_bf16x2(acc[k].x * li, acc[k].y * li);
                w2.y = ptx::pack_bf16x2(acc[k].z * li, acc[k].w * li);
                *reinterpret_cast<uint2 *>(og + ((size_t)(m.t0 + jj) * a.Hq + g * G + ii) * kD +
                                           d4 * 4) = w2;
              }
            }
          }
          if (tid == 0) a.ws.counters[r * a.Hkv + g] = 0;
        }
        ptx::named_bar_sync(kBarAllSoftmax, kSoftmaxThreads);
      }

      pidx = pnext;
      have = have2;
      if (have) cur = nxt;
    }
  }
  __syncthreads();
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tk
}  // namespace dspark
