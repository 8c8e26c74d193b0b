// Tensor-core verify attention for sm_100a (bf16, D = 128, page size a multiple of 64).
//
// Same work partition and split-KV merge as the CUDA-core kernel (attn_common.cuh): a persistent
// CTA per SM walks a contiguous range of (request, KV head, 64-key tile) units; every KV byte is
// read once for all G*Q_r query rows of its (request, KV head) — the flattened, unpadded verify
// batch of "刚融完500亿…专治AI“嘴慢”" (engineering table, row "内核利用率暴跌").
//
// Per CTA (192 threads):
//   warp 4      TMA producer: per tile, one 64-row x 128-B box per d-half of the page's K and V
//               tiles (128-byte swizzle) into a 4-stage shared-memory ring (32 KB per stage).
//   warp 5      MMA issuer (one thread): S = Q.K^T (M 128, N 64, K 128) into a double-buffered
//               TMEM tile, then O += P.V (M 128, N 128, K 64) into the piece's TMEM accumulator.
//   warps 0-3   softmax + epilogue.  TMEM lane quadrant w is readable only by warp w, so each
//               query row is replicated C times in the A operand (C = 4 for <= 32 rows, 2 for
//               <= 64, 1 otherwise): copy c lives in lanes [c*128/C, (c+1)*128/C) and its warps
//               handle keys [c*64/C, (c+1)*64/C) of every tile, which spreads the exp2 work of
//               a row over C SM sub-partitions.  Partial row maxima are exchanged through shared
//               memory (named barrier), P (bf16) is written to shared memory (128-byte swizzle)
//               for the P.V MMA, and O is rescaled in TMEM only when the running maximum grows by
//               more than 2^8.  The request's own verify tokens are one more tile at the end of
//               the segment: TMA loads their K/V rows through 3-D tensor maps over k_new/v_new
//               (16 tokens of one KV head) and the softmax applies the causal rule from the
//               markers (token j sees verify tokens 0..j).  The epilogue reads O from TMEM and
//               writes the output, or a split-KV partial that the last piece merges.
// The next piece's queries are staged as soon as the current piece's last S MMA has landed,
// before the current epilogue, so the tensor core and TMA keep streaming across pieces.
// Every mbarrier wait is bounded (ptx::mbar_wait); on timeout the CTA records
// DSPARK_DERR_TIMEOUT, skips the remaining work and still releases its TMEM.
#pragma once

#include "attn_generic.cuh"
#include "ptx_sm100.cuh"

namespace dspark {
namespace tc {

constexpr int kNK = 64;                              // keys per tile
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kD = 128;
constexpr uint32_t kHalfTile = 64 * 128;             // 64 rows x 128 B: one d-half of a K or V tile
constexpr uint32_t kStageBytes = 4 * kHalfTile;      // K h0 | K h1 | V h0 | V h1
constexpr uint32_t kQBytes = 2 * 128 * 128;          // 2 d-halves x 128 A-rows x 128 B
constexpr uint32_t kPBytes = 128 * 128;              // 128 A-rows x 64 keys x 2 B
constexpr uint32_t kOffQ = kStages * kStageBytes;
constexpr uint32_t kOffP = kOffQ + kQBytes;
constexpr uint32_t kOffAux = kOffP + 2 * kPBytes;
constexpr uint32_t kAuxBytes = 4096;
constexpr uint32_t kSmemBytes = kOffAux + kAuxBytes + 1024;  // + 1024-B alignment slack

// aux region layout (bytes)
constexpr uint32_t kBarKvFull = 0, kBarKvEmpty = 32, kBarSFull = 64, kBarPFull = 80,
                   kBarODone = 96, kBarQFull = 112, kBarQEmpty = 120, kBarOFree = 128;
constexpr uint32_t kAuxTmem = 160, kAuxAbort = 164, kAuxLast = 168, kAuxPmax = 256,
                   kAuxLsum = 256 + 2 * 128 * 4;

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // S tiles: columns [0, 64) and [64, 128)
constexpr uint32_t kColO = 256;   // O accumulators: [256, 384) and [384, 512)
constexpr float kRescaleLog2 = 8.f;

constexpr int kNewRows = 16;                         // verify tokens per new-token tile (K + 1 <= 16)
constexpr uint32_t kNewBytes = 4 * kNewRows * 128;   // K and V, two d-halves each

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, kNK, 0, 0);
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, kD, 0, 1);

struct Meta {
  int t0, Q, n, rows, C, ncache, ntiles;  // ntiles = cache tiles + the new-token tile
  bool valid, last, newtile;
};

// Serial validation of one piece; every role computes it identically.
__device__ __forceinline__ Meta piece_meta(const AttnArgs &a, int r, int ta, int tb, int tiles,
                                           bool raise) {
  Meta m;
  m.t0 = __ldg(a.q_offsets + r);
  m.Q = __ldg(a.q_offsets + r + 1) - m.t0;
  m.n = __ldg(a.kv_len + r);
  bool ok = (m.Q >= 1 && m.Q <= a.K + 1 && m.t0 >= 0 && m.t0 + m.Q <= a.T_cap);
  if (!ok && raise) raise_error(DSPARK_DERR_OFFSETS);
  const bool okn =
      (m.n >= 0 && (int64_t)(m.n + a.page_size - 1) / a.page_size <= a.max_pages);
  if (ok && !okn && raise) raise_error(DSPARK_DERR_KV_LEN);
  ok = ok && okn;
  if (ok) {
    for (int j = 0; j < m.Q; ++j) {
      if (__ldg(a.markers + 2 * (m.t0 + j)) != r ||
          __ldg(a.markers + 2 * (m.t0 + j) + 1) != m.n + j) {
        if (raise) raise_error(DSPARK_DERR_MARKER);
        ok = false;
        break;
      }
    }
  }
  m.valid = ok;
  m.rows = ok ? a.G * m.Q : 0;
  m.C = m.rows <= 32 ? 4 : (m.rows <= 64 ? 2 : 1);
  m.ncache = (ok && m.n > 0) ? (tb - ta) : 0;
  m.last = (tb == tiles);
  m.newtile = ok && m.last;
  m.ntiles = m.ncache + (m.newtile ? 1 : 0);
  return m;
}

struct PieceIter {
  int u, u1, W;
  __device__ __forceinline__ void init(const AttnArgs &a) {
    const int total = __ldg(a.ws.tile_prefix + a.R);
    W = (total + gridDim.x - 1) / gridDim.x;
    u = blockIdx.x * W;
    u1 = min(u + W, total);
  }
  __device__ __forceinline__ bool next(const AttnArgs &a, int &r, int &g, int &ta, int &tb,
                                       int &tiles, int &s0) {
    if (u >= u1) return false;
    find_segment(a.ws.tile_prefix, a.R, a.Hkv, u, r, g, tiles, s0);
    ta = u - s0;
    tb = min(tiles, ta + (u1 - u));
    u += tb - ta;
    return true;
  }
};

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

// Per-thread state of the softmax warps for the current piece.
struct SoftmaxState {
  float m_run;   // running row maximum (log2 domain) the P values of this piece are relative to
  float l_part;  // partial row sum over this copy's keys
};

// One tile for the thread's A-row t: S slice from TMEM, masking, row maximum across copies
// (named barrier 1), conditional O rescale, P (bf16) into shared memory.  NKC = keys per copy.
template <int NKC>
__device__ __forceinline__ void softmax_tile(const AttnArgs &a, SoftmaxState &st, uint32_t tmem,
                                             uint32_t lane_base, uint32_t base, uint32_t aux,
                                             float *pmax_buf, volatile int *abort_flag,
                                             uint32_t g_, int vk, int jrow, int t, int copy,
                                             int rho, int rpc, bool active, uint32_t ob) {
  constexpr int C = kNK / NKC;
  const uint32_t b = g_ & 1;
  float s[NKC];
  const uint32_t s_taddr = tmem + lane_base + kColS + b * kNK + copy * NKC;
#pragma unroll
  for (int c16 = 0; c16 < NKC / 16; ++c16) {
    float v[16];
    ptx::tmem_ld16(s_taddr + c16 * 16, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) s[c16 * 16 + i] = v[i];
  }
  ptx::tmem_wait_ld();
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < NKC; ++i) {
    const int key = copy * NKC + i;
    const float x = (key < vk && key <= jrow) ? s[i] * a.scale_log2 : -INFINITY;
    s[i] = x;
    mx = fmaxf(mx, x);
  }
  pmax_buf[b * 128 + t] = mx;
  ptx::named_bar_sync(1, kSoftmaxThreads);
  float mt = -INFINITY;
#pragma unroll
  for (int cc = 0; cc < C; ++cc) mt = fmaxf(mt, pmax_buf[b * 128 + rho + cc * rpc]);
  const float m_new = fmaxf(st.m_run, mt);
  float alpha = 1.f;
  bool resc = false;
  if (st.m_run == -INFINITY) {
    st.m_run = m_new;                    // first tile of the piece: O starts fresh
  } else if (m_new > st.m_run + kRescaleLog2) {
    alpha = ex2(st.m_run - m_new);
    st.m_run = m_new;
    st.l_part *= alpha;
    resc = true;
  }
  if (copy == 0 && __any_sync(0xffffffffu, resc)) {
    // O holds the earlier tiles relative to the old maximum: rescale it in TMEM once the
    // previous P.V has landed
    const uint32_t gp = g_ - 1;
    ptx::mbar_wait(aux + kBarODone + 8u * (gp & 1), (gp >> 1) & 1, abort_flag);
    ptx::tc_fence_after();
    const uint32_t o_taddr = tmem + lane_base + kColO + ob * 128;
#pragma unroll 1
    for (int c16 = 0; c16 < 8; ++c16) {
      float v[16];
      ptx::tmem_ld16(o_taddr + c16 * 16, v);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] *= alpha;
      ptx::tmem_st16(o_taddr + c16 * 16, v);
    }
    ptx::tmem_wait_st();
  }
  // P buffer b was last read by the P.V of tile g_ - 2
  if (g_ >= 2) ptx::mbar_wait(aux + kBarODone + 8u * b, ((g_ - 2) >> 1) & 1, abort_flag);
  const uint32_t p_row = base + kOffP + b * kPBytes + (uint32_t)rho * 128;
  float lsum = 0.f;
#pragma unroll
  for (int c8 = 0; c8 < NKC / 8; ++c8) {
    uint32_t w4[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float p0 = ex2(s[c8 * 8 + 2 * h] - st.m_run);
      const float p1 = ex2(s[c8 * 8 + 2 * h + 1] - st.m_run);
      const __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
      const float2 back = __bfloat1622float2(hb);
      lsum += back.x + back.y;
      w4[h] = *reinterpret_cast<const uint32_t *>(&hb);
    }
    if (active) {
      const uint32_t kc = (uint32_t)(copy * (NKC / 8) + c8);
      st_shared_v4(p_row + ((kc ^ ((uint32_t)rho & 7)) << 4), w4[0], w4[1], w4[2], w4[3]);
    }
  }
  st.l_part += lsum;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_kv, const __grid_constant__ CUtensorMap tmap_kn,
               const __grid_constant__ CUtensorMap tmap_vn, AttnArgs a, int oob_row) {
  extern __shared__ __align__(1024) unsigned char tc_smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzle atoms
  const uint32_t raw_u32 = ptx::smem_u32(tc_smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  unsigned char *gbase = tc_smem_raw + (base - raw_u32);
  const uint32_t aux = base + kOffAux;
  unsigned char *gaux = gbase + kOffAux;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gaux + kAuxAbort);
  float *pmax_buf = reinterpret_cast<float *>(gaux + kAuxPmax);
  float *lsum_buf = reinterpret_cast<float *>(gaux + kAuxLsum);
  volatile int *s_last = reinterpret_cast<volatile int *>(gaux + kAuxLast);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto bar = [&](uint32_t off, int i) { return aux + off + 8u * (uint32_t)i; };

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(bar(kBarKvFull, i), 1);
      ptx::mbar_init(bar(kBarKvEmpty, i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(kBarSFull, i), 1);
      ptx::mbar_init(bar(kBarPFull, i), kSoftmaxThreads);
      ptx::mbar_init(bar(kBarODone, i), 1);
      ptx::mbar_init(bar(kBarOFree, i), kSoftmaxThreads);
    }
    ptx::mbar_init(bar(kBarQFull, 0), kSoftmaxThreads);
    ptx::mbar_init(bar(kBarQEmpty, 0), 1);
    *abort_flag = 0;
    *s_last = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    ptx::prefetch_tmap(&tmap_kv);
    ptx::prefetch_tmap(&tmap_kn);
    ptx::prefetch_tmap(&tmap_vn);
  }
  if (warp == 5) {
    ptx::tmem_alloc(aux + kAuxTmem, kTmemCols);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(gaux + kAuxTmem);

  PieceIter it;
  it.init(a);
  int r, g, ta, tb, tiles, s0;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t gt = 0, issued = 0;
      while (it.next(a, r, g, ta, tb, tiles, s0)) {
        const Meta m = piece_meta(a, r, ta, tb, tiles, false);
        for (int j = 0; j < m.ntiles; ++j, ++gt) {
          const uint32_t st = gt % kStages;
          ptx::mbar_wait(bar(kBarKvEmpty, st), ((gt / kStages) & 1) ^ 1, abort_flag);
          if (*abort_flag) continue;
          const uint32_t sb = base + st * kStageBytes;
          const uint32_t fb = bar(kBarKvFull, st);
          if (j < m.ncache) {
            const int key0 = (ta + j) * kNK;
            const int page = __ldg(a.block_table + (size_t)r * a.max_pages + key0 / a.page_size);
            int rowK = oob_row, rowV = oob_row;
            if (page >= 0 && page < a.num_pages) {
              rowK = ((page * 2) * a.Hkv + g) * a.page_size + key0 % a.page_size;
              rowV = rowK + a.Hkv * a.page_size;
            } else {
              raise_error(DSPARK_DERR_PAGE);
            }
            ptx::mbar_arrive_expect_tx(fb, kStageBytes);
            ptx::tma_load_2d(sb, &tmap_kv, fb, 0, rowK);
            ptx::tma_load_2d(sb + kHalfTile, &tmap_kv, fb, 64, rowK);
            ptx::tma_load_2d(sb + 2 * kHalfTile, &tmap_kv, fb, 0, rowV);
            ptx::tma_load_2d(sb + 3 * kHalfTile, &tmap_kv, fb, 64, rowV);
          } else {  // the request's own verify tokens: 16 token rows of KV head g
            ptx::mbar_arrive_expect_tx(fb, kNewBytes);
            ptx::tma_load_3d(sb, &tmap_kn, fb, 0, g, m.t0);
            ptx::tma_load_3d(sb + kHalfTile, &tmap_kn, fb, 64, g, m.t0);
            ptx::tma_load_3d(sb + 2 * kHalfTile, &tmap_vn, fb, 0, g, m.t0);
            ptx::tma_load_3d(sb + 3 * kHalfTile, &tmap_vn, fb, 64, g, m.t0);
          }
          issued = gt + 1;
        }
      }
      // never leave the CTA with a bulk copy in flight: wait for the last use of every stage
      volatile int no_abort = 0;
      for (uint32_t k = 0; k < kStages && k < issued; ++k) {
        const uint32_t g_ = issued - 1 - k;
        ptx::mbar_wait(bar(kBarKvFull, g_ % kStages), (g_ / kStages) & 1, &no_abort);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t gt = 0, pq = 0;
      while (it.next(a, r, g, ta, tb, tiles, s0)) {
        const Meta m = piece_meta(a, r, ta, tb, tiles, false);
        if (m.ntiles == 0) continue;
        const uint32_t ob = pq & 1;
        ptx::mbar_wait(bar(kBarQFull, 0), pq & 1, abort_flag);
        ptx::mbar_wait(bar(kBarOFree, ob), ((pq >> 1) & 1) ^ 1, abort_flag);
        ptx::tc_fence_after();
        const uint32_t q_addr = base + kOffQ;
        auto issue_pv = [&](uint32_t g_, int jj) {
          ptx::mbar_wait(bar(kBarPFull, g_ & 1), (g_ >> 1) & 1, abort_flag);
          ptx::tc_fence_after();
          if (*abort_flag) return;
          const uint32_t p_addr = base + kOffP + (g_ & 1) * kPBytes;
          const uint32_t v_addr = base + (g_ % kStages) * kStageBytes + 2 * kHalfTile;
          const uint32_t d_tmem = tmem + kColO + ob * 128;
          const int ksteps = (jj < m.ncache) ? kNK / 16 : kNewRows / 16;
          for (int k = 0; k < ksteps; ++k) {
            const uint64_t ad = ptx::smem_desc_sw128(p_addr + k * 32, 16, 1024);
            const uint64_t bd = ptx::smem_desc_sw128(v_addr + k * 2048, kHalfTile, 1024);
            ptx::mma_bf16_ss(d_tmem, ad, bd, kIdescPV, (jj > 0 || k > 0) ? 1u : 0u);
          }
          ptx::mma_commit(bar(kBarODone, g_ & 1));
          ptx::mma_commit(bar(kBarKvEmpty, g_ % kStages));
        };
        for (int j = 0; j < m.ntiles; ++j) {
          const uint32_t g_ = gt + j;
          const uint32_t st = g_ % kStages;
          ptx::mbar_wait(bar(kBarKvFull, st), (g_ / kStages) & 1, abort_flag);
          ptx::tc_fence_after();
          if (!*abort_flag) {
            const uint32_t k_addr = base + st * kStageBytes;
            const uint32_t d_tmem = tmem + kColS + (g_ & 1) * kNK;
#pragma unroll
            for (int k = 0; k < kD / 16; ++k) {
              const uint32_t h = k >> 2, kk = k & 3;
              const uint64_t ad = ptx::smem_desc_sw128(q_addr + h * 16384 + kk * 32, 16, 1024);
              const uint64_t bd = ptx::smem_desc_sw128(k_addr + h * kHalfTile + kk * 32, 16, 1024);
              ptx::mma_bf16_ss(d_tmem, ad, bd, kIdescS, k > 0 ? 1u : 0u);
            }
            ptx::mma_commit(bar(kBarSFull, g_ & 1));
            // the piece's last S read of Q: the next piece may stage its queries
            if (j == m.ntiles - 1) ptx::mma_commit(bar(kBarQEmpty, 0));
          }
          if (j > 0) issue_pv(g_ - 1, j - 1);
        }
        issue_pv(gt + m.ntiles - 1, m.ntiles - 1);
        gt += m.ntiles;
        ++pq;
      }
      if (gt > 0 && !*abort_flag) {  // every MMA of this CTA has completed before TMEM is released
        volatile int no_abort = 0;
        ptx::mbar_wait(bar(kBarODone, (gt - 1) & 1), ((gt - 1) >> 1) & 1, &no_abort);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int t = tid;  // A-row of this thread (0..127)
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q);
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.out);
    const int G = a.G;
    uint32_t gt = 0, pq = 0, qidx = 0;

    // queries of a piece, replicated per copy, into the Q buffer once the previous piece's
    // last S MMA no longer reads it
    auto stage_q = [&](const Meta &mq, int gq) {
      const int rpcq = 128 / mq.C, rq = t % rpcq;
      ptx::mbar_wait(bar(kBarQEmpty, 0), (qidx & 1) ^ 1, abort_flag);
      if (rq < mq.rows) {
        const int j = rq / G, i = rq % G;
        const uint4 *src = reinterpret_cast<const uint4 *>(
            qg + ((size_t)(mq.t0 + j) * a.Hq + gq * G + i) * kD);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint4 v = __ldg(src + c);
          const uint32_t addr = base + kOffQ + (c >> 3) * 16384 + t * 128 +
                                ((((uint32_t)c & 7) ^ ((uint32_t)t & 7)) << 4);
          st_shared_v4(addr, v.x, v.y, v.z, v.w);
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(bar(kBarQFull, 0));
      ++qidx;
    };

    bool have = it.next(a, r, g, ta, tb, tiles, s0);
    Meta m;
    if (have) {
      m = piece_meta(a, r, ta, tb, tiles, t == 0);
      if (m.ntiles > 0) stage_q(m, g);
    }
    while (have) {
      const int rpc = 128 / m.C;         // A-rows per copy
      const int copy = t / rpc, rho = t % rpc;
      const bool active = m.valid && rho < m.rows;
      SoftmaxState sm;
      sm.m_run = -INFINITY;
      sm.l_part = 0.f;
      const uint32_t ob = pq & 1;
      for (int j = 0; j < m.ntiles; ++j) {
        const uint32_t g_ = gt + j;
        const uint32_t b = g_ & 1;
        const bool cache_tile = j < m.ncache;
        const int vk = cache_tile ? min(kNK, m.n - (ta + j) * kNK) : m.Q;  // valid keys
        const int jrow = cache_tile ? 0x7fffffff : rho / G;                // causal bound
        ptx::mbar_wait(bar(kBarSFull, b), (g_ >> 1) & 1, abort_flag);
        ptx::tc_fence_after();
        if (m.C == 4)
          softmax_tile<16>(a, sm, tmem, lane_base, base, aux, pmax_buf, abort_flag, g_, vk, jrow,
                           t, copy, rho, rpc, active, ob);
        else if (m.C == 2)
          softmax_tile<32>(a, sm, tmem, lane_base, base, aux, pmax_buf, abort_flag, g_, vk, jrow,
                           t, copy, rho, rpc, active, ob);
        else
          softmax_tile<64>(a, sm, tmem, lane_base, base, aux, pmax_buf, abort_flag, g_, vk, jrow,
                           t, copy, rho, rpc, active, ob);
        const int vrows = cache_tile ? kNK : kNewRows;  // V rows the P.V MMA reads
        if (vk < vrows) {
          // keys past the valid ones: their V rows may hold anything; zero them so that
          // P = 0 times V stays 0
          ptx::mbar_wait(bar(kBarKvFull, g_ % kStages), (g_ / kStages) & 1, abort_flag);
          const uint32_t v_addr = base + (g_ % kStages) * kStageBytes + 2 * kHalfTile;
          for (int idx = t; idx < (vrows - vk) * 16; idx += kSoftmaxThreads) {
            const uint32_t row = vk + idx / 16, half = (idx % 16) / 8, c = idx % 8;
            st_shared_v4(v_addr + half * kHalfTile + row * 128 + c * 16, 0u, 0u, 0u, 0u);
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kBarPFull, b));
      }

      // stage the next piece's queries now, so the MMAs of the next piece overlap this epilogue
      int r2, g2, ta2, tb2, tiles2, s02;
      const bool have2 = it.next(a, r2, g2, ta2, tb2, tiles2, s02);
      Meta m2;
      if (have2) {
        m2 = piece_meta(a, r2, ta2, tb2, tiles2, t == 0);
        if (m2.ntiles > 0) stage_q(m2, g2);
      }

      // ---------------------------------------------------------------- epilogue
      lsum_buf[t] = sm.l_part;
      ptx::named_bar_sync(2, kSoftmaxThreads);
      if (m.ntiles > 0) {
        const uint32_t gl = gt + m.ntiles - 1;
        ptx::mbar_wait(bar(kBarODone, gl & 1), (gl >> 1) & 1, abort_flag);
        ptx::tc_fence_after();
      }
      const bool whole = (ta == 0 && tb == tiles);
      const int W = it.W;
      float *part = a.ws.partials +
                    (size_t)partial_slot(blockIdx.x, s0, W) * a.rows_max * (kD + 2);
      if (copy == 0 && m.ntiles > 0) {  // warp-uniform: copy-0 warps own the O rows
        float l = 0.f;
        for (int cc = 0; cc < m.C; ++cc) l += lsum_buf[rho + cc * rpc];
        const int j = active ? rho / G : 0, i = active ? rho % G : 0;
        const size_t orow = ((size_t)(m.t0 + j) * a.Hq + g * G + i) * kD;
        const uint32_t o_taddr = tmem + lane_base + kColO + ob * 128;
        const float inv = 1.f / l;
#pragma unroll 1
        for (int c16 = 0; c16 < 8; ++c16) {
          float o[16];
          ptx::tmem_ld16(o_taddr + c16 * 16, o);
          ptx::tmem_wait_ld();
          if (active) {
            if (whole) {
              uint32_t w8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) w8[e] = ptx::pack_bf16x2(o[2 * e] * inv, o[2 * e + 1] * inv);
              uint4 *dst = reinterpret_cast<uint4 *>(og + orow + c16 * 16);
              dst[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
              dst[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
            } else {
              // rows are 130 floats apart: 8-byte aligned, so float2 stores
              float2 *dst = reinterpret_cast<float2 *>(part + (size_t)rho * (kD + 2) + c16 * 16);
#pragma unroll
              for (int e = 0; e < 8; ++e) dst[e] = make_float2(o[2 * e], o[2 * e + 1]);
            }
          }
        }
        if (active && !whole) {
          part[(size_t)rho * (kD + 2) + kD] = sm.m_run;
          part[(size_t)rho * (kD + 2) + kD + 1] = l;
        }
      }
      if (m.ntiles > 0) {
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kBarOFree, ob));
        gt += m.ntiles;
        ++pq;
      }

      if (!whole) {  // split segment: publish the partial, the last piece merges
        __threadfence();
        ptx::named_bar_sync(2, kSoftmaxThreads);
        if (t == 0) {
          const int pieces = (s0 + tiles - 1) / W - s0 / W + 1;
          const int prev = atomicAdd(a.ws.counters + r * a.Hkv + g, 1);
          *s_last = (prev == pieces - 1);
        }
        ptx::named_bar_sync(2, kSoftmaxThreads);
        if (*s_last) {
          __threadfence();
          const int c_first = s0 / W, c_last = (s0 + tiles - 1) / W;
          const size_t pstride = (size_t)a.rows_max * (kD + 2);
          const float *P0 = a.ws.partials;
          // per row: merged maximum and 1 / merged sum (threads t < rows)
          float *Ms = pmax_buf, *Li = lsum_buf;
          if (t < m.rows) {
            float M = -INFINITY;
            for (int cc = c_first; cc <= c_last; ++cc)
              M = fmaxf(M, __ldcg(P0 + (size_t)partial_slot(cc, s0, W) * pstride +
                                  (size_t)t * (kD + 2) + kD));
            float L = 0.f;
            for (int cc = c_first; cc <= c_last; ++cc) {
              const float *Pp = P0 + (size_t)partial_slot(cc, s0, W) * pstride + (size_t)t * (kD + 2);
              const float mp = __ldcg(Pp + kD);
              if (mp != -INFINITY) L += __ldcg(Pp + kD + 1) * ex2(mp - M);
            }
            Ms[t] = M;
            Li[t] = 1.f / L;
          }
          ptx::named_bar_sync(2, kSoftmaxThreads);
          // thread t owns head-dim column t; 8 rows at a time keep 8 x pieces loads in flight
          const int d = t;
          for (int row0 = 0; row0 < m.rows; row0 += 8) {
            float o[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) o[k] = 0.f;
            for (int cc = c_first; cc <= c_last; ++cc) {
              const float *Pp = P0 + (size_t)partial_slot(cc, s0, W) * pstride;
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int row = row0 + k;
                if (row < m.rows) {
                  const float mp = __ldcg(Pp + (size_t)row * (kD + 2) + kD);
                  const float v = __ldcg(Pp + (size_t)row * (kD + 2) + d);
                  if (mp != -INFINITY) o[k] = fmaf(v, ex2(mp - Ms[row]), o[k]);
                }
              }
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int row = row0 + k;
              if (row < m.rows) {
                const int jj = row / G, ii = row % G;
                og[((size_t)(m.t0 + jj) * a.Hq + g * G + ii) * kD + d] =
                    __float2bfloat16_rn(o[k] * Li[row]);
              }
            }
          }
          if (t == 0) a.ws.counters[r * a.Hkv + g] = 0;
        }
        ptx::named_bar_sync(2, kSoftmaxThreads);
      }

      have = have2;
      if (have) {
        m = m2;
        r = r2; g = g2; ta = ta2; tb = tb2; tiles = tiles2; s0 = s02;
      }
    }
  }

  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc
}  // namespace dspark
