// Tensor-core verify attention for sm_100a (bf16, D = 128, page size a multiple of 64,
// K + 1 <= 16, G * (K + 1) <= 64).
//
// Same work partition and split-KV merge as the CUDA-core kernel (attn_common.cuh): a persistent
// CTA per SM walks a contiguous range of (request, KV head, unit) work, the units of a segment
// being its 64-key cache tiles followed by one unit for the request's own verify tokens; every
// KV byte is read once for all G*Q_r query rows of its (request, KV head) — the flattened,
// unpadded verify batch of "刚融完500亿…专治AI“嘴慢”" (engineering table, row "内核利用率暴跌").
//
// A tcgen05 MMA costs about the same time whatever its N (up to 256) on B200, so the kernel
// minimises instructions per key: two 64-key pages form one 128-key tile, S = Q.K^T of a tile is
// 8 MMAs (M 128, N 128, K 16) and O += P.V is 8 MMAs (M 128, N 128, K 16).
//
// Per CTA (352 threads, 11 warps):
//   warp 8      TMA producer of K: per 64-key page, one 64-row x 128-B box per d-half (128-byte
//               swizzle) into two rings of 6 page slots; the two pages of a tile go to slots 2p
//               and 2p+1, which are contiguous, so one descriptor spans the tile.  An odd page
//               or the verify-token unit leaves slot 2p+1 empty.  Verify tokens come through
//               3-D tensor maps over k_new / v_new (16 tokens of one KV head).
//   warp 10     TMA producer of V (same layout, its own barriers: K is released after S, V only
//               after P.V).
//   warp 9      MMA issuer (one thread, polling): A operands (Q, P; bf16) in tensor memory, B
//               operands (K, V) in shared memory, fp32 accumulators in tensor memory.
//   warps 0-7   softmax + epilogue.  TMEM lane quadrant q is readable only by warps q and q + 4,
//               so each query row is replicated C times (C = 4 for <= 32 rows, else 2): copy c
//               lives in lanes [c*128/C, (c+1)*128/C) and handles keys [c*128/C, (c+1)*128/C) of
//               every tile, and the quadrant's two warps split those keys in halves, spreading
//               the exp2 work of a row over 2C warps.  Partial row maxima are exchanged through
//               shared memory (named barrier); each thread writes P for its keys (zeros for the
//               other copies' keys) into its lane's P columns, so every copy accumulates a
//               partial O over its keys and the epilogue sums the copies.  O is rescaled in
//               TMEM only when the running maximum grows by more than 2^8.  The verify-token
//               unit applies the causal rule from the markers (token j sees verify tokens 0..j).
// TMEM columns: S [0,256) (two 128-column tiles), Q [256,320), P [320,384), O [384,512).
// The next piece's queries are staged as soon as the current piece's last S MMA has landed,
// before the current epilogue, so the tensor core and TMA keep streaming across pieces.
// Every mbarrier wait is bounded (ptx::mbar_wait); on timeout the CTA records
// DSPARK_DERR_TIMEOUT, skips the remaining work and still releases its TMEM.
#pragma once

#include "attn_generic.cuh"
#include "ptx_sm100.cuh"

namespace dspark {
namespace tc {

constexpr int kPage = 64;                            // keys per page slot
constexpr int kTK = 128;                             // keys per tile (two page slots)
// page slots per K ring and per V ring (even: a tile takes two).  K is released as soon as S has
// been computed, V only after P.V, so V holds its slots longer.
constexpr int kSlotsK = 6, kSlotsV = 6;
constexpr int kPairsK = kSlotsK / 2, kPairsV = kSlotsV / 2;
constexpr int kMaxSlots = 8;
static_assert(kSlotsK % 2 == 0 && kSlotsV % 2 == 0 && kSlotsK <= kMaxSlots && kSlotsV <= kMaxSlots,
              "slot counts");
constexpr int kSoftmaxWarps = 8;                     // two per TMEM lane quadrant
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kWarpK = kSoftmaxWarps, kWarpMma = kSoftmaxWarps + 1, kWarpV = kSoftmaxWarps + 2;
constexpr int kThreads = kSoftmaxThreads + 96;
constexpr int kD = 128;
constexpr int kNewRows = 16;                         // verify tokens per unit (K + 1 <= 16)
constexpr uint32_t kSlotBytes = 64 * 128;            // 64 rows x 128 B: one d-half of a page
constexpr uint32_t kRingBytesK = kSlotsK * kSlotBytes;  // one K ring (d-half 0 or 1)
constexpr uint32_t kRingBytesV = kSlotsV * kSlotBytes;  // one V ring
constexpr uint32_t kHalfPageBytes = 2 * kSlotBytes;  // K (or V) of a page, both d-halves
constexpr uint32_t kNewHalfBytes = 2 * kNewRows * 128;  // K (or V) of the verify-token unit
constexpr uint32_t kOffAux = 2 * kRingBytesK + 2 * kRingBytesV;
constexpr uint32_t kAuxBytes = 4096;
// staging: the next piece's query rows (<= 64 x 256 B), then the epilogue's 128 x 32 fp32
constexpr uint32_t kOffStage = kOffAux + kAuxBytes;
constexpr uint32_t kStageBytes = 16384;
constexpr uint32_t kSmemBytes = kOffStage + kStageBytes + 1024;  // + alignment slack
constexpr int kPS = part_stride(kD);                 // floats per split-KV partial row

// aux region layout (bytes)
constexpr uint32_t kBarKFull = 0, kBarVFull = 64, kBarKEmpty = 128, kBarVEmpty = 192,
                   kBarSFull = 256, kBarPFull = 272, kBarODone = 280, kBarQFull = 288,
                   kBarQEmpty = 296, kBarOFree = 304, kBarDrain = 312;
constexpr uint32_t kAuxTmem = 320, kAuxAbort = 324, kAuxLast = 328, kAuxSplit = 336,
                   kAuxPmax = 512,
                   kAuxLsum = 512 + 2 * kSoftmaxThreads * 4;

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColQ = 256;
constexpr uint32_t kColP = 320;
constexpr uint32_t kColO = 384;
constexpr float kRescaleLog2 = 8.f;

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, kTK, 0, 0);  // Q (K-major) x K^T
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, kD, 0, 1);  // P (K-major) x V (MN-major)

struct Meta {
  int t0, Q, n, rows, C, npages, ncache, ntiles;  // npages: cache pages of the piece
  bool valid, last, newtile;                      // ncache: their 128-key tiles
};

// Metadata of one piece [ta, tb) of a segment with `tiles` units, from the plan's per-request
// record (one 16-byte load); every role computes it identically.
__device__ __forceinline__ Meta piece_meta(const AttnArgs &a, int r, int ta, int tb, int tiles,
                                           bool raise) {
  Meta m;
  const int4 rec = __ldg(a.ws.req + r);
  m.t0 = rec.x;
  m.Q = rec.y;
  m.n = rec.z;
  bool ok = rec.w != 0;
  const bool okn = (int64_t)(m.n + a.page_size - 1) / a.page_size <= a.max_pages;
  if (ok && !okn && raise) raise_error(DSPARK_DERR_KV_LEN);
  ok = ok && okn;
  m.valid = ok;
  m.rows = ok ? a.G * m.Q : 0;
  m.C = m.rows <= 32 ? 4 : 2;
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
  __device__ __forceinline__ void init(const AttnArgs &a) {
    const int total = __ldg(&a.ws.hdr->total);
    const int ctas = __ldg(&a.ws.hdr->tc_ctas);
    if (ctas == (int)gridDim.x) {  // the plan's cost-balanced ranges
      rg.begin = a.ws.cta_begin;
      rg.W = 0;
      rg.ctas = ctas;
      rg.total = total;
      const int4 st = __ldg(a.ws.cta_start + blockIdx.x);
      r = st.x; g = st.y; s0 = st.z; tiles = st.w;
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

// Walks the tiles of this CTA's pieces in order (pieces without tiles are skipped).  gt = global
// tile index of the CTA, pq = index of the current piece among the pieces with tiles.
struct TileCursor {
  PieceIter it;
  Meta m;
  int r, g, ta, tb, tiles, s0, j;
  uint32_t gt, pq;
  bool ok;
  __device__ __forceinline__ bool next_piece(const AttnArgs &a) {
    while (it.next(a, r, g, ta, tb, tiles, s0)) {
      m = piece_meta(a, r, ta, tb, tiles, false);
      if (m.ntiles > 0) {
        j = 0;
        return true;
      }
    }
    return false;
  }
  __device__ __forceinline__ void init(const AttnArgs &a) {
    it.init(a);
    gt = 0;
    pq = 0;
    ok = next_piece(a);
  }
  __device__ __forceinline__ void advance(const AttnArgs &a) {
    ++gt;
    if (++j == m.ntiles) {
      ++pq;
      ok = next_piece(a);
    }
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

// One tile for the thread's lane and key half: S slice from TMEM, masking (valid keys, causal
// bound), row maximum across copies and halves (named barrier 1), conditional rescale of this
// thread's half of the lane's O, P (bf16) for its keys into the lane's P columns.  NKC = keys per
// copy (each of the quadrant's two warps takes NKC / 2 of them).  `gt` = global tile index.
template <int NKC>
__device__ __forceinline__ void softmax_tile(const AttnArgs &a, SoftmaxState &st, uint32_t tmem,
                                             uint32_t lane_base, uint32_t aux, float *pmax_buf,
                                             volatile int *abort_flag, uint32_t gt, int vk,
                                             int jrow, int t, int hf, int copy, int rho, int rpc,
                                             bool active) {
  constexpr int C = kTK / NKC;
  constexpr int NKH = NKC / 2;
  const uint32_t b = gt & 1;
  float s[NKH];
  const int key0 = copy * NKC + hf * NKH;
  const uint32_t s_taddr = tmem + lane_base + kColS + b * kTK + key0;
#pragma unroll
  for (int c16 = 0; c16 < NKH / 16; ++c16) {
    float v[16];
    ptx::tmem_ld16(s_taddr + c16 * 16, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) s[c16 * 16 + i] = v[i];
  }
  ptx::tmem_wait_ld();
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < NKH; ++i) {
    const int key = key0 + i;
    const float x = (active && key < vk && key <= jrow) ? s[i] * a.scale_log2 : -INFINITY;
    s[i] = x;
    mx = fmaxf(mx, x);
  }
  pmax_buf[b * kSoftmaxThreads + hf * 128 + t] = mx;
  ptx::named_bar_sync(1, kSoftmaxThreads);
  float mt = -INFINITY;
#pragma unroll
  for (int cc = 0; cc < C; ++cc) {
    mt = fmaxf(mt, pmax_buf[b * kSoftmaxThreads + rho + cc * rpc]);
    mt = fmaxf(mt, pmax_buf[b * kSoftmaxThreads + 128 + rho + cc * rpc]);
  }
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
  // compute P before waiting for the tensor core
  float lsum = 0.f;
  uint32_t w[NKH / 2];
#pragma unroll
  for (int h = 0; h < NKH / 2; ++h) {
    const float p0 = active ? ex2(s[2 * h] - st.m_run) : 0.f;
    const float p1 = active ? ex2(s[2 * h + 1] - st.m_run) : 0.f;
    const __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
    const float2 back = __bfloat1622float2(hb);
    lsum += back.x + back.y;
    w[h] = *reinterpret_cast<const uint32_t *>(&hb);
  }
  st.l_part += lsum;
  // the single P tile and this lane's O were last used by the P.V of tile gt - 1
  if (gt >= 1) {
    ptx::mbar_wait(aux + kBarODone, (gt - 1) & 1, abort_flag);
    ptx::tc_fence_after();
  }
  if (__any_sync(0xffffffffu, resc)) {
    // this lane's O holds the earlier tiles relative to the old maximum: rescale it in TMEM
    // (each of the quadrant's two warps takes half of the columns)
    const uint32_t o_taddr = tmem + lane_base + kColO + hf * 64;
#pragma unroll 1
    for (int c32 = 0; c32 < 2; ++c32) {
      float v[32];
      ptx::tmem_ld32(o_taddr + c32 * 32, v);
      ptx::tmem_wait_ld();
      uint32_t ow[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) ow[i] = __float_as_uint(v[i] * alpha);
      ptx::tmem_st<32>(o_taddr + c32 * 32, ow);
    }
  }
  ptx::tmem_st<NKH / 2>(tmem + lane_base + kColP + key0 / 2, w);
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
  const uint32_t stage = base + kOffStage;
  volatile int *s_last = reinterpret_cast<volatile int *>(gaux + kAuxLast);
  volatile int *s_split = reinterpret_cast<volatile int *>(gaux + kAuxSplit);  // [3]
  // ring r (0 = K d-half 0, 1 = K d-half 1, 2 = V d-half 0, 3 = V d-half 1), page slot s
  auto ring = [&](int rg, uint32_t s) {
    return base + (rg < 2 ? (uint32_t)rg * kRingBytesK
                          : 2 * kRingBytesK + (uint32_t)(rg - 2) * kRingBytesV) + s * kSlotBytes;
  };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto bar = [&](uint32_t off, int i) { return aux + off + 8u * (uint32_t)i; };

  if (tid == 0) {
    for (int i = 0; i < kSlotsK; ++i) {
      ptx::mbar_init(bar(kBarKFull, i), 1);
      ptx::mbar_init(bar(kBarKEmpty, i), 1);
    }
    for (int i = 0; i < kSlotsV; ++i) {
      ptx::mbar_init(bar(kBarVFull, i), 1);
      ptx::mbar_init(bar(kBarVEmpty, i), 1);
    }
    for (int i = 0; i < 2; ++i) ptx::mbar_init(bar(kBarSFull, i), 1);
    ptx::mbar_init(bar(kBarPFull, 0), kSoftmaxThreads);
    ptx::mbar_init(bar(kBarODone, 0), 1);
    ptx::mbar_init(bar(kBarQFull, 0), kSoftmaxThreads);
    ptx::mbar_init(bar(kBarQEmpty, 0), 1);
    ptx::mbar_init(bar(kBarOFree, 0), kSoftmaxThreads);
    ptx::mbar_init(bar(kBarDrain, 0), 1);
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

  PieceIter it;
  it.init(a);
  int r, g, ta, tb, tiles, s0;

  if (warp == kWarpK || warp == kWarpV) {
    // ------------------------------------------------------------------ TMA producers
    // one warp loads K, another V (a bulk L2 prefetch of later pages was tried and only
    // lengthened the loads' latency).  Tile gt uses page slots 2(gt mod 3) and 2(gt mod 3) + 1
    // of both rings' families.  The whole warp walks the tiles; lane 0 waits on the barriers
    // and issues the copies.  The block-table entries come 32 at a time, lane i holding entry
    // base + i, and the chunk after the current one is loaded ahead: a page's lookup is a
    // register shuffle, so no copy waits for a dependent global load (under the kernel's own
    // traffic that load took about 1000 cycles and held back every page's copy).
    const bool is_k = (warp == kWarpK);
    const uint32_t full0 = is_k ? kBarKFull : kBarVFull, empty0 = is_k ? kBarKEmpty : kBarVEmpty;
    const int rg0 = is_k ? 0 : 2;
    const CUtensorMap *nmap = is_k ? &tmap_kn : &tmap_vn;
    const int nslots = is_k ? kSlotsK : kSlotsV;
    // every cached page is read by exactly one CTA once: let it leave L2 first, so that the
    // split-KV partials written early in the kernel are still there when they are merged
    const uint64_t stream_policy = ptx::l2_policy_evict_first();
    int last_use[kMaxSlots];  // latest slot use that was armed (TMA or empty arrive), -1 if none
#pragma unroll
    for (int k = 0; k < kMaxSlots; ++k) last_use[k] = -1;
    auto bt_chunk = [&](int rr, int base) -> int {
      const int i = base + lane;
      return (i < a.max_pages) ? __ldg(a.block_table + (size_t)rr * a.max_pages + i) : -1;
    };
    int creq = -1, cbase = 0, cval = -1, nbase = 0, nval = -1;
    TileCursor tc;
    tc.init(a);
    while (__shfl_sync(0xffffffffu, (tc.ok && !*abort_flag) ? 1 : 0, 0)) {
      const Meta &m = tc.m;
      bool stop = false;
      for (int h = 0; h < 2; ++h) {   // the tile's two page slots
        const uint32_t sl = 2 * tc.gt + h, slot = sl % nslots;
        if (lane == 0) ptx::mbar_wait(bar(empty0, slot), ((sl / nslots) & 1) ^ 1, abort_flag);
        stop = __shfl_sync(0xffffffffu, *abort_flag, 0) != 0;
        if (stop) break;
        const uint32_t fb = bar(full0, slot);
        const int pg = 2 * tc.j + h;     // page of the piece in this slot
        if (tc.j < m.ncache && pg < m.npages) {
          const int key0 = (tc.ta + pg) * kPage;
          const int bi = key0 / a.page_size;  // block-table index of the page
          if (tc.r != creq || bi < cbase || bi >= cbase + 32) {
            if (tc.r == creq && bi >= nbase && bi < nbase + 32) {
              cbase = nbase;
              cval = nval;
            } else {
              cbase = bi;
              cval = bt_chunk(tc.r, cbase);
            }
            creq = tc.r;
            nbase = cbase + 32;
            nval = bt_chunk(tc.r, nbase);  // the next chunk, ahead of its use
          }
          const int page = __shfl_sync(0xffffffffu, cval, bi - cbase);
          if (lane == 0) {
            int row = oob_row;
            if (page >= 0 && page < a.num_pages) {
              row = ((page * 2 + (is_k ? 0 : 1)) * a.Hkv + tc.g) * a.page_size + key0 % a.page_size;
            } else if (is_k) {
              raise_error(DSPARK_DERR_PAGE);
            }
            ptx::mbar_arrive_expect_tx(fb, kHalfPageBytes);
            ptx::tma_load_2d_hint(ring(rg0, slot), &tmap_kv, fb, 0, row, stream_policy);
            ptx::tma_load_2d_hint(ring(rg0 + 1, slot), &tmap_kv, fb, 64, row, stream_policy);
          }
        } else if (tc.j == m.ncache && h == 0) {  // the verify tokens: 16 rows of KV head g
          if (lane == 0) {
            ptx::mbar_arrive_expect_tx(fb, kNewHalfBytes);
            ptx::tma_load_3d(ring(rg0, slot), nmap, fb, 0, tc.g, m.t0);
            ptx::tma_load_3d(ring(rg0 + 1, slot), nmap, fb, 64, tc.g, m.t0);
          }
        } else {
          if (lane == 0) ptx::mbar_arrive(fb);  // empty slot: completes its phase without data
        }
        last_use[slot] = (int)sl;
      }
      if (stop) break;
      tc.advance(a);
    }
    // never leave the CTA with a bulk copy in flight: wait for the latest armed use of every
    // slot (its phase is the newest one the slot's barrier can complete)
    if (lane == 0) {
      volatile int no_abort = 0;
      for (int k = 0; k < nslots; ++k)
        if (last_use[k] >= 0)
          ptx::mbar_wait(bar(full0, k), ((uint32_t)last_use[k] / nslots) & 1, &no_abort);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    // Two cursors: S(js) for the next tile whose K has landed, P.V(jp) for the oldest tile whose
    // P is written.  Whichever is ready is issued (P.V first), so a late K load never holds back
    // the P.V of an earlier tile.  S runs at most one tile ahead of P.V (two S buffers: S(js)
    // overwrites S(js - 2), which the softmax warps have read once P(js - 2) is published).
    if (lane == 0) {
      TileCursor cs, cp;
      cs.init(a);
      cp.init(a);
      long long idle_since = clock64();
      while (cp.ok && !*abort_flag) {
        bool progress = false;
        if (cp.gt < cs.gt) {
          const uint32_t pair = cp.gt % kPairsV, ph = (cp.gt / kPairsV) & 1;
          if ((cp.j > 0 || ptx::mbar_test(bar(kBarOFree, 0), (cp.pq & 1) ^ 1)) &&
              ptx::mbar_test(bar(kBarPFull, 0), cp.gt & 1) &&
              ptx::mbar_test(bar(kBarVFull, 2 * pair), ph) &&
              ptx::mbar_test(bar(kBarVFull, 2 * pair + 1), ph)) {
            ptx::tc_fence_after();
            const Meta &m = cp.m;
            const int jj = cp.j;
            const int ksteps = (jj < m.ncache) ? (min(kTK, m.npages * kPage - jj * kTK) / 16)
                                               : kNewRows / 16;
            // fully unrolled k-steps with compile-time descriptor offsets: the issue rate of
            // tcgen05.mma drops several-fold when its operands are formed in a run-time loop
            const uint64_t bd0 = ptx::smem_desc_sw128(ring(2, 2 * pair), kRingBytesV, 1024);
            const uint32_t acc0 = jj > 0 ? 1u : 0u;
            if (ksteps == kTK / 16) {
#pragma unroll
              for (int k = 0; k < kTK / 16; ++k)
                ptx::mma_bf16_ts(tmem + kColO, tmem + kColP + k * 8, bd0 + (uint64_t)(k * 128),
                                 kIdescPV, k > 0 ? 1u : acc0);
            } else if (ksteps == kPage / 16) {
#pragma unroll
              for (int k = 0; k < kPage / 16; ++k)
                ptx::mma_bf16_ts(tmem + kColO, tmem + kColP + k * 8, bd0 + (uint64_t)(k * 128),
                                 kIdescPV, k > 0 ? 1u : acc0);
            } else {
              ptx::mma_bf16_ts(tmem + kColO, tmem + kColP, bd0, kIdescPV, acc0);
            }
            ptx::mma_commit(bar(kBarODone, 0));
            ptx::mma_commit(bar(kBarVEmpty, 2 * pair));
            ptx::mma_commit(bar(kBarVEmpty, 2 * pair + 1));
            cp.advance(a);
            progress = true;
          }
        }
        if (!progress && cs.ok && cs.gt <= cp.gt + 1) {
          const uint32_t pair = cs.gt % kPairsK, ph = (cs.gt / kPairsK) & 1;
          if ((cs.j > 0 || ptx::mbar_test(bar(kBarQFull, 0), cs.pq & 1)) &&
              ptx::mbar_test(bar(kBarKFull, 2 * pair), ph) &&
              ptx::mbar_test(bar(kBarKFull, 2 * pair + 1), ph)) {
            ptx::tc_fence_after();
            const uint32_t d_tmem = tmem + kColS + (cs.gt & 1) * kTK;
#pragma unroll
            for (int k = 0; k < kD / 16; ++k) {
              const uint32_t h = k >> 2, kk = k & 3;
              const uint64_t bd = ptx::smem_desc_sw128(ring(h, 2 * pair) + kk * 32, 16, 1024);
              ptx::mma_bf16_ts(d_tmem, tmem + kColQ + k * 8, bd, kIdescS, k > 0 ? 1u : 0u);
            }
            ptx::mma_commit(bar(kBarSFull, cs.gt & 1));
            ptx::mma_commit(bar(kBarKEmpty, 2 * pair));
            ptx::mma_commit(bar(kBarKEmpty, 2 * pair + 1));
            // the piece's last S read of Q: the next piece may stage its queries
            if (cs.j == cs.m.ntiles - 1) ptx::mma_commit(bar(kBarQEmpty, 0));
            cs.advance(a);
            progress = true;
          }
        }
        if (progress) {
          idle_since = clock64();
        } else if (clock64() - idle_since > ptx::kWaitLimitCycles) {
          *abort_flag = 1;
          raise_error(DSPARK_DERR_TIMEOUT);
        }
      }
      // Every MMA this thread issued has completed before the CTA releases its shared memory
      // and TMEM, also after an abort (which can leave S MMAs issued after the last P.V): one
      // more commit tracks all of them, and its wait is bounded but ignores the abort flag.
      if (cs.gt > 0 || cp.gt > 0) {
        ptx::mma_commit(bar(kBarDrain, 0));
        volatile int no_abort = 0;
        ptx::mbar_wait(bar(kBarDrain, 0), 0, &no_abort);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int t = tid & 127;   // TMEM lane of this thread (its warp's lane quadrant)
    const int hf = tid >> 7;   // which half of each copy's keys (and of O's columns) it takes
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(a.q);
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.out);
    const int G = a.G;
    uint32_t gt = 0, qidx = 0;

    // A piece's query rows (row rq = j * G + i: token j, query head g * G + i) into the staging
    // area with asynchronous 16-byte copies, chunk c of row rq at chunk slot c ^ (rq & 7) so the
    // lane-per-row reads of q_commit spread over the banks.
    auto q_prefetch = [&](const Meta &mq, int gq) {
      for (int idx = tid; idx < mq.rows * 16; idx += kSoftmaxThreads) {
        const int rq = idx >> 4, c = idx & 15;
        const int j = rq / G, i = rq % G;
        ptx::cp_async16(stage + rq * 256 + ((c ^ (rq & 7)) << 4),
                        qg + ((size_t)(mq.t0 + j) * a.Hq + gq * G + i) * kD + c * 8);
      }
      ptx::cp_async_commit();
    };
    // Staged rows into this lane's Q columns (replicated per copy; inactive lanes get zeros) once
    // the previous piece's last S MMA no longer reads them.
    auto q_commit = [&](const Meta &mq) {
      ptx::cp_async_wait_all();
      ptx::named_bar_sync(1, kSoftmaxThreads);  // every thread's copies have landed
      const int rq = t % (128 / mq.C);
      ptx::mbar_wait(bar(kBarQEmpty, 0), (qidx & 1) ^ 1, abort_flag);
      ptx::tc_fence_after();
      {  // this thread writes the lane's Q columns of d-half hf
        const int h = hf;
        uint32_t w[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (rq < mq.rows) v = ptx::ld_shared_v4(stage + rq * 256 + (((h * 8 + c) ^ (rq & 7)) << 4));
          w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
        }
        ptx::tmem_st<32>(tmem + lane_base + kColQ + h * 32, w);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(kBarQFull, 0));
      ++qidx;
      ptx::named_bar_sync(1, kSoftmaxThreads);  // every lane has read the staging area
    };

    bool have = it.next(a, r, g, ta, tb, tiles, s0);
    Meta m;
    if (have) {
      m = piece_meta(a, r, ta, tb, tiles, tid == 0);
      if (m.ntiles > 0) {
        q_prefetch(m, g);
        q_commit(m);
      }
    }
    while (have) {
      // look one piece ahead: its metadata now, its queries on their way into the staging area
      // while this piece's tiles stream
      int r2, g2, ta2, tb2, tiles2, s02;
      const bool have2 = it.next(a, r2, g2, ta2, tb2, tiles2, s02);
      Meta m2;
      if (have2) {
        m2 = piece_meta(a, r2, ta2, tb2, tiles2, tid == 0);
        if (m2.ntiles > 0) q_prefetch(m2, g2);
      }

      const int rpc = 128 / m.C;         // lanes per copy
      const int copy = t / rpc, rho = t % rpc;
      const bool active = m.valid && rho < m.rows;
      // A split piece whose other pieces have all published by the time it starts (nearly every
      // CTA's last piece: the next CTA took the segment's rest first) merges without publishing
      // its own partial; this early read keeps the counter's latency off the epilogue.
      const bool split = !(ta == 0 && tb == tiles);
      int pre_count = -1;
      if (tid == 0 && split) {
        pre_count = ptx::ld_acquire_gpu(a.ws.counters + r * a.Hkv + g);
        // the CTAs holding this segment's pieces and the slot of its first piece's partial
        // (read by everyone after the epilogue's first barrier)
        const int c_first = ta == 0 ? (int)blockIdx.x : it.rg.cta_of(s0);
        const int c_last = tb == tiles ? (int)blockIdx.x : it.rg.cta_of(s0 + tiles - 1);
        s_split[0] = c_first;
        s_split[1] = c_last;
        s_split[2] = 2 * c_first + (s0 != it.rg.start(c_first) ? 1 : 0);
      }
      SoftmaxState sm;
      sm.m_run = -INFINITY;
      sm.l_part = 0.f;
      for (int j = 0; j < m.ntiles; ++j) {
        const uint32_t gt_ = gt + j;
        const bool cache_tile = j < m.ncache;
        // valid keys: the tile's pages that belong to this piece, cut at the cache length
        const int vk = cache_tile ? min(min(2, m.npages - 2 * j) * kPage, m.n - (ta + 2 * j) * kPage)
                                  : m.Q;
        const int jrow = cache_tile ? 0x7fffffff : rho / G;                      // causal bound
        ptx::mbar_wait(bar(kBarSFull, gt_ & 1), (gt_ >> 1) & 1, abort_flag);
        ptx::tc_fence_after();
        if (j == 0) {
          // this lane's P columns outside its copy's keys must read as zero (the previous
          // piece's P.V MMAs have completed: its epilogue waited for them).  Each of the
          // quadrant's two warps zeroes its own key half of the other copies, so the two never
          // write the same columns.
          uint32_t z[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) z[c] = 0u;
          const int ph = kTK / m.C / 4;  // P columns of one copy's key half (8 or 16)
          for (int cc = 0; cc < m.C; ++cc) {
            if (cc == copy) continue;
            const uint32_t col = tmem + lane_base + kColP + cc * 2 * ph + hf * ph;
            if (ph == 8) {
              uint32_t z8[8];
#pragma unroll
              for (int c = 0; c < 8; ++c) z8[c] = 0u;
              ptx::tmem_st<8>(col, z8);
            } else {
              ptx::tmem_st<16>(col, z);
            }
          }
        }
        if (m.C == 4)
          softmax_tile<32>(a, sm, tmem, lane_base, aux, pmax_buf, abort_flag, gt_, vk, jrow, t,
                           hf, copy, rho, rpc, active);
        else
          softmax_tile<64>(a, sm, tmem, lane_base, aux, pmax_buf, abort_flag, gt_, vk, jrow, t,
                           hf, copy, rho, rpc, active);
        // V rows the P.V MMA reads past the valid keys may hold anything: zero them so that
        // P = 0 times V stays 0 (the MMA reads whole 16-key steps of valid pages)
        const int vrows = cache_tile ? min(kTK, (vk + kPage - 1) / kPage * kPage) : kNewRows;
        if (vk < vrows) {
          const uint32_t pair = gt_ % kPairsV;
          ptx::mbar_wait(bar(kBarVFull, 2 * pair + vk / kPage), (gt_ / kPairsV) & 1, abort_flag);
          for (int idx = tid; idx < (vrows - vk) * 16; idx += kSoftmaxThreads) {
            const uint32_t row = vk + idx / 16, half = (idx % 16) / 8, c = idx % 8;
            st_shared_v4(ring(2 + half, 2 * pair) + row * 128 + c * 16, 0u, 0u, 0u, 0u);
          }
          ptx::fence_proxy_async_smem();
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kBarPFull, 0));
      }

      // the next piece's queries into tensor memory, so its S MMAs overlap this epilogue
      if (have2 && m2.ntiles > 0) q_commit(m2);

      // ---------------------------------------------------------------- epilogue
      // Each copy holds a partial O over its own keys.  Four rounds of 32 columns: the lane's two
      // threads put its columns into the staging area (16 each), then thread (copy, half, rho)
      // sums the copies of row rho for its 32 / (2 C) columns of the round and writes them
      // (bf16 output, or the fp32 partial of a split segment).
      lsum_buf[tid] = sm.l_part;
      if (m.ntiles > 0) {
        ptx::mbar_wait(bar(kBarODone, 0), (gt + m.ntiles - 1) & 1, abort_flag);
        ptx::tc_fence_after();
      }
      if (tid == 0 && split) {  // 2: merge at once (read after the next barrier)
        const int pieces = s_split[1] - s_split[0] + 1;
        *s_last = (pre_count == pieces - 1) ? 2 : 0;
      }
      ptx::named_bar_sync(2, kSoftmaxThreads);
      const bool whole = (ta == 0 && tb == tiles);
      const int c_first = s_split[0], c_last = s_split[1], slot_first = s_split[2];
      const int my_slot = ((int)blockIdx.x == c_first) ? slot_first : 2 * (int)blockIdx.x;
      float *part = a.ws.partials + (size_t)my_slot * a.rows_max * kPS;
      if (m.ntiles > 0) {
        float l = 0.f;
        for (int cc = 0; cc < m.C; ++cc) l += lsum_buf[rho + cc * rpc] + lsum_buf[128 + rho + cc * rpc];
        const float inv = 1.f / l;
        const int j = rho / G, i = rho % G;
        const size_t orow = ((size_t)(m.t0 + j) * a.Hq + g * G + i) * kD;
        const uint32_t o_taddr = tmem + lane_base + kColO + hf * 16;
        const int nc = 16 / m.C;  // columns of a round this thread finishes (4 or 8)
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
          float o[16];
          ptx::tmem_ld16(o_taddr + c32 * 32, o);
          ptx::tmem_wait_ld();
          if (c32 == 3) {  // O fully read: the next piece's P.V may overwrite it
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar(kBarOFree, 0));
          }
#pragma unroll
          for (int k = 0; k < 4; ++k)
            st_shared_v4(stage + t * 128 + (((hf * 4 + k) ^ (t & 7)) << 4), __float_as_uint(o[4 * k]),
                         __float_as_uint(o[4 * k + 1]), __float_as_uint(o[4 * k + 2]),
                         __float_as_uint(o[4 * k + 3]));
          ptx::named_bar_sync(2, kSoftmaxThreads);
          if (active) {
            float acc[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] = 0.f;
            const int k0 = (copy * 2 + hf) * (nc / 4);  // first float4 chunk of these columns
            for (int cc = 0; cc < m.C; ++cc) {
              const int row = rho + cc * rpc;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                if (k < nc / 4) {
                  const uint4 v = ptx::ld_shared_v4(stage + row * 128 + (((k0 + k) ^ (row & 7)) << 4));
                  acc[4 * k] += __uint_as_float(v.x);
                  acc[4 * k + 1] += __uint_as_float(v.y);
                  acc[4 * k + 2] += __uint_as_float(v.z);
                  acc[4 * k + 3] += __uint_as_float(v.w);
                }
              }
            }
            const int col0 = c32 * 32 + (copy * 2 + hf) * nc;
            if (whole) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                if (k < nc / 4) {
                  uint2 w2;
                  w2.x = ptx::pack_bf16x2(acc[4 * k] * inv, acc[4 * k + 1] * inv);
                  w2.y = ptx::pack_bf16x2(acc[4 * k + 2] * inv, acc[4 * k + 3] * inv);
                  *reinterpret_cast<uint2 *>(og + orow + col0 + 4 * k) = w2;
                }
              }
            } else {
              float4 *dst = reinterpret_cast<float4 *>(part + (size_t)rho * kPS + col0);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                if (k < nc / 4)
                  dst[k] = make_float4(acc[4 * k], acc[4 * k + 1], acc[4 * k + 2], acc[4 * k + 3]);
            }
          }
          ptx::named_bar_sync(2, kSoftmaxThreads);  // before the next round reuses the staging
        }
        if (active && copy == 0 && hf == 0 && !whole) {
          part[(size_t)rho * kPS + kD] = sm.m_run;
          part[(size_t)rho * kPS + kD + 1] = l;
        }
        gt += m.ntiles;
      } else if (!whole) {
        // a piece holding only tail units of its segment: a partial without keys
        for (int idx = tid; idx < m.rows * kPS; idx += kSoftmaxThreads)
          part[idx] = (idx % kPS == kD) ? -INFINITY : 0.f;
      }

      if (!whole) {  // split segment: publish the partial, the last piece merges
        if (*s_last != 2) {
          __threadfence();
          ptx::named_bar_sync(2, kSoftmaxThreads);
          if (tid == 0) {
            const int pieces = c_last - c_first + 1;
            const int prev = atomicAdd(a.ws.counters + r * a.Hkv + g, 1);
            *s_last = (prev == pieces - 1);
          }
        } else {
          // every other piece published before this one started (tid 0's acquire read of the
          // counter, ordered for the CTA by the barriers): no publish, no count; the merge below
          // reads this CTA's own partial after the barrier and resets the counter
        }
        ptx::named_bar_sync(2, kSoftmaxThreads);
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
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc
}  // namespace dspark
