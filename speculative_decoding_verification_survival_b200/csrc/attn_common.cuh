// Work partition and split-KV merge shared by the verify-attention kernels.
//
// The flattened verify batch ("刚融完500亿…专治AI“嘴慢”", engineering table row "内核利用率暴跌":
// every verify token is an independent element, no per-request padding) is turned into a
// sequence of work units: for each request r (in order) and each KV head g, the request's cache
// is cut into tiles of kTileKeys positions, followed by kSegTail units standing for the request's
// own verify tokens (so a request with an empty cache still has work units).  A segment = all units of one
// (r, g); all G*Q_r query rows of the segment are processed together, so every KV byte is read
// once.
//
// The unit sequence is split into equal contiguous ranges, one per persistent CTA (W units
// each).  A segment cut by a range boundary is computed in pieces; each piece writes an
// un-normalised (m, l, acc) partial and the last piece to arrive (atomic counter, no waiting)
// merges them.  CTA c writes at most two partials: slot 2c for its first segment, 2c+1 for its
// last one.
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kTileKeys = 64;
constexpr int kMaxCtasPerSm = 4;

struct AttnPlanHeader {
  int R, Hkv, rows_max, D;
  int tile_keys, total;  // total = units of the whole batch
  int tc_ctas, tc_W;     // the tensor-core kernel's grid and units per CTA
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Floats per row of a split-KV partial: acc[D], then m and l, padded so rows stay 16-byte aligned.
__host__ __device__ constexpr int part_stride(int D) { return D + 4; }

struct AttnWs {
  AttnPlanHeader *hdr;
  int *tile_prefix;  // [R + 1]: first unit of request r (units of all its Hkv segments)
  int *counters;     // [R * Hkv] arrival counters of split segments (kept at zero between calls)
  int4 *req;         // [R]: per request {t0, Q, kv_len, schedule valid} written by the plan
  int4 *cta_start;   // [max_ctas]: first segment of tensor-core CTA c {r, g, s0, units}, r < 0: none
  float *partials;   // [2 * max_ctas][rows_max][part_stride(D)]: acc[D], m, l per row
};

__host__ __device__ inline size_t attn_ws_layout(int R, int Hkv, int rows_max, int D,
                                                 int max_ctas, AttnWs *ws, void *base) {
  size_t off = 0;
  const size_t o_hdr = off;                off += align256(sizeof(AttnPlanHeader));
  const size_t o_pre = off;                off += align256((size_t)(R + 1) * sizeof(int));
  const size_t o_cnt = off;                off += align256((size_t)R * Hkv * sizeof(int));
  const size_t o_req = off;                off += align256((size_t)R * sizeof(int4));
  const size_t o_cst = off;                off += align256((size_t)max_ctas * sizeof(int4));
  const size_t o_par = off;
  off += align256((size_t)2 * max_ctas * rows_max * part_stride(D) * sizeof(float));
  if (ws) {
    char *b = static_cast<char *>(base);
    ws->hdr = reinterpret_cast<AttnPlanHeader *>(b + o_hdr);
    ws->tile_prefix = reinterpret_cast<int *>(b + o_pre);
    ws->counters = reinterpret_cast<int *>(b + o_cnt);
    ws->req = reinterpret_cast<int4 *>(b + o_req);
    ws->cta_start = reinterpret_cast<int4 *>(b + o_cst);
    ws->partials = reinterpret_cast<float *>(b + o_par);
  }
  return off;
}

// Units of one (request, KV head) segment: one per 64-key cache tile, then kSegTail units for
// the verify tokens.  The verify tokens are one tile of work plus the segment's epilogue and the
// pipeline refill of the next segment, which together cost about as much time as eight cache
// tiles (measured: a weight of 1, 3, 5, 8 gave 183, 167, 150, 140 us on 64 requests of 512..4096
// cached keys), so the tail is weighted that way for the equal split across CTAs.  A CTA range that covers only tail units of a segment (not its last
// unit) is an empty piece: it contributes a partial with no keys.
constexpr int kSegTail = 8;
__host__ __device__ inline int segment_units(int n) {
  return (n + kTileKeys - 1) / kTileKeys + kSegTail;
}
// Cache tiles of a segment with `units` units.
__host__ __device__ inline int segment_cache_tiles(int units) { return units - kSegTail; }

// Plan: tile_prefix (exclusive scan of Hkv * segment_units(kv_len)), counters = 0, and one
// record per request: its flattened offset t0, token count Q, cache length, and whether the
// flattening is well formed (1 <= Q <= K + 1 inside [0, T_cap), and token j of the request
// carries the marker (r, kv_len + j) — the layout the scheduler's flattening step produces).
// A malformed request raises its error bit here, once per step, and is skipped by the
// attention calls that use this plan.
__device__ __forceinline__ void find_segment(const int *__restrict__ tile_prefix, int R, int Hkv,
                                             int u, int &r, int &g, int &tiles, int &seg_start);

// It also records where each of the tensor-core kernel's `tc_ctas` CTAs starts (its first
// segment), so that kernel walks segments in order without searching.
__global__ void __launch_bounds__(1024)
attn_plan_kernel(const int32_t *__restrict__ kv_len, const int32_t *__restrict__ q_offsets,
                 const int32_t *__restrict__ markers, int R, int T_cap, int K, int Hkv,
                 int rows_max, int D, int tc_ctas, AttnWs ws) {
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (R + blockDim.x - 1) / blockDim.x;
  int local = 0;
  for (int i = 0; i < per; ++i) {
    const int r = tid * per + i;
    if (r < R) {
      int n = kv_len[r];
      if (n < 0) { raise_error(DSPARK_DERR_KV_LEN); n = 0; }
      local += Hkv * segment_units(n);
    }
  }
  int incl = local;
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = (lane < (int)(blockDim.x >> 5)) ? warp_tot[lane] : 0;
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    warp_tot[lane] = v;
  }
  __syncthreads();
  int off = (warp ? warp_tot[warp - 1] : 0) + incl - local;
  for (int i = 0; i < per; ++i) {
    const int r = tid * per + i;
    if (r < R) {
      ws.tile_prefix[r] = off;
      int n = max(kv_len[r], 0);
      off += Hkv * segment_units(n);
      if (r == R - 1) ws.tile_prefix[R] = off;
    }
  }
  for (int i = tid; i < R * Hkv; i += blockDim.x) ws.counters[i] = 0;
  for (int r = tid; r < R; r += blockDim.x) {
    const int t0 = q_offsets[r], Q = q_offsets[r + 1] - t0, n = kv_len[r];
    bool ok = Q >= 1 && Q <= K + 1 && t0 >= 0 && t0 <= T_cap - Q;
    if (!ok) raise_error(DSPARK_DERR_OFFSETS);
    ok = ok && n >= 0;
    if (ok) {
      bool good = true;
      for (int j = 0; j < Q; ++j)
        good &= (markers[2 * (t0 + j)] == r) & (markers[2 * (t0 + j) + 1] == n + j);
      if (!good) raise_error(DSPARK_DERR_MARKER);
      ok = good;
    }
    ws.req[r] = make_int4(t0, Q, n, ok ? 1 : 0);
  }
  __syncthreads();  // tile_prefix complete (global writes of this block)
  const int total = ws.tile_prefix[R];
  const int W = (total + tc_ctas - 1) / tc_ctas;
  for (int c = tid; c < tc_ctas; c += blockDim.x) {
    int4 st = make_int4(-1, 0, 0, 0);
    if (c * W < total) {
      int r, g, tiles, s0;
      find_segment(ws.tile_prefix, R, Hkv, c * W, r, g, tiles, s0);
      st = make_int4(r, g, s0, tiles);
    }
    ws.cta_start[c] = st;
  }
  if (tid == 0) {
    ws.hdr->R = R;
    ws.hdr->Hkv = Hkv;
    ws.hdr->rows_max = rows_max;
    ws.hdr->D = D;
    ws.hdr->tile_keys = kTileKeys;
    ws.hdr->total = total;
    ws.hdr->tc_ctas = tc_ctas;
    ws.hdr->tc_W = W;
  }
}

// A contiguous piece of one segment handled by one CTA.
struct SegPiece {
  int r, g;         // request, KV head
  int ta, tb;       // tile range [ta, tb) within the segment
  int tiles;        // tiles in the whole segment
  int seg_start;    // global index of the segment's first unit
  bool first_of_cta;
};

// Locate the segment containing global unit u (binary search over requests).  Plain loads: the
// plan kernel calls it on a prefix it has just written.
__device__ __forceinline__ void find_segment(const int *__restrict__ tile_prefix, int R, int Hkv,
                                             int u, int &r, int &g, int &tiles, int &seg_start) {
  int lo = 0, hi = R - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_prefix[mid] <= u) lo = mid; else hi = mid - 1;
  }
  r = lo;
  const int base = tile_prefix[r];
  tiles = (tile_prefix[r + 1] - base) / Hkv;
  g = (u - base) / tiles;
  seg_start = base + g * tiles;
}

// Slot of the partial written for segment (start s0, tiles nt) by CTA c, given W units per CTA.
__device__ __forceinline__ int partial_slot(int c, int s0, int W) {
  const int first_cta = s0 / W;
  return 2 * c + ((c == first_cta && s0 != c * W) ? 1 : 0);
}

}  // namespace dspark
