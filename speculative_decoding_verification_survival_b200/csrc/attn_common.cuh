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
// The unit sequence is split into contiguous ranges, one per persistent CTA.  A segment cut by a
// range boundary is computed in pieces; each piece writes an un-normalised (m, l, acc) partial
// and the last piece to arrive (atomic counter, no waiting) merges them.  CTA c writes at most
// two partials: slot 2c for its first segment, 2c+1 for its last one.  The tensor-core kernel's
// ranges come from the plan, which chooses them to minimise the largest modelled cost of a CTA
// (cache pages, the verify-token tile, a fixed cost per piece and per merge); the CUDA-core
// kernel splits the units into equal ranges.
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kTileKeys = 64;
constexpr int kMaxCtasPerSm = 4;

struct AttnPlanHeader {
  int R, Hkv, rows_max, D;
  int tile_keys, total;  // total = units of the whole batch
  int tc_ctas;           // the tensor-core kernel's grid (ranges in AttnWs::cta_begin)
  float tc_bound;        // the largest modelled CTA cost of those ranges
};

// Cost model of the tensor-core kernel's work, in units of one 64-key cache page (about 0.75 us
// of a CTA's time at full clock).  A segment's verify tokens and its query rows cost 4, a piece
// (its epilogue and the refill of the pipeline for the next piece) 7, merging the partials of a
// split segment 6: the best of a sweep of the three constants, timed on workloads of 64 to 1024
// requests; the plateau is flat to about 1%.  The head piece of a split segment usually merges,
// as the next CTA finishes the segment's rest first.
constexpr float kCostNewTile = 4.0f;
constexpr float kCostPiece = 7.0f;
constexpr float kCostMerge = 6.0f;
// Candidate cost bounds the plan tests at once (one per thread of its single CTA).
constexpr int kPlanCandidates = 1024;
// Requests whose unit prefix the plan keeps in shared memory for the candidate fills (more are
// read from the workspace).
constexpr int kPlanSmemRequests = 4096;

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Floats per row of a split-KV partial: acc[D], then m and l, padded so rows stay 16-byte aligned.
__host__ __device__ constexpr int part_stride(int D) { return D + 4; }

struct AttnWs {
  AttnPlanHeader *hdr;
  int *tile_prefix;  // [R + 1]: first unit of request r (units of all its Hkv segments)
  int *counters;     // [R * Hkv] arrival counters of split segments (kept at zero between calls)
  int4 *req;         // [R]: per request {t0, Q, kv_len, schedule valid} written by the plan
  int4 *cta_start;   // [max_ctas]: first segment of tensor-core CTA c {r, g, s0, units}, r < 0: none
  int *cta_begin;    // [max_ctas + 1]: first unit of tensor-core CTA c; [tc_ctas] = total
  float *partials;   // [2 * max_ctas][rows_max][part_stride(D)]: acc[D], m, l per row
  float *seg_cost;   // [R]: modelled cost of a whole segment of request r (plan scratch)
  int *seg_c;        // [R]: the same as an integer (plan scratch past kPlanSmemRequests)
  int4 *cta_req;     // [max_ctas]: the request record of tensor-core CTA c's first segment
  int *cand_begin;   // [kPlanCandidates][max_ctas + 1]: each candidate fill's range starts
};

__host__ __device__ inline size_t attn_ws_layout(int R, int Hkv, int rows_max, int D,
                                                 int max_ctas, AttnWs *ws, void *base) {
  size_t off = 0;
  const size_t o_hdr = off;                off += align256(sizeof(AttnPlanHeader));
  const size_t o_pre = off;                off += align256((size_t)(R + 1) * sizeof(int));
  const size_t o_cnt = off;                off += align256((size_t)R * Hkv * sizeof(int));
  const size_t o_req = off;                off += align256((size_t)R * sizeof(int4));
  const size_t o_cst = off;                off += align256((size_t)max_ctas * sizeof(int4));
  const size_t o_beg = off;                off += align256((size_t)(max_ctas + 1) * sizeof(int));
  const size_t o_par = off;
  off += align256((size_t)2 * max_ctas * rows_max * part_stride(D) * sizeof(float));
  const size_t o_sc = off;                 off += align256((size_t)R * sizeof(float));
  const size_t o_crq = off;                off += align256((size_t)max_ctas * sizeof(int4));
  const size_t o_sgc = off;                off += align256((size_t)R * sizeof(int));
  const size_t o_cbg = off;
  off += align256((size_t)kPlanCandidates * (max_ctas + 1) * sizeof(int));
  if (ws) {
    char *b = static_cast<char *>(base);
    ws->hdr = reinterpret_cast<AttnPlanHeader *>(b + o_hdr);
    ws->tile_prefix = reinterpret_cast<int *>(b + o_pre);
    ws->counters = reinterpret_cast<int *>(b + o_cnt);
    ws->req = reinterpret_cast<int4 *>(b + o_req);
    ws->cta_start = reinterpret_cast<int4 *>(b + o_cst);
    ws->cta_begin = reinterpret_cast<int *>(b + o_beg);
    ws->partials = reinterpret_cast<float *>(b + o_par);
    ws->seg_cost = reinterpret_cast<float *>(b + o_sc);
    ws->cta_req = reinterpret_cast<int4 *>(b + o_crq);
    ws->cand_begin = reinterpret_cast<int *>(b + o_cbg);
    ws->seg_c = reinterpret_cast<int *>(b + o_sgc);
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

// Greedy fill of CTAs in unit order under a cost bound: a segment goes whole into the current
// CTA if it fits; otherwise the CTA takes a head piece of an even number of cache pages (at
// least 2, with the piece and merge costs) and the rest continues in the next CTAs (which may
// cut it again); a bound under which not even a two-page piece fits counts as infeasible.  A
// range boundary never falls inside a segment's verify-token units.  Returns the number of CTAs
// used (stops counting past `cap`); when `begin` is given, records the first unit of every CTA
// used (begin[0] = 0).
__device__ int plan_fill(const int *__restrict__ tile_prefix, const float *seg_cost, int R, int Hkv,
                         float bound, int cap, int *begin) {
  int used = 1;
  float cur = 0.f;
  if (begin) begin[0] = 0;
  for (int r = 0; r < R && used <= cap; ++r) {
    // a segment's cost when whole: its cache pages, its verify tokens and one piece
    const float full = seg_cost[r];
    const float all = (float)Hkv * full;
    if (cur + all <= bound) {  // the request's Hkv segments all fit: the usual case
      cur += all;
      continue;
    }
    const int u = (int)(full - kCostNewTile - kCostPiece);  // cache pages of a segment
    const int seg_units = u + kSegTail;
    for (int g = 0; g < Hkv && used <= cap; ++g) {
      if (cur + full <= bound) { cur += full; continue; }
      const int s0 = tile_prefix[r] + g * seg_units;
      int done = 0;  // cache pages of this segment placed in earlier CTAs
      int head = (int)floorf(bound - cur - kCostPiece - kCostMerge);
      head &= ~1;
      if (head >= 2 && head < u) done = head;  // head piece in the current CTA
      // the rest starts a new CTA; middle pieces fill whole CTAs while it does not fit
      while (true) {
        ++used;
        if (begin && used <= cap) begin[used - 1] = s0 + done;
        const float rest = (float)(u - done) + kCostNewTile + kCostPiece;
        if (rest <= bound || used > cap) { cur = rest; break; }
        // a segment cut from its start here (no head piece placed above) has its head now
        const int mid = (int)floorf(bound - kCostPiece - (done == 0 ? kCostMerge : 0.f)) & ~1;
        if (mid < 2) return cap + 1;  // not even a two-page piece fits: the bound is infeasible
        done = min(u, done + mid);
      }
    }
  }
  return used;
}

// The same greedy fill, jumping over the whole segments that fit.  The costs are integers and a
// whole segment of request r costs its units plus kNew + kPiece - kSegTail, so the cost of all
// segments of the requests before r is pq(r) = tile_prefix[r] + r * Hkv * (kNew + kPiece -
// kSegTail): the run of whole segments that fits in a CTA's remaining capacity is found by a
// binary search on it, and only the segments that are cut take the steps above.  A fill costs
// O(CTAs * log R) instead of O(R * Hkv), with the same ranges as plan_fill for the same bound.
// The caller checks that pq(R) fits an int.
__device__ int plan_fill_jump(const int *tile_prefix, const int *segc, int R, int Hkv,
                              float bound, int cap, int *begin) {
  const int B = (int)floorf(bound);  // every cost is an integer: cost <= bound <=> cost <= B
  constexpr int kNew = (int)kCostNewTile, kPiece = (int)kCostPiece, kMerge = (int)kCostMerge;
  const int step = Hkv * (kNew + kPiece - kSegTail);
  auto pq = [&](int r) { return tile_prefix[r] + r * step; };
  int used = 1, cur = 0;
  if (begin) begin[0] = 0;
  int r = 0, g = 0;  // the next segment
  while (r < R && used <= cap) {
    const int start = pq(r) + g * segc[r];
    const int limit = start + (B - cur);  // the cost prefix this CTA can reach
    // the last request whose start the CTA reaches: largest r2 in [r, R] with pq(r2) <= limit,
    // by a galloping search from r (a CTA spans few requests), then bisection
    int lo = r, stp = 1;
    while (lo + stp <= R && pq(lo + stp) <= limit) {
      lo += stp;
      stp <<= 1;
    }
    int hi = min(R, lo + stp - 1);
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pq(mid) <= limit) lo = mid; else hi = mid - 1;
    }
    const int r2 = lo;
    if (r2 == R) break;  // everything left fits
    const int p2 = pq(r2), c2 = segc[r2];
    // segments of r2 that fit whole: floor((limit - p2) / c2) by a float quotient and a fix-up
    // (small integers, exact in float)
    int g2 = (int)__fdividef((float)(limit - p2), (float)c2);
    if ((g2 + 1) * c2 <= limit - p2) ++g2;
    if (g2 * c2 > limit - p2) --g2;
    g2 = min(Hkv - 1, g2);
    cur += p2 + g2 * c2 - start;
    r = r2;
    g = g2;
    // segment (r, g) does not fit whole: cut it
    const int u = c2 - kNew - kPiece;  // cache pages of a segment
    const int s0 = tile_prefix[r] + g * (u + kSegTail);
    int done = 0;
    const int head = (B - cur - kPiece - kMerge) & ~1;
    if (head >= 2 && head < u) done = head;  // head piece in the current CTA
    while (true) {
      ++used;
      if (begin && used <= cap) begin[used - 1] = s0 + done;
      const int rest = (u - done) + kNew + kPiece;
      if (rest <= B || used > cap) { cur = rest; break; }
      const int midp = (B - kPiece - (done == 0 ? kMerge : 0)) & ~1;
      if (midp < 2) return cap + 1;  // not even a two-page piece fits: the bound is infeasible
      done = min(u, done + midp);
    }
    if (++g == Hkv) {
      g = 0;
      ++r;
    }
  }
  return used;
}

// It also records where each of the tensor-core kernel's `tc_ctas` CTAs starts (its first
// unit and first segment), so that kernel walks segments in order without searching.
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

  // Cost-balanced ranges: every thread runs the greedy fill below for one candidate bound on a
  // CTA's modelled cost; the smallest bound that needs at most tc_ctas CTAs wins and its fill
  // is run once more to record where each CTA starts.
  __shared__ float s_tot;
  __shared__ int s_best;
  float seg_max = 0.f, mine = 0.f;
  for (int r = tid; r < R; r += blockDim.x) {
    const float u = (float)((ws.tile_prefix[r + 1] - ws.tile_prefix[r]) / Hkv - kSegTail);
    const float full = u + kCostNewTile + kCostPiece;
    mine += Hkv * full;
    seg_max = fmaxf(seg_max, full);
  }
  mine = warp_sum(mine);
  seg_max = warp_max(seg_max);
  __shared__ float s_part[32], s_pmax[32];
  if (lane == 0) { s_part[warp] = mine; s_pmax[warp] = seg_max; }
  if (tid == 0) s_best = kPlanCandidates;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f, mx = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) { t += s_part[w]; mx = fmaxf(mx, s_pmax[w]); }
    s_tot = t;
    s_pmax[0] = mx;
  }
  __syncthreads();
  // Each of the first kPlanCandidates threads runs the greedy fill for one candidate bound in
  // (lo, hi] (hi always fits), reading the segment costs from shared memory; the smallest that
  // needs at most tc_ctas CTAs wins and its fill is run once more to record where each CTA
  // starts.
  const float lo = s_tot / (float)tc_ctas;
  const float hi = lo + s_pmax[0] + kCostMerge + kCostPiece;
  // The fills read the unit prefix from shared memory when it fits; a cost total that does not
  // fit an int (far beyond any real batch) falls back to the segment-by-segment float fill.
  __shared__ int s_tp[kPlanSmemRequests + 1], s_c[kPlanSmemRequests];
  const bool staged = R <= kPlanSmemRequests;
  int *segc = staged ? s_c : ws.seg_c;
  if (staged)
    for (int r = tid; r <= R; r += blockDim.x) s_tp[r] = ws.tile_prefix[r];
  for (int r = tid; r < R; r += blockDim.x)  // a whole segment's cost, per request
    segc[r] = (ws.tile_prefix[r + 1] - ws.tile_prefix[r]) / Hkv - kSegTail + (int)kCostNewTile +
              (int)kCostPiece;
  const long long cost_total =
      (long long)total + (long long)R * Hkv * (long long)(kCostNewTile + kCostPiece - kSegTail);
  const bool jump = cost_total < (long long)INT_MAX / 2;
  if (!jump)
    for (int r = tid; r < R; r += blockDim.x)
      ws.seg_cost[r] = (float)((ws.tile_prefix[r + 1] - ws.tile_prefix[r]) / Hkv - kSegTail) +
                       kCostNewTile + kCostPiece;
  __syncthreads();
  const int *tp = staged ? s_tp : ws.tile_prefix;
  // Every cost is an integer, so bounds with the same integer part give the same fill: the
  // candidates are integers from floor(lo) + 1 up, at a spacing that covers (lo, hi] with at
  // most kPlanCandidates of them (the last one is hi or more: always feasible).  Small batches
  // then test a few dozen bounds, not a thousand copies of them.
  const int ilo = (int)floorf(lo);
  const int span = max(1, (int)ceilf(hi) - ilo);
  const int spacing = (span + kPlanCandidates - 1) / kPlanCandidates;
  const int ncand = (span + spacing - 1) / spacing;
  // Each fill records its range starts in a scratch row of its own; the winner's row is then
  // copied, so no fill runs twice.
  __shared__ int s_used[kPlanCandidates];
  if (tid < ncand) {
    const float cand = (float)(ilo + (tid + 1) * spacing);
    int *mine = ws.cand_begin + (size_t)tid * (tc_ctas + 1);
    const int need = jump ? plan_fill_jump(tp, segc, R, Hkv, cand, tc_ctas, mine)
                          : plan_fill(ws.tile_prefix, ws.seg_cost, R, Hkv, cand, tc_ctas, mine);
    s_used[tid] = need;
    if (need <= tc_ctas) atomicMin(&s_best, tid);
  }
  __syncthreads();
  const int best = min(s_best, ncand - 1);
  const float bound = (float)(ilo + (best + 1) * spacing);
  const int used = min(s_used[best], tc_ctas);
  const int *win = ws.cand_begin + (size_t)best * (tc_ctas + 1);
  // the winner's starts; trailing CTAs get empty ranges (had no bound fitted, the last CTA would
  // take the rest)
  for (int c = tid; c <= tc_ctas; c += blockDim.x) ws.cta_begin[c] = c < used ? win[c] : total;
  if (tid == 0) ws.hdr->tc_bound = bound;
  __syncthreads();
  // (the request records written above are visible to the whole block since its barriers)
  for (int c = tid; c < tc_ctas; c += blockDim.x) {
    int4 st = make_int4(-1, 0, 0, 0), rq = make_int4(0, 0, 0, 0);
    const int u0 = ws.cta_begin[c];
    if (u0 < ws.cta_begin[c + 1]) {
      int r, g, tiles, s0;
      find_segment(ws.tile_prefix, R, Hkv, u0, r, g, tiles, s0);
      st = make_int4(r, g, s0, tiles);
      rq = ws.req[r];
    }
    ws.cta_start[c] = st;
    ws.cta_req[c] = rq;  // with the start record, so a CTA's first piece needs no dependent load
  }
  if (tid == 0) {
    ws.hdr->R = R;
    ws.hdr->Hkv = Hkv;
    ws.hdr->rows_max = rows_max;
    ws.hdr->D = D;
    ws.hdr->tile_keys = kTileKeys;
    ws.hdr->total = total;
    ws.hdr->tc_ctas = tc_ctas;
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

// The tensor-core kernel's CTA ranges: the plan's (begin[c] .. begin[c + 1]) when the grid is
// the one the plan prepared, else equal ranges of W units.
struct Ranges {
  const int *begin;  // nullptr: equal ranges
  int W, ctas, total;
  __device__ __forceinline__ int start(int c) const {
    return begin ? __ldcg(begin + c) : min(c * W, total);
  }
  // The CTA whose range holds unit u: the last c with start(c) <= u (empty ranges end the list).
  __device__ __forceinline__ int cta_of(int u) const {
    if (!begin) return u / W;
    int lo = 0, hi = ctas - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldcg(begin + mid) <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
  // Slot of the partial CTA c writes for the segment starting at unit s0: 2c for the CTA's
  // first segment, 2c + 1 for a segment that starts inside its range and continues past it.
  __device__ __forceinline__ int slot(int c, int s0) const {
    return 2 * c + ((c == cta_of(s0) && s0 != start(c)) ? 1 : 0);
  }
};

}  // namespace dspark
