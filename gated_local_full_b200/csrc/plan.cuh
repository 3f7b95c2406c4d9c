// Work partition of one decode-attention launch.
//
// The rows of a launch (every batch row for Local, the gate's compacted rows
// for Full) and their KV heads form segments; a segment is a run of 16-token
// tiles. The partition decides which tiles each CTA of the persistent grid
// reads:
//   * aligned, when the segments fit the grid: each segment gets its own CTAs
//     in proportion to its length (at least one, at most one per min_tiles
//     tiles) and every CTA works inside one segment;
//   * even otherwise: the tile space is split evenly and a CTA may span
//     several segments.
// Aligned is used only if no CTA would get more than 1.2x the even share.
//
// plan_rows runs on warp 0 of a block and leaves the per-row arrays in shared
// memory; plan_cta turns them into one CTA's share. Its global loads bypass
// L1 (ld.global.cg), so a guess made before a dependency wait leaves no stale
// line behind for the loads after it. The attention kernel can
// run both itself, or read a plan that another kernel wrote once for all the
// launches that share it (the Local launches of a decode step).
#pragma once

#include "oda_internal.cuh"

namespace oda {

struct PlanIn {
  int B;                       // rows of the call
  const int32_t* count;        // Full: device count of compacted rows; Local: null
  const int32_t* idx;          // Full: compacted row ids; Local: null
  const int32_t* seq_lens;     // [B] t
  int hkv, sink, window, max_blocks;
  int min_tiles;               // smallest share of tiles per CTA
  int grid;                    // CTAs of the attention launch
  int* err;
  bool report;                 // record errors (one block per launch does)
  const int32_t* range_lo;     // paged source only: per row, first position of the region
  const int32_t* range_hi;     // ... and one past its last (null: the whole history 1..t)
};

struct PlanHead {
  int nr, tot, P, al;
};

// Warp 0 only. Writes rowb/rowt [nr], rowstart/rowcs [nr+1], and for the
// paged source rowlo [nr] (the region's first position; rowt is its last).
__device__ __forceinline__ PlanHead plan_rows(const PlanIn& p, int* rowb, int* rowt,
                                              int* rowstart, int* rowcs, int* rowlo = nullptr) {
  const int lane = threadIdx.x & 31;
  const bool ring = p.count == nullptr;
  // with B <= 32 every lane loads one row's length and one compacted id
  // before the count, so the three loads travel together instead of chaining
  const bool small = p.B <= 32;
  const int tl = (small && lane < p.B) ? __ldcg(p.seq_lens + lane) : 0;
  const int il = (small && !ring && lane < p.B) ? __ldcg(p.idx + lane) : 0;
  int nr;
  if (ring) {
    nr = p.B;
  } else {
    nr = *reinterpret_cast<const volatile int32_t*>(p.count);
    if (nr < 0 || nr > p.B) {
      if (lane == 0 && p.report) record_error(p.err, ODA_ERR_BOUNDS);
      nr = nr < 0 ? 0 : p.B;
    }
  }
  int carry = 0;
  for (int base = 0; base < nr; base += 32) {
    const int i = base + lane;
    int nt = 0;
    const int bl = i < nr ? (ring ? i : (small ? il : __ldcg(p.idx + i))) : 0;
    const bool okl = bl >= 0 && bl < p.B;
    const int ts = __shfl_sync(0xffffffffu, tl, okl ? (bl & 31) : 0);   // all lanes shuffle
    if (i < nr) {
      const int t = !okl ? 0 : (small ? ts : __ldcg(p.seq_lens + bl));
      int first = 1, last = t;                   // positions first..last are read
      if (!okl || t < 1) {
        if (p.report) record_error(p.err, ODA_ERR_BOUNDS);
      } else if (ring) {
        nt = (p.sink + min(t, p.window) + ODA_TILE - 1) / ODA_TILE;
      } else {
        bool ok = true;
        if (p.range_lo) {                        // the region [lo, hi), within 1..t
          const int rl = __ldcg(p.range_lo + bl), rh = __ldcg(p.range_hi + bl);
          ok = rl >= 1 && rh > rl && rh - 1 <= t;
          first = rl;
          last = rh - 1;
        }
        const int tend = (last + ODA_TILE - 1) / ODA_TILE;   // tiles up to the last position
        if (!ok || tend > p.max_blocks) {
          if (p.report) record_error(p.err, ODA_ERR_BOUNDS);
        } else {
          nt = tend - (first - 1) / ODA_TILE;
        }
      }
      rowb[i] = okl ? bl : 0;
      rowt[i] = ring ? t : last;
      if (rowlo) rowlo[i] = first;
    }
    int v = nt * p.hkv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (i < nr) rowstart[i + 1] = carry + v;
    carry += __shfl_sync(0xffffffffu, v, 31);
  }
  __syncwarp();                                  // rowstart[] visible to every lane
  const int tot = carry;
  int P = p.grid;
  if (tot > 0) P = min(P, max(1, (tot + p.min_tiles - 1) / p.min_tiles));
  // per-row CTA counts of the aligned partition, their prefix, the worst load
  int carry2 = 0, worst = 0;
  for (int base = 0; base < nr; base += 32) {
    const int i = base + lane;
    int n = 0;
    if (i < nr) {
      const int nt = (rowstart[i + 1] - (i == 0 ? 0 : rowstart[i])) / p.hkv;
      if (nt > 0) {
        n = ((unsigned)nt < (1u << 31) / (unsigned)P)
                ? (int)(((unsigned)nt * (unsigned)P) / (unsigned)tot)
                : (int)(((long long)nt * P) / tot);
        n = max(min(n, nt / p.min_tiles), 1);
        worst = max(worst, (nt + n - 1) / n);
      }
    }
    int v = n * p.hkv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (i < nr) rowcs[i + 1] = carry2 + v;
    carry2 += __shfl_sync(0xffffffffu, v, 31);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) worst = max(worst, __shfl_xor_sync(0xffffffffu, worst, o));
  if (lane == 0) {
    rowstart[0] = 0;
    rowcs[0] = 0;
  }
  __syncwarp();
  const int even = tot > 0 ? (tot + P - 1) / P : 0;
  PlanHead h;
  h.nr = nr;
  h.tot = tot;
  h.P = P;
  h.al = (tot > 0 && carry2 <= p.grid && 5 * worst <= 6 * even) ? 1 : 0;
  return h;
}

// One CTA's share: out = {lo, hi, pbase, nparts, part}; lo == hi: no work.
__device__ __forceinline__ void plan_cta(int cta, const PlanHead& h, const int* rowstart,
                                         const int* rowcs, int hkv, int out[5]) {
  out[0] = out[1] = out[2] = out[3] = out[4] = 0;
  if (h.tot <= 0) return;
  if (h.al) {
    if (cta >= rowcs[h.nr]) return;
    int r0 = 0, r1 = h.nr - 1;                   // row with rowcs[r0] <= cta < rowcs[r0+1]
    while (r0 < r1) {
      const int mid = (r0 + r1 + 1) >> 1;
      if (rowcs[mid] <= cta) r0 = mid; else r1 = mid - 1;
    }
    const int nt = (rowstart[r0 + 1] - rowstart[r0]) / hkv;
    const int n = (rowcs[r0 + 1] - rowcs[r0]) / hkv;
    // the row's n * hkv CTAs interleave its segments (CTA l of the row works
    // segment l % hkv): the CTAs dispatched last, which start and stream
    // later, are spread over every segment, whose pools absorb them
    const int g = (cta - rowcs[r0]) % hkv, part = (cta - rowcs[r0]) / hkv;
    const int s0 = rowstart[r0] + g * nt;
    if ((unsigned)nt < (1u << 31) / (unsigned)(n + 1)) {
      out[0] = s0 + (int)(((unsigned)part * (unsigned)nt) / (unsigned)n);
      out[1] = s0 + (int)(((unsigned)(part + 1) * (unsigned)nt) / (unsigned)n);
    } else {
      out[0] = s0 + (int)(((long long)part * nt) / n);
      out[1] = s0 + (int)(((long long)(part + 1) * nt) / n);
    }
    out[2] = rowcs[r0] + g * n;
    out[3] = n;
    out[4] = part;
  } else if (cta < h.P) {
    out[0] = (int)(((long long)cta * h.tot) / h.P);
    out[1] = (int)(((long long)(cta + 1) * h.tot) / h.P);
  }
}

// Layout of a plan in global memory (int32), for max_batch rows and `grid` CTAs.
struct PlanLayout {
  static __host__ __device__ int head() { return 0; }                       // [8]
  static __host__ __device__ int rowb(int) { return 8; }                    // [max_batch]
  static __host__ __device__ int rowt(int mb) { return 8 + mb; }           // [max_batch]
  static __host__ __device__ int rowstart(int mb) { return 8 + 2 * mb; }   // [max_batch+1]
  static __host__ __device__ int cta(int mb) { return 8 + 3 * mb + 1 + 7; } // [grid][8]
  static __host__ __device__ size_t ints(int mb, int grid) { return (size_t)cta(mb) + 8 * grid; }
};

// One block (warp 0 for the rows; every thread for the CTAs) writes a plan.
// smem: 4*max_batch + 2 ints.
__device__ __forceinline__ void plan_write(const PlanIn& p, int max_batch, int* plan, int* smem) {
  int* rowb = smem;
  int* rowt = rowb + max_batch;
  int* rowstart = rowt + max_batch;
  int* rowcs = rowstart + max_batch + 1;
  __shared__ PlanHead hs;
  if (threadIdx.x < 32) {
    const PlanHead h = plan_rows(p, rowb, rowt, rowstart, rowcs);
    if (threadIdx.x == 0) hs = h;
  }
  __syncthreads();
  const PlanHead h = hs;
  if (threadIdx.x == 0) {
    plan[PlanLayout::head() + 0] = h.nr;
    plan[PlanLayout::head() + 1] = h.tot;
    plan[PlanLayout::head() + 2] = h.P;
    plan[PlanLayout::head() + 3] = h.al;
  }
  for (int i = threadIdx.x; i < h.nr; i += blockDim.x) {
    plan[PlanLayout::rowb(max_batch) + i] = rowb[i];
    plan[PlanLayout::rowt(max_batch) + i] = rowt[i];
  }
  for (int i = threadIdx.x; i <= h.nr; i += blockDim.x)
    plan[PlanLayout::rowstart(max_batch) + i] = rowstart[i];
  for (int c = threadIdx.x; c < p.grid; c += blockDim.x) {
    int o[5];
    plan_cta(c, h, rowstart, rowcs, p.hkv, o);
    int* d = plan + PlanLayout::cta(max_batch) + 8 * c;
    d[0] = o[0]; d[1] = o[1]; d[2] = o[2]; d[3] = o[3]; d[4] = o[4];
  }
}

}  // namespace oda
