// Decode attention over the Local (ring) or Full (paged) access set.
//
// What it computes ([SUM] Methodology / Local-First Decoding): for a request
// at position t and query head h,
//   o_h = sum_{j in S} softmax_j(q_h . k_j / sqrt(d)) v_j,
// with S = S^L_t (ring source) or S^F_t = {1..t} (paged source, only for the
// rows the gate compacted into idx[0..count)), and KV head floor(h / G).
//
// How (B200 design, none of it from the pages):
//   * The work of one launch is the concatenation of "segments", one per
//     (row, KV head), each a run of 16-token tiles of [2][16][d] elements
//     (K rows then V rows, contiguous in both the ring and the paged cache).
//     A persistent grid sized to the SMs takes it: either each segment gets
//     its own CTAs in proportion to its length (aligned), with the last
//     tiles of a long segment in a pool that CTAs draw from one at a time,
//     or the tile space is split evenly (plan.cuh).
//   * Each warp streams its own tiles through NS shared-memory stages with
//     cp.async.bulk (TMA bulk copies) completing on mbarriers; waits are
//     bounded and a timeout is recorded, never trapped.
//   * q.k: a K/V row is LPR 16-byte chunks; lane (row group, chunk) holds its
//     chunk's dimensions of the G query heads in fp32 pairs and multiplies
//     with packed FMAs; a transposing butterfly over the row group's lanes
//     leaves one score per lane. Online softmax in base 2 (log2(e)/sqrt(d)
//     folded into the scores), fp32 accumulation on the CUDA cores: with
//     G = 2 query heads per KV head the contraction is too thin for tensor
//     cores.
//   * Warps of a CTA merge their states in shared memory. Then either CTAs
//     sharing a segment write (m, l, acc) partials and the last one to take
//     the segment's ticket merges them and writes the output, or (Local at
//     small batch) one thread-block cluster serves each segment and its
//     ranks merge through distributed shared memory.
//   * Launches chain with programmatic dependent launch; before its
//     dependency wait a kernel only warms L2 with the K/V it will read.

#include <mutex>

#include <cooperative_groups.h>
#include <stdlib.h>

#include "oda_internal.cuh"
#include "plan.cuh"

using namespace oda;

// Launch shape. The defaults were chosen by measurement on B200; the macros
// let a build try others without editing the source.
#ifndef ODA_ATTN_WARPS
#define ODA_ATTN_WARPS 6
#endif
#ifndef ODA_ATTN_STAGES
#define ODA_ATTN_STAGES 2
#endif
#ifndef ODA_RING_TILES_PER_WARP
#define ODA_RING_TILES_PER_WARP 1
#endif
#ifndef ODA_PREFETCH_TILES  // tiles per CTA warmed in L2 before the dependency wait
#define ODA_PREFETCH_TILES 16
#endif
#ifndef ODA_POOL_PERCENT
#define ODA_POOL_PERCENT 15
#endif
#ifndef ODA_FULL_TILES_PER_WARP
#define ODA_FULL_TILES_PER_WARP 1
#endif

namespace {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per barrier wait

struct AttnArgs {
  const void* q;
  void* out;
  float* lse;
  const int32_t* seq_lens;
  const void* kv;               // layer base (ring or paged cache)
  const int32_t* block_table;
  const int32_t* idx;
  const int32_t* count;
  long long num_blocks;
  int max_blocks;
  int B;
  int hkv;
  int sink;
  int window;
  int ring_blocks;
  int max_batch;
  int min_tiles_per_cta;
  float qscale;                 // log2(e) / sqrt(d)
  float* partials;               // [max_parts][G][d] accumulators, then [max_parts][G][2] (m, l)
  int max_parts;
  int* tickets;                 // per segment: CTAs done (reset by the last)
  int* dyn;                     // per segment: tiles handed out dynamically (reset by the last)
  const int* plan;              // precomputed partition, or null: compute it here
  int cluster;                  // cluster mode: CTAs per segment (= cluster size)
  int early;                    // stage the first tiles before the dependency wait
  const int32_t* range_lo;      // paged source: per-row region [lo, hi), or null (1..t)
  const int32_t* range_hi;
  int* err;
};

// 16-byte chunk of one K or V row, widened to float pairs (even, odd dims).
template <typename T>
struct Chunk;

template <>
struct Chunk<__nv_bfloat16> {
  static __device__ __forceinline__ void widen(const uint4 w, float2 (&x)[4]) {
    bf16x2_to_f32(w.x, x[0].x, x[0].y);
    bf16x2_to_f32(w.y, x[1].x, x[1].y);
    bf16x2_to_f32(w.z, x[2].x, x[2].y);
    bf16x2_to_f32(w.w, x[3].x, x[3].y);
  }
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float2 (&x)[4]) {
    widen(*reinterpret_cast<const uint4*>(p), x);
  }
};

template <>
struct Chunk<float> {
  static __device__ __forceinline__ void widen(const uint4 w, float2 (&x)[2]) {
    x[0] = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
    x[1] = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
  }
  static __device__ __forceinline__ void load(const float* p, float2 (&x)[2]) {
    widen(*reinterpret_cast<const uint4*>(p), x);
  }
};


// Bits [lo, hi) of a 16-bit tile mask whose bit 0 is slot `base`.
__device__ __forceinline__ uint32_t range_bits(int lo, int hi, int base) {
  int l = min(max(lo - base, 0), 16);
  int h = min(max(hi - base, 0), 16);
  if (h <= l) return 0u;
  return ((1u << h) - 1u) & ~((1u << l) - 1u);
}

// Pool size of an aligned segment of nt tiles over np CTAs of W warps.
__device__ __forceinline__ int pool_tiles(int nt, int np, int W) {
  return max(2 * np * W, nt * ODA_POOL_PERCENT / 100);
}

// Segment cursor over the CTA's tile range [lo, hi): segment (i, g) covers
// [s1 - nt, s1); rows with nt == 0 are skipped.
struct Cursor {
  int k;    // absolute tile index; == hi when exhausted
  int i;    // row slot
  int g;    // KV head
  int nt;   // tiles per segment of row i
  int s1;   // segment end
};

__device__ __forceinline__ void locate(const int* rowstart, int nrows, int hkv, int k, Cursor& c) {
  // largest i in [0, nrows) with rowstart[i] <= k
  int lo = 0, hi = nrows - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (rowstart[mid] <= k) lo = mid; else hi = mid - 1;
  }
  c.i = lo;
  c.nt = (rowstart[lo + 1] - rowstart[lo]) / hkv;
  const int rel = k - rowstart[lo];
  c.g = rel / c.nt;
  c.s1 = rowstart[lo] + (c.g + 1) * c.nt;
}

// Move c to the first tile >= c.k that belongs to this warp (offset `w`
// from its segment's start within [lo, hi), stride W), crossing segments.
__device__ __forceinline__ void normalize(const int* rowstart, int hkv, int hi, int w, Cursor& c) {
  while (c.k >= min(c.s1, hi)) {
    if (c.s1 >= hi) { c.k = hi; return; }
    int s0 = c.s1;
    if (++c.g == hkv) {
      c.g = 0;
      ++c.i;
      c.nt = (rowstart[c.i + 1] - rowstart[c.i]) / hkv;
    }
    c.s1 = s0 + c.nt;
    c.k = s0 + w;
  }
}

template <typename T, int D, int G>
struct Geom {
  static constexpr int ROWB = D * (int)sizeof(T);   // bytes of one K or V row
  static constexpr int LPR = ROWB / 16;             // lanes per row (one 16-byte chunk each)
  static constexpr int DPL = D / LPR;               // dims per lane
  static constexpr int RPW = 32 / LPR;              // row groups per warp
  static constexpr int TPL = 16 / RPW;              // tokens per lane per tile
  static constexpr int V = G * TPL;                 // q.k partial sums per lane per tile
  static constexpr int NVL = V >= LPR ? V / LPR : 1;  // scores per lane after the reduction
  static constexpr int DUP = V >= LPR ? 1 : LPR / V;  // lanes holding the same score
  static constexpr int LPHG = TPL * DUP / NVL;      // lanes of one query head in a row group
  static constexpr int R = LPR == 8 ? 3 : (LPR == 16 ? 4 : 5);  // butterfly rounds
  static_assert(LPR == 8 || LPR == 16 || LPR == 32, "row must be 128, 256 or 512 bytes");
};

template <typename T, int D, int G, int W, int NS, bool RING, bool CL>
__global__ void __launch_bounds__(W * 32, 2)
attn_kernel(const AttnArgs a) {
  using Gm = Geom<T, D, G>;
  constexpr int TILE_ELEMS = 2 * ODA_TILE * D;
  constexpr int TILE_BYTES = TILE_ELEMS * (int)sizeof(T);
  constexpr int LPR = Gm::LPR, DPL = Gm::DPL, RPW = Gm::RPW, TPL = Gm::TPL;
  constexpr int V = Gm::V, NVL = Gm::NVL, DUP = Gm::DUP, LPHG = Gm::LPHG;
  constexpr int DP2 = DPL / 2;                 // float pairs per lane
  constexpr int PW = G * 16 * 2;               // floats of {p, p} pairs per warp

  extern __shared__ __align__(128) unsigned char smem[];
  T* tiles = reinterpret_cast<T*>(smem);
  float* wstate = reinterpret_cast<float*>(smem + (size_t)W * NS * TILE_BYTES);  // [W][G][D+2]
  uint64_t* bars = reinterpret_cast<uint64_t*>(wstate + W * G * (D + 2) + (W * G * (D + 2)) % 2);
  float* pbuf = reinterpret_cast<float*>(bars + W * NS);          // [W][G][RPW][TPL] x {p,p}
  int* rowstart = reinterpret_cast<int*>(pbuf + W * PW);          // [max_batch+1]
  int* rowb = rowstart + (a.max_batch + 1);
  int* rowt = rowb + a.max_batch;
  int* rowcs = rowt + a.max_batch;                                 // [max_batch+1] CTA prefix
  int* sflag = rowcs + (a.max_batch + 1);
  int* sinfo = sflag + 4;                                          // [16] partition of this CTA
  int* stile = sinfo + 16;                                         // [W][NS] tile of each stage
  unsigned char* badst = reinterpret_cast<unsigned char*>(stile + W * NS);  // [W][NS]
  float* racc = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(badst + W * NS) + 15) & ~uintptr_t(15));  // CL: [cs][G*D/cs]
  float* rml = racc + G * D;                   // CL: [16][G] pushed (m, l) pairs
  constexpr int QCH = G * D * (int)sizeof(T) / 16;  // 16-byte chunks of one segment's queries
  uint4* sq = reinterpret_cast<uint4*>(rml + 32 * G);   // [QCH] the current segment's queries
  int* st_t = reinterpret_cast<int*>(sq + QCH);         // cluster mode: the row's t
  int* rowlo = st_t + 4;                                // paged: [max_batch] first position read
  int* spool = rowlo + a.max_batch;                     // [W][4] pool grabs ahead (lane 0)

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int rg = lane / LPR;                   // row group: tokens rg, rg+RPW, ...
  const int li = lane % LPR;                   // 16-byte chunk of the row this lane owns
  const int hq = a.hkv * G;
  if (tid < W * NS) mbar_init(smem_addr(&bars[tid]), 1);
  fence_mbar_init();
  // Early mode: the caller guarantees that the K/V source, the lengths, the
  // block table and the compacted ids were complete before the previous
  // kernel on the stream passed its own dependency wait (every kernel of this
  // library waits before it lets dependents start), so this launch works out
  // its partition and issues its first tile copies into shared memory before
  // its own wait. The queries, the scratch (partials, tickets, pool counters)
  // and the outputs are touched only after the wait.
  const bool early = a.early != 0;
  if constexpr (CL) {
    cluster_arrive_relaxed();                    // "started": waited for before any remote store
    const int cs = a.cluster;
    const int sg = (int)blockIdx.x / cs, rank = (int)blockIdx.x % cs;
    if (early) {
      // this segment's queries into L2 (a prefetch returns no value)
      if (tid == 0)
        bulk_prefetch_l2(reinterpret_cast<const T*>(a.q) +
                             ((long long)(sg / a.hkv) * hq + (sg % a.hkv) * G) * D,
                         G * D * (int)sizeof(T));
    } else {
      // Before the dependency wait, warm L2 with this rank's share of a full
      // ring (its share once t >= w). This reads no value: L2 is the point of
      // coherence, so the loads after the wait still see every earlier write,
      // and the prefetch overlaps the tail of the preceding kernel.
      const int rb = a.ring_blocks;
      const int k0 = (rank * rb) / cs, k1 = ((rank + 1) * rb) / cs;
      const T* base = reinterpret_cast<const T*>(a.kv) + (long long)sg * rb * TILE_ELEMS;
      for (int k = k0 + tid; k < k1; k += W * 32)
        bulk_prefetch_l2(base + (long long)k * TILE_ELEMS, TILE_BYTES);
    }
  }
  // ------------------------------------------------------- rows, partition
  // Either read the plan another kernel wrote once for every launch that
  // shares it (one round trip of independent loads), or work it out here on
  // warp 0; one barrier then publishes it through sinfo.
  auto partition = [&](bool report) {          // warp 0, non-cluster modes
    if (a.plan) {
      const int* pl = a.plan;
      const int mb = a.max_batch;
      const int hv = lane < 8 ? __ldcg(pl + PlanLayout::head() + lane) : 0;
      const int dv = (lane >= 8 && lane < 13)
          ? __ldcg(pl + PlanLayout::cta(mb) + 8 * (int)blockIdx.x + (lane - 8))
          : 0;
      for (int i = lane; i < a.B; i += 32) {
        rowb[i] = __ldcg(pl + PlanLayout::rowb(mb) + i);
        rowt[i] = __ldcg(pl + PlanLayout::rowt(mb) + i);
      }
      for (int i = lane; i <= a.B; i += 32) rowstart[i] = __ldcg(pl + PlanLayout::rowstart(mb) + i);
      if (lane < 4) sinfo[lane] = hv;                 // nr, tot, P, al
      if (lane >= 8 && lane < 13) sinfo[4 + lane - 8] = dv;   // lo, hi, pbase, nparts, part
      if (lane == 0) sinfo[9] = (int)blockIdx.x;
    } else {
      PlanIn pin;
      pin.B = a.B;
      pin.count = RING ? nullptr : a.count;
      pin.idx = a.idx;
      pin.seq_lens = a.seq_lens;
      pin.hkv = a.hkv;
      pin.sink = a.sink;
      pin.window = a.window;
      pin.max_blocks = a.max_blocks;
      pin.min_tiles = a.min_tiles_per_cta;
      pin.grid = (int)gridDim.x;
      pin.err = a.err;
      pin.report = report && blockIdx.x == 0;
      pin.range_lo = a.range_lo;
      pin.range_hi = a.range_hi;
      const PlanHead h = plan_rows(pin, rowb, rowt, rowstart, rowcs, RING ? nullptr : rowlo);
      if (lane == 0) {
        int o[5];
        plan_cta((int)blockIdx.x, h, rowstart, rowcs, a.hkv, o);
        sinfo[0] = h.nr; sinfo[1] = h.tot; sinfo[2] = h.P; sinfo[3] = h.al;
        sinfo[4] = o[0]; sinfo[5] = o[1]; sinfo[6] = o[2]; sinfo[7] = o[3]; sinfo[8] = o[4];
        sinfo[9] = (int)blockIdx.x;
      }
    }
  };

#if ODA_PREFETCH_TILES > 0
  static_assert(ODA_PREFETCH_TILES <= 32, "one prefetched tile per lane of warp 0");
  if constexpr (!CL) {
    // Without early staging: before the dependency wait, warp 0 works out the partition from values
    // that the preceding launch may still be writing, and warms L2 with the
    // first tiles of this CTA's static share. Nothing read here is used after
    // the wait (the partition is worked out again), and an L2 prefetch reads
    // no value, so a stale guess only costs bandwidth; every address is
    // bounds-checked like the loads proper.
    if (!early && warp == 0) {
      partition(false);
      __syncwarp();
      const int nr = sinfo[0], tot = sinfo[1];
      int plo = sinfo[4], phi = sinfo[5];
      if (nr > 0 && nr <= a.B && tot > 0 && plo >= 0 && plo < phi && phi <= tot) {
        Cursor c;
        locate(rowstart, nr, a.hkv, plo, c);
        const int nt = c.nt, s0 = c.s1 - c.nt, np = sinfo[7], pt = sinfo[8];
        if (sinfo[3] && np > 0 && nt >= 8 * np * W) {
          const int p0 = nt - pool_tiles(nt, np, W);
          plo = s0 + (int)(((long long)pt * p0) / np);
          phi = s0 + (int)(((long long)(pt + 1) * p0) / np);
        }
        const int k = plo + lane;
        if (lane < ODA_PREFETCH_TILES && k < phi) {
          Cursor ck;
          locate(rowstart, nr, a.hkv, k, ck);
          const int jt = k - (rowstart[ck.i] + ck.g * ck.nt);
          const int b = rowb[ck.i];
          const T* kb = reinterpret_cast<const T*>(a.kv);
          const bool ok = b >= 0 && b < a.B && ck.g >= 0 && ck.g < a.hkv && jt >= 0;
          if (RING) {
            if (ok && jt < a.ring_blocks)
              bulk_prefetch_l2(kb + (((long long)b * a.hkv + ck.g) * a.ring_blocks + jt) * TILE_ELEMS,
                               TILE_BYTES);
          } else if (ok && jt + (rowlo[ck.i] - 1) / ODA_TILE < a.max_blocks) {
            const int blk = __ldcg(a.block_table + (long long)b * a.max_blocks + jt +
                                   (rowlo[ck.i] - 1) / ODA_TILE);
            if (blk >= 0 && (long long)blk < a.num_blocks)
              bulk_prefetch_l2(kb + ((long long)blk * a.hkv + ck.g) * TILE_ELEMS, TILE_BYTES);
          }
        }
      }
      __syncwarp();
    }
  }
#endif
  if (!early) {
    pdl_wait();
    pdl_launch_dependents();
  }
  float* pacc = a.partials;                                         // [max_parts][G][D]
  float* pml = a.partials + (size_t)a.max_parts * G * D;            // [max_parts][G][2]

  if (warp == 0) {
    if (CL) {
      // cluster mode: segment = cluster; the ranks split the whole ring
      // evenly, whatever t is (tiles past the valid slots are masked), so the
      // first copies need no global load; t itself is read by the consumer
      if (lane == 0) {
        const int cs = a.cluster;
        const int sg = (int)blockIdx.x / cs, rank = (int)blockIdx.x % cs;
        const int g = sg % a.hkv;
        const int nt = a.ring_blocks;
        rowb[0] = sg / a.hkv;                    // < B: the grid is B * hkv * cs
        rowstart[0] = 0;
        rowstart[1] = nt * a.hkv;
        sinfo[0] = 1; sinfo[1] = nt * a.hkv; sinfo[2] = (int)gridDim.x; sinfo[3] = 1;
        sinfo[4] = g * nt + (rank * nt) / cs;
        sinfo[5] = g * nt + ((rank + 1) * nt) / cs;
        sinfo[6] = 0; sinfo[7] = cs; sinfo[8] = rank; sinfo[9] = (int)blockIdx.x;
      }
    } else {
      partition(true);
    }
  }
  __syncthreads();
  const int nrows = sinfo[0];
  const int total = sinfo[1];
  const int P = sinfo[2];
  const bool aligned = sinfo[3] != 0;
  int lo = sinfo[4], hi = sinfo[5];
  const int pbase_al = sinfo[6], nparts_al = sinfo[7], part_al = sinfo[8];
  // partial slot of this CTA: its segment's own range in the aligned partition
  const int vcta = (sinfo[3] && !CL) ? pbase_al + part_al : sinfo[9];
  const int cta = (int)blockIdx.x;
  // Cluster mode: each rank owns G*D/cs output elements of the segment. A
  // rank merges its warps' states (or takes an empty one) and pushes, with
  // remote shared-memory stores, its accumulator for every element to the
  // element's owner and each head's (m, l) to every rank. The caller has
  // waited for the barrier every rank arrived at on entry, so every target
  // CTA has started.
  auto cluster_push = [&](bool filled) {
    if constexpr (CL) {
      namespace cg = cooperative_groups;
      cg::cluster_group cl = cg::this_cluster();
      const int cs = a.cluster;
      const int rank = (int)cl.block_rank();
      const int per = (G * D) / cs;
      for (int o = tid; o < G * D; o += W * 32) {
        const int h = o / D, dd = o % D;
        float mt = -INFINITY, lt = 0.f, at = 0.f;
        if (filled) {
          for (int w2 = 0; w2 < W; ++w2) mt = fmaxf(mt, wstate[(w2 * G + h) * (D + 2) + D]);
          if (mt != -INFINITY) {
            for (int w2 = 0; w2 < W; ++w2) {
              const float* st = wstate + (w2 * G + h) * (D + 2);
              if (st[D] == -INFINITY) continue;
              const float sc2 = fast_exp2(st[D] - mt);
              lt += st[D + 1] * sc2;
              at += st[dd] * sc2;
            }
          }
        }
        cl.map_shared_rank(racc, o / per)[rank * per + o % per] = at;
        if (dd < cs)
          reinterpret_cast<float2*>(cl.map_shared_rank(rml, dd))[rank * G + h] =
              make_float2(mt, lt);
      }
    }
  };
  const bool has_work = nrows > 0 && total > 0 && lo < hi;

  // K/V is read once per launch: stream it through L2 (the ring too, so no
  // layer's window stays resident from one step to the next)
  const uint64_t policy = l2_policy_evict_first();
  const T* kvbase = reinterpret_cast<const T*>(a.kv);

  // -------------------------------------------------------- tile producer
  // Each warp walks its CTA's tile range with stride W. In the aligned
  // partition a long segment keeps its last ODA_POOL_PERCENT % of tiles in a
  // pool: a warp that finishes its static share takes pool tiles one at a
  // time from the segment's counter, so warps that stream faster take more
  // and the segment's CTAs finish together. Grabs run ahead of use without
  // waiting on a round trip: three tiles before the end of its static share
  // a warp takes three counter values, one tile later it looks up the first
  // two tiles' blocks, and from then on each grab's counter value is looked
  // up one tile after it was taken and used one tile after that. The pool
  // counters are scratch: they are touched only after the wait.
  Cursor prod;
  prod.k = prod.i = prod.g = prod.nt = prod.s1 = 0;
  int seg_b = 0, seg_g0 = 0, seg_nt = 0, seg_s0 = 0, sigma0 = 0;
  int pool0 = 0;                             // first pool tile (relative); == nt: no pool
  bool use_pool = false;
  // lane 0: the next pool tile and its block in registers; the one after it,
  // its block and a counter value not looked up yet in spool[warp] (q1, qb1, gp)
  int q0 = 0, qb0 = -1;
  int* sp = spool + 4 * warp;
  int pool_state = 0;                        // warp-uniform: 0 none, 1 counters taken, 2 armed
  auto lookup = [&](int q) -> int {          // lane 0: the block of pool tile q
    // (the pool belongs to the first segment, row sigma0 / hkv)
    return (!RING && q < seg_nt)
               ? a.block_table[(long long)seg_b * a.max_blocks +
                               (rowlo[sigma0 / a.hkv] - 1) / ODA_TILE + q]
               : -1;
  };
  auto prime_pool = [&]() {                  // warp, after the dependency wait, per refill
    if (pool_state == 0 && prod.k + 3 * W >= hi) {
      if (lane == 0) sp[2] = atomicAdd(&a.dyn[sigma0], 3);
      pool_state = 1;
    } else if (pool_state == 1 && prod.k + 2 * W >= hi) {
      if (lane == 0) {
        const int g3 = sp[2];
        q0 = pool0 + g3;
        qb0 = lookup(q0);
        sp[0] = q0 + 1;
        sp[1] = lookup(q0 + 1);
        sp[2] = g3 + 2;
      }
      pool_state = 2;
    }
  };

  // Block ids of the producer's next 32 tiles of the current row, one per
  // lane, so the per-tile issue does not wait on a global load.
  int bc_row = -1, bc_base = 0, bc_val = -1;

  // Warp-uniform: the next tile of this warp. Returns false when done.
  // Sets (k, i, g, nt, blk); blk < -1 means "look it up in the block cache".
  auto next_tile = [&](int& k, int& i, int& g, int& nt, int& blk) -> bool {
    if (prod.k < hi) {
      k = prod.k; i = prod.i; g = prod.g; nt = prod.nt; blk = -2;
      prod.k += W;
      normalize(rowstart, a.hkv, hi, warp, prod);
      return true;
    }
    if (!use_pool || pool_state < 2) return false;
    const int rel = __shfl_sync(0xffffffffu, q0, 0);
    blk = __shfl_sync(0xffffffffu, qb0, 0);
    if (rel >= seg_nt) return false;
    if (lane == 0) {
      q0 = sp[0];
      qb0 = sp[1];
      const int q1 = pool0 + sp[2];          // taken one tile ago
      sp[0] = q1;
      sp[1] = lookup(q1);                    // needed one tile from now
      sp[2] = atomicAdd(&a.dyn[sigma0], 1);
    }
    k = seg_s0 + rel; i = prod.i; g = prod.g; nt = seg_nt;
    return true;
  };

  // Warp-uniform; lane 0 issues the copy and records the stage's tile.
  auto issue = [&](int k, int i, int g, int nt, int blk_in, int stage) {
    const int b = rowb[i];
    const int jt = k - (rowstart[i] + g * nt);
    const T* src;
    bool bad = false;
    if (RING) {
      src = kvbase + (((long long)b * a.hkv + g) * a.ring_blocks + jt) * TILE_ELEMS;
    } else {
      int blk = blk_in;
      if (blk < -1) {
        if (i != bc_row || jt < bc_base || jt >= bc_base + 32 * W || (jt - bc_base) % W != 0) {
          bc_row = i;
          bc_base = jt;
          const int jl = jt + lane * W;
          const int tb = (rowlo[i] - 1) / ODA_TILE;
          bc_val = jl < nt ? a.block_table[(long long)b * a.max_blocks + tb + jl] : -1;
        }
        blk = __shfl_sync(0xffffffffu, bc_val, (jt - bc_base) / W);
      }
      bad = blk < 0 || (long long)blk >= a.num_blocks;
      src = kvbase + ((long long)blk * a.hkv + g) * TILE_ELEMS;
    }
    if (lane == 0) {
      const uint32_t bar = smem_addr(&bars[warp * NS + stage]);
      stile[warp * NS + stage] = k;
      badst[warp * NS + stage] = bad ? 1 : 0;
      if (bad) {
        record_error(a.err, ODA_ERR_BOUNDS);
        mbar_arrive(bar);
      } else {
        const uint32_t dst = smem_addr(tiles + (size_t)(warp * NS + stage) * TILE_ELEMS);
        mbar_arrive_expect_tx(bar, TILE_BYTES);
        bulk_g2s(dst, src, TILE_BYTES, bar, policy);
      }
    }
  };

  // A segment's queries (and, in cluster mode, its row's t) are read once per
  // CTA by warp 0 into shared memory: one request per CTA instead of one per
  // warp keeps the hot lines of q from queueing at their L2 slice. Cluster
  // mode has one segment per CTA, loaded here while the first copies fly.
  // The copies are asynchronous (cp.async, no registers held) and awaited by
  // warp 0 after whatever the caller overlaps with them (cluster mode: the
  // wait for every rank); a barrier of the caller's then publishes them.
  auto load_q = [&](int row, int g, bool with_t) {   // warp 0: issue
    const unsigned char* src = reinterpret_cast<const unsigned char*>(a.q) +
                               ((long long)row * hq + g * G) * D * (long long)sizeof(T);
    for (int c = lane; c < QCH; c += 32) cp_async16(smem_addr(sq + c), src + 16 * c);
    if (with_t && lane == 0) cp_async4(smem_addr(st_t), a.seq_lens + row);
  };
  auto store_q = [&](bool) {                         // warp 0: the copies have landed
    cp_async_wait_all();
  };
  // Without early staging the first segment's queries are requested before
  // the first tile copies, so they do not queue behind them.
  bool q_loaded = false;
  int issued = 0;
  bool prod_done = false;
  if (has_work) {
    prod.k = lo;
    locate(rowstart, nrows, a.hkv, lo, prod);
    seg_b = rowb[prod.i];
    seg_g0 = prod.g;
    seg_nt = prod.nt;
    seg_s0 = prod.s1 - prod.nt;
    sigma0 = prod.i * a.hkv + prod.g;
    pool0 = seg_nt;
    if (!CL && aligned && seg_nt >= 8 * nparts_al * W) {
      pool0 = seg_nt - pool_tiles(seg_nt, nparts_al, W);
      // static share of this CTA within [0, pool0)
      lo = seg_s0 + (int)(((long long)part_al * pool0) / nparts_al);
      hi = seg_s0 + (int)(((long long)(part_al + 1) * pool0) / nparts_al);
    }
    use_pool = pool0 < seg_nt;
    q0 = seg_nt;
    if (!early) {
      if (warp == 0) load_q(seg_b, seg_g0, CL);
      q_loaded = true;
    }
    if (!CL && early && tid == 0)
      // the first segment's queries into L2 (a prefetch returns no value)
      bulk_prefetch_l2(reinterpret_cast<const T*>(a.q) +
                           ((long long)seg_b * hq + prod.g * G) * D,
                       G * D * (int)sizeof(T));
    prod.k = lo + warp;
    if (prod.k >= hi) prod.k = hi;
    normalize(rowstart, a.hkv, hi, warp, prod);
#pragma unroll 1
    for (int st2 = 0; st2 < NS; ++st2) {
      int k, i, g, nt, blk;
      if (!next_tile(k, i, g, nt, blk)) { prod_done = true; break; }
      issue(k, i, g, nt, blk, st2);
      ++issued;
    }
  }
  if (early) {
    pdl_wait();
    pdl_launch_dependents();
  }

  // (cluster mode never leaves early: every CTA takes part in the merge)
  if (!CL && !has_work) return;
  if (CL && !has_work) {
    cluster_wait();                              // every rank has started
    cluster_push(false);                         // an empty state: m = -inf, l = acc = 0
  } else {

  uint4 qraw[G];
  int tpre = 0;
  if constexpr (CL) {
    if (warp == 0 && !q_loaded) load_q(seg_b, seg_g0, true);
    cluster_wait();                              // every rank has started (overlaps the loads)
    if (warp == 0) store_q(true);
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h) qraw[h] = sq[h * LPR + li];
    tpre = st_t[0];
  }
  __syncwarp();
  int consumed = 0;
  int waited = 0;        // tiles whose copy is known to have landed
  bool aborted = false;

  // ------------------------------------------------------- segment loop
  Cursor seg;
  seg.k = lo;
  locate(rowstart, nrows, a.hkv, lo, seg);
  while (true) {
    const int b = rowb[seg.i];
    int t;
    if (CL) {
      t = tpre;                                  // loaded once per CTA
      if (t < 1) {
        if (tid == 0 && (int)blockIdx.x % a.cluster == 0) record_error(a.err, ODA_ERR_BOUNDS);
        t = 0;                                   // every slot masked: an empty state
      }
    } else {
      t = rowt[seg.i];
    }
    // paged source: positions first..t are read; relative to the segment's
    // first tile they are the slots [plo, phi)
    int plo = 0, phi = t;
    if constexpr (!RING) {
      const int first = rowlo[seg.i];
      const int base = (first - 1) / ODA_TILE * ODA_TILE;
      plo = first - 1 - base;
      phi = t - base;
    }
    const int s0 = seg.s1 - seg.nt;

    // this lane's DPL dims of the G query heads (exact, unscaled)
    float2 q2[G][DP2];
    if constexpr (!CL) {
      if (warp == 0) {
        if (!q_loaded) load_q(b, seg.g, false);   // else requested with the first copies
        store_q(false);
      }
      q_loaded = false;
      __syncthreads();
#pragma unroll
      for (int h = 0; h < G; ++h) qraw[h] = sq[h * LPR + li];
    }
#pragma unroll
    for (int h = 0; h < G; ++h) Chunk<T>::widen(qraw[h], q2[h]);
    float m_run[G], l_run[G];
    float2 acc[G][DP2];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_run[h] = -INFINITY;
      l_run[h] = 0.f;
#pragma unroll
      for (int e = 0; e < DP2; ++e) acc[h][e] = make_float2(0.f, 0.f);
    }

    // ring validity constants of this row
    const int mw = min(t, a.window);
    const int nsv = min(max(t - a.window, 0), a.sink);

#pragma unroll 1
    while (consumed < issued) {
      const int stage = consumed % NS;
      const int ktile = stile[warp * NS + stage];
      if (ktile >= seg.s1) break;              // the next tile belongs to a later segment
      const uint32_t parity = (uint32_t)((consumed / NS) & 1);
      if (!aborted) {
        // every lane waits; the warp proceeds only if all of them saw the data
        const bool ok = __all_sync(0xffffffffu,
            mbar_wait_bounded(smem_addr(&bars[warp * NS + stage]), parity, kWaitLimitNs));
        if (ok) {
          ++waited;
        } else {
          aborted = true;
          if (lane == 0) record_error(a.err, ODA_ERR_TIMEOUT);
        }
      }
      const int jt = ktile - s0;
      uint32_t mask;
      if (RING) {
        const int base = jt * ODA_TILE;
        mask = range_bits(a.sink, a.sink + mw, base) | range_bits(0, nsv, base);
      } else {
        mask = range_bits(plo, phi, jt * ODA_TILE);
      }
      if (badst[warp * NS + stage] || aborted) mask = 0;

      if (mask) {
        const T* tk = tiles + (size_t)(warp * NS + stage) * TILE_ELEMS;
        const T* tv = tk + ODA_TILE * D;
        // ---- q.k partial sums over this lane's chunk: x[h*TPL + u], token rg + RPW*u
        float x[V];
#pragma unroll
        for (int u = 0; u < TPL; ++u) {
          float2 kf[DP2];
          Chunk<T>::load(tk + (rg + RPW * u) * D + li * DPL, kf);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < DP2; ++e) s2 = __ffma2_rn(q2[h][e], kf[e], s2);
            x[h * TPL + u] = s2.x + s2.y;
          }
        }
        // ---- transposing butterfly over the LPR lanes of the row group
        {
          int c = V;
#pragma unroll
          for (int r = 0; r < Gm::R; ++r) {
            const int off = LPR >> (r + 1);
            if (c > 1) {
              const bool upper = (lane & off) != 0;
              const int half = c >> 1;
#pragma unroll
              for (int i2 = 0; i2 < V / 2; ++i2) {
                if (i2 < half) {
                  const float send = upper ? x[i2] : x[i2 + half];
                  const float keep = upper ? x[i2 + half] : x[i2];
                  x[i2] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
              }
              c = half;
            } else {
              x[0] += __shfl_xor_sync(0xffffffffu, x[0], off);
            }
          }
        }
        // scores of this lane: index v = h*TPL + u, token rg + RPW*u
        float sc[NVL];
        int myh = 0;
#pragma unroll
        for (int e = 0; e < NVL; ++e) {
          const int v = V >= LPR ? li * NVL + e : li / DUP;
          const int u = v % TPL;
          myh = v / TPL;
          const int j = rg + RPW * u;
          sc[e] = ((mask >> j) & 1u) ? x[e] * a.qscale : -INFINITY;
        }
        // ---- per-head tile max (within the row group, then across groups)
        float mx = sc[0];
#pragma unroll
        for (int e = 1; e < NVL; ++e) mx = fmaxf(mx, sc[e]);
#pragma unroll
        for (int o = DUP; o < LPHG; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float m_new[G], alpha[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float th = __shfl_sync(0xffffffffu, mx, h * LPHG);
          m_new[h] = fmaxf(m_run[h], th);
          alpha[h] = (m_run[h] == -INFINITY) ? 0.f : fast_exp2(m_run[h] - m_new[h]);
        }
        float mine = m_new[0];
#pragma unroll
        for (int h = 1; h < G; ++h) if (myh == h) mine = m_new[h];
        float p[NVL];
        float ps = 0.f;
#pragma unroll
        for (int e = 0; e < NVL; ++e) {
          p[e] = (sc[e] == -INFINITY) ? 0.f : fast_exp2(sc[e] - mine);
          ps += p[e];
        }
#pragma unroll
        for (int o = DUP; o < LPHG; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float tsum = __shfl_sync(0xffffffffu, ps, h * LPHG);
          l_run[h] = l_run[h] * alpha[h] + tsum;
          m_run[h] = m_new[h];
          const float2 a2 = make_float2(alpha[h], alpha[h]);
#pragma unroll
          for (int e = 0; e < DP2; ++e) acc[h][e] = __fmul2_rn(acc[h][e], a2);
        }
        // ---- {p, p} pairs to shared memory, laid out [G][RPW][TPL]
        float2* pw = reinterpret_cast<float2*>(pbuf + warp * PW);
        if (li % DUP == 0) {
#pragma unroll
          for (int e = 0; e < NVL; ++e) {
            const int v = V >= LPR ? li * NVL + e : li / DUP;
            pw[((v / TPL) * RPW + rg) * TPL + v % TPL] = make_float2(p[e], p[e]);
          }
        }
        __syncwarp();
        // ---- P.V over this row group's tokens
        if (mask == 0xFFFFu) {
#pragma unroll
          for (int u = 0; u < TPL; ++u) {
            float2 vf[DP2];
            Chunk<T>::load(tv + (rg + RPW * u) * D + li * DPL, vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float2 pp = pw[(h * RPW + rg) * TPL + u];
#pragma unroll
              for (int e = 0; e < DP2; ++e) acc[h][e] = __ffma2_rn(pp, vf[e], acc[h][e]);
            }
          }
        } else {
#pragma unroll 1
          for (int u = 0; u < TPL; ++u) {
            if (!((mask >> (rg + RPW * u)) & 1u)) continue;   // masked slots may hold garbage
            float2 vf[DP2];
            Chunk<T>::load(tv + (rg + RPW * u) * D + li * DPL, vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float2 pp = pw[(h * RPW + rg) * TPL + u];
#pragma unroll
              for (int e = 0; e < DP2; ++e) acc[h][e] = __ffma2_rn(pp, vf[e], acc[h][e]);
            }
          }
        }
      }
      __syncwarp();
      // refill the stage just consumed
      if (!prod_done && !aborted) {
        int k, i, g, nt, blk;
        if (use_pool) prime_pool();
        if (next_tile(k, i, g, nt, blk)) {
          issue(k, i, g, nt, blk, stage);
          ++issued;
        } else {
          prod_done = true;
        }
        __syncwarp();
      }
      ++consumed;
    }

    // ---------------------------------------------- merge warps of the CTA
    // row groups hold disjoint tokens under the same running max: add them
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < DP2; ++e) {
          acc[h][e].x += __shfl_xor_sync(0xffffffffu, acc[h][e].x, o);
          acc[h][e].y += __shfl_xor_sync(0xffffffffu, acc[h][e].y, o);
        }
    float* ws = wstate + (size_t)warp * G * (D + 2);
    if (rg == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < DP2; ++e)
          *reinterpret_cast<float2*>(ws + h * (D + 2) + li * DPL + 2 * e) = acc[h][e];
    }
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        ws[h * (D + 2) + D] = m_run[h];
        ws[h * (D + 2) + D + 1] = l_run[h];
      }
    }
    __syncthreads();

    if constexpr (CL) {
      // cluster mode (one segment per CTA, so the loop ends here): merge the
      // warps and push each output element's accumulator straight to the
      // rank that owns it, and each head's (m, l) to every rank
      cluster_push(true);
      break;
    }

    const int sigma = seg.i * a.hkv + seg.g;
    // the segment's partials are pbase .. pbase+nparts-1; this CTA writes mypart
    int pbase, nparts, mypart;
    if (aligned) {
      pbase = pbase_al;
      nparts = nparts_al;
      mypart = vcta;
    } else {
      const long long Pll = P;
      const int c_first = (int)(((long long)(s0 + 1) * Pll - 1) / total);
      const int c_last = (int)(((long long)seg.s1 * Pll - 1) / total);
      pbase = c_first + sigma;
      nparts = c_last - c_first + 1;
      mypart = cta + sigma;
    }
    const int hglob0 = seg.g * G;
    T* outp = reinterpret_cast<T*>(a.out);

    for (int o = tid; o < G * D; o += W * 32) {
      const int h = o / D, dd = o % D;
      float mt = -INFINITY;
      for (int w2 = 0; w2 < W; ++w2) mt = fmaxf(mt, wstate[(w2 * G + h) * (D + 2) + D]);
      float lt = 0.f, at = 0.f;
      if (mt != -INFINITY) {
        for (int w2 = 0; w2 < W; ++w2) {
          const float* st = wstate + (w2 * G + h) * (D + 2);
          if (st[D] == -INFINITY) continue;
          const float sc2 = fast_exp2(st[D] - mt);
          lt += st[D + 1] * sc2;
          at += st[dd] * sc2;
        }
      }
      if (nparts == 1) {
        const long long orow = ((long long)b * hq + hglob0 + h) * D;
        outp[orow + dd] = (T)(lt > 0.f ? at / lt : 0.f);
        if (dd == 0 && a.lse)
          a.lse[(long long)b * hq + hglob0 + h] =
              lt > 0.f ? (mt + fast_log2(lt)) * 0.69314718055994531f : -INFINITY;
      } else {
        const long long pidx = (long long)mypart * G + h;
        pacc[pidx * D + dd] = at;
        if (dd == 0) { pml[pidx * 2] = mt; pml[pidx * 2 + 1] = lt; }
      }
    }
    if (nparts > 1) {
      __syncthreads();
      if (tid == 0) {
        const int prev = ticket_add(&a.tickets[sigma], 1);   // releases this CTA's partial
        sflag[0] = (prev == nparts - 1) ? 1 : 0;
      }
      __syncthreads();
      if (sflag[0]) {
        // (the last ticket acquired every other CTA's partial)
        // Last CTA of the segment: merge its nparts partials. The accumulator
        // loads are issued before the (m, l) reduction so both travel in one
        // L2 round trip.
        constexpr int NCH = G * D / 4;                 // float4 chunks of the output
        constexpr int SPLIT = (W * 32) / NCH > 0 ? (W * 32) / NCH : 1;
        constexpr int MAXB = G >= 4 ? 4 : (G == 2 ? 16 : 8);   // partial chunks held per thread
        float* sml = wstate;                           // [nparts][G][2]
        float* ssc = sml + 2 * nparts * G;             // [nparts][G] scale factors
        float* stot = ssc + nparts * G;                // [2G]: m_tot, l_tot
        const int comb_off = (3 * nparts * G + 2 * G + 3) & ~3;
        float4* scomb = reinterpret_cast<float4*>(wstate + comb_off);   // [SPLIT-1][NCH]
        const bool fits = comb_off + 4 * NCH * (SPLIT - 1) <= W * G * (D + 2) &&
                          (SPLIT > 1 || NCH <= W * 32) && nparts <= SPLIT * MAXB * 4;
        if (!fits) {
          // many partials (few segments over a large grid): one output element
          // per thread, partials in turn
          for (int o = tid; o < G * D; o += W * 32) {
            const int h = o / D, dd = o % D;
            float mt = -INFINITY;
            for (int j = 0; j < nparts; ++j)
              mt = fmaxf(mt, __ldcg(pml + ((long long)(pbase + j) * G + h) * 2));
            float lt = 0.f, at = 0.f;
            if (mt != -INFINITY) {
              for (int j = 0; j < nparts; ++j) {
                const long long pidx = (long long)(pbase + j) * G + h;
                const float pm = __ldcg(pml + pidx * 2);
                if (pm == -INFINITY) continue;
                const float sc2 = fast_exp2(pm - mt);
                lt += __ldcg(pml + pidx * 2 + 1) * sc2;
                at += __ldcg(pacc + pidx * D + dd) * sc2;
              }
            }
            const long long orow = ((long long)b * hq + hglob0 + h) * D;
            outp[orow + dd] = (T)(lt > 0.f ? at / lt : 0.f);
            if (dd == 0 && a.lse)
              a.lse[(long long)b * hq + hglob0 + h] =
                  lt > 0.f ? (mt + fast_log2(lt)) * 0.69314718055994531f : -INFINITY;
          }
        } else {
          // thread -> (output chunk ch, partials part, part + SPLIT, ...)
          const int ch = tid % NCH;
          const int part = (tid / NCH < SPLIT && tid < NCH * SPLIT) ? tid / NCH : SPLIT;
          const int hch = (ch * 4) / D;
          float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
          float4 v4[MAXB];
          int nb = 0;                                   // chunks loaded in the first batch
          if (part < SPLIT) {
#pragma unroll
            for (int u = 0; u < MAXB; ++u) {
              const int j = part + u * SPLIT;
              if (j < nparts) {
                v4[u] = __ldcg(reinterpret_cast<const float4*>(
                    pacc + (long long)(pbase + j) * G * D) + ch);
                nb = u + 1;
              }
            }
          }
          // (a) every partial's (m, l)
          for (int i = tid; i < nparts * G; i += W * 32) {
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(
                pml + ((long long)(pbase + i / G) * G + (i % G)) * 2));
            sml[2 * i] = ml.x;
            sml[2 * i + 1] = ml.y;
          }
          __syncthreads();
          // (b) one warp per head: max, per-partial scales, normaliser
          if (warp < G) {
            const int h = warp;
            float mx = -INFINITY;
            for (int j = lane; j < nparts; j += 32) mx = fmaxf(mx, sml[2 * (j * G + h)]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float ls = 0.f;
            for (int j = lane; j < nparts; j += 32) {
              const float pm = sml[2 * (j * G + h)];
              const float s2 = (pm == -INFINITY || mx == -INFINITY) ? 0.f : fast_exp2(pm - mx);
              ssc[j * G + h] = s2;
              ls += sml[2 * (j * G + h) + 1] * s2;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
            if (lane == 0) { stot[h] = mx; stot[G + h] = ls; }
          }
          __syncthreads();
          // (c) weighted sums of the held chunks, then any remaining batches
          if (part < SPLIT) {
#pragma unroll
            for (int u = 0; u < MAXB; ++u) {
              if (u < nb) {
                const float w4 = ssc[(part + u * SPLIT) * G + hch];
                s4.x = fmaf(v4[u].x, w4, s4.x); s4.y = fmaf(v4[u].y, w4, s4.y);
                s4.z = fmaf(v4[u].z, w4, s4.z); s4.w = fmaf(v4[u].w, w4, s4.w);
              }
            }
            for (int j = part + MAXB * SPLIT; j < nparts; j += SPLIT) {
              const float4 x4 = __ldcg(reinterpret_cast<const float4*>(
                  pacc + (long long)(pbase + j) * G * D) + ch);
              const float w4 = ssc[j * G + hch];
              s4.x = fmaf(x4.x, w4, s4.x); s4.y = fmaf(x4.y, w4, s4.y);
              s4.z = fmaf(x4.z, w4, s4.z); s4.w = fmaf(x4.w, w4, s4.w);
            }
            if (part > 0) scomb[(part - 1) * NCH + ch] = s4;
          }
          __syncthreads();
          if (part == 0) {
            for (int p2 = 1; p2 < SPLIT; ++p2) {
              const float4 o4 = scomb[(p2 - 1) * NCH + ch];
              s4.x += o4.x; s4.y += o4.y; s4.z += o4.z; s4.w += o4.w;
            }
            const int dd = (ch * 4) % D;
            const float mt = stot[hch], lt = stot[G + hch];
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            const long long orow = ((long long)b * hq + hglob0 + hch) * D + dd;
            outp[orow + 0] = (T)(s4.x * inv);
            outp[orow + 1] = (T)(s4.y * inv);
            outp[orow + 2] = (T)(s4.z * inv);
            outp[orow + 3] = (T)(s4.w * inv);
            if (dd == 0 && a.lse)
              a.lse[(long long)b * hq + hglob0 + hch] =
                  lt > 0.f ? (mt + fast_log2(lt)) * 0.69314718055994531f : -INFINITY;
          }
        }
        if (tid == 0) {
          a.tickets[sigma] = 0;
          if (aligned) a.dyn[sigma] = 0;
        }
      }
    } else if (aligned && tid == 0) {
      a.dyn[sigma] = 0;     // this CTA alone worked the segment
    }
    __syncthreads();

    // ------------------------------------------------------ next segment
    if (seg.s1 >= hi) break;
    {
      int sN = seg.s1;
      do {
        if (++seg.g == a.hkv) {
          seg.g = 0;
          ++seg.i;
          seg.nt = (rowstart[seg.i + 1] - rowstart[seg.i]) / a.hkv;
        }
        seg.s1 = sN + seg.nt;
      } while (seg.nt == 0 && seg.s1 < hi);
      if (seg.nt == 0) break;
    }
  }

  // Drain: never leave a bulk copy landing in shared memory after exit. A
  // copy whose wait already timed out is not waited for again.
  if (issued > waited) {
    for (int k = waited + (aborted ? 1 : 0); k < issued; ++k) {
      const int stage = k % NS;
      const uint32_t parity = (uint32_t)((k / NS) & 1);
      const bool ok = __all_sync(0xffffffffu,
          mbar_wait_bounded(smem_addr(&bars[warp * NS + stage]), parity, kWaitLimitNs));
      if (!ok) {
        if (lane == 0) record_error(a.err, ODA_ERR_TIMEOUT);
        break;
      }
    }
  }
  }  // has_work

  if constexpr (CL) {
    // Merge of the cluster's split KV (the pushes are in cluster_push).
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    constexpr int GD = G * D;
    const int cs = a.cluster;
    const int rank = (int)cl.block_rank();
    const int per = GD / cs;
    cluster_arrive();                            // release: the pushes above
    cluster_wait();                              // acquire: every rank's pushes
    const int b = rowb[0], g = ((int)blockIdx.x / cs) % a.hkv;
    const float2* ml = reinterpret_cast<const float2*>(rml);
    T* outp = reinterpret_cast<T*>(a.out);
    // cs consecutive lanes combine one owned element: lane r of the group
    // takes rank r's (m, l, acc), and xor shuffles within the group (cs
    // divides 32) give the maximum and the rescaled sums in a fixed order.
    // per * cs = G * D is a multiple of 32, so a warp is wholly in or out.
    for (int base = 0; base < per * cs; base += W * 32) {
      const int it = base + tid;
      if (it >= per * cs) break;
      const int ol = it / cs, r = it % cs;
      const int o = rank * per + ol;
      const int h = o / D, dd = o % D;
      const float2 v = ml[r * G + h];
      float mt = v.x;
      for (int x = 1; x < cs; x <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, x));
      const float sc2 = (v.x == -INFINITY) ? 0.f : fast_exp2(v.x - mt);
      float lt = v.y * sc2, at = racc[r * per + ol] * sc2;
      for (int x = 1; x < cs; x <<= 1) {
        lt += __shfl_xor_sync(0xffffffffu, lt, x);
        at += __shfl_xor_sync(0xffffffffu, at, x);
      }
      if (r == 0) {
        const long long orow = ((long long)b * hq + g * G + h) * D;
        outp[orow + dd] = (T)(lt > 0.f ? at / lt : 0.f);
        if (dd == 0 && a.lse)
          a.lse[(long long)b * hq + g * G + h] =
              lt > 0.f ? (mt + fast_log2(lt)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }
}

template <typename T, int D, int G>
struct Shape {
  // warps per CTA: 16 KB tiles (fp32, d = 128) get fewer warps to fit stages
  static constexpr int W = (sizeof(T) * D >= 512) ? 4 : ODA_ATTN_WARPS;
  static constexpr int NS = ODA_ATTN_STAGES;                  // stages per warp
  // smallest share of tiles a CTA takes, so a short launch uses fewer CTAs
  static constexpr int MIN_TILES_RING = W * ODA_RING_TILES_PER_WARP;
  static constexpr int MIN_TILES_FULL = W * ODA_FULL_TILES_PER_WARP;
};

// Cluster-merge Local launches whose CTAs hold at most ODA_CL_WIDE_WARPS tiles
// each (a full ring over a 16-CTA cluster) use one warp per tile and a single
// stage, so no warp works two tiles in turn.
#ifndef ODA_CL_WIDE_WARPS
#define ODA_CL_WIDE_WARPS 9
#endif
struct ShapeWide {
  static constexpr int W = ODA_CL_WIDE_WARPS;
  static constexpr int NS = 1;
};

template <typename T, int D, int G, int W, int NS>
size_t smem_bytes_wn(int max_batch) {
  constexpr size_t TILE_BYTES = 2 * ODA_TILE * D * sizeof(T);
  size_t s = (size_t)W * NS * TILE_BYTES;
  s += (size_t)W * G * (D + 2) * 4 + 4;
  s += (size_t)W * NS * 8;
  s += (size_t)W * 32 * G * 4;
  s += (size_t)(4 * max_batch + 2) * 4;
  s += 16 + 64;
  s += (size_t)W * NS * 4;
  s += (size_t)W * NS;
  s += 16 + (size_t)(G * D + 32 * G) * 4;     // cluster mode: pushed accumulators, (m, l)
  s += (size_t)G * D * sizeof(T) + 16;          // the segment's queries, t
  s += (size_t)max_batch * 4;                   // first position read per row (paged)
  s += (size_t)W * 4 * 4;                       // pool grabs ahead, per warp
  return (s + 127) & ~(size_t)127;
}

template <typename T, int D, int G, bool RING>
size_t smem_bytes(int max_batch) {
  return smem_bytes_wn<T, D, G, Shape<T, D, G>::W, Shape<T, D, G>::NS>(max_batch);
}

template <typename T, int D, int G, bool RING, bool CL = false>
auto kernel_ptr() {
  return attn_kernel<T, D, G, Shape<T, D, G>::W, Shape<T, D, G>::NS, RING, CL>;
}

// Cluster-merge Local kernel of shape (W, NS): sets its attributes and returns
// the largest cluster size (16, 8, 4, 2) of which the GPU holds at least one
// cluster, capped by ODA_LOCAL_CLUSTER; 0 if none. `ctas` receives the CTAs
// one wave holds.
template <typename T, int D, int G, int W, int NS>
int cluster_setup(oda_ctx* ctx, int& ctas) {
  auto kc = attn_kernel<T, D, G, W, NS, true, true>;
  const size_t sm = smem_bytes_wn<T, D, G, W, NS>(ctx->cfg.max_batch);
  ctas = 0;
  int occ = 0;
  if (raise_smem_limit(reinterpret_cast<const void*>(kc), sm) != cudaSuccess ||
      cudaFuncSetAttribute(kc, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess ||
      occupancy_cached(&occ, reinterpret_cast<const void*>(kc), W * 32, sm) != cudaSuccess ||
      occ < 1) {
    cudaGetLastError();
    return 0;
  }
  ctas = ctx->num_sms * occ;
  // ODA_LOCAL_CLUSTER caps the cluster size (0 or 1: always the global merge)
  int cap = 16;
  if (const char* e = getenv("ODA_LOCAL_CLUSTER")) cap = atoi(e);
  for (int cs = 16; cs >= 2; cs >>= 1) {
    if (cs > cap) continue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs);
    cfg.blockDim = dim3(W * 32);
    cfg.dynamicSmemBytes = sm;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int ncl = 0;
    if (cudaOccupancyMaxActiveClusters(&ncl, kc, &cfg) == cudaSuccess && ncl > 0) return cs;
    cudaGetLastError();
  }
  return 0;
}

template <typename T, int D, int G, bool RING>
oda_status setup_one(oda_ctx* ctx, int& ctas) {
  auto k = kernel_ptr<T, D, G, RING>();
  const size_t sm = smem_bytes<T, D, G, RING>(ctx->cfg.max_batch);
  ODA_CUDA_TRY(raise_smem_limit(reinterpret_cast<const void*>(k), sm));
  int occ = 0;
  ODA_CUDA_TRY(occupancy_cached(&occ, reinterpret_cast<const void*>(k), Shape<T, D, G>::W * 32, sm));
  if (occ < 1) return ODA_ERR_SHAPE;
  ctas = ctx->num_sms * occ;
  if (RING) {
    int c0 = 0, c1 = 0;
    ctx->local_cluster_max =
        cluster_setup<T, D, G, Shape<T, D, G>::W, Shape<T, D, G>::NS>(ctx, c0);
    ctx->local_wide_cluster_max = cluster_setup<T, D, G, ShapeWide::W, ShapeWide::NS>(ctx, c1);
    ctx->local_wide_ctas = c1;
  }
  return ODA_OK;
}

template <typename T, int D, int G, int W, int NS>
oda_status launch_cluster(oda_ctx* ctx, const AttnArgs& a, int grid, int cs, cudaStream_t st) {
  auto k = attn_kernel<T, D, G, W, NS, true, true>;
  const size_t sm = smem_bytes_wn<T, D, G, W, NS>(ctx->cfg.max_batch);
  ctx->local_last_smem = sm;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(W * 32);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k, a) == cudaSuccess ? ODA_OK : ODA_ERR_CUDA;
}

template <typename T, int D, int G, bool RING>
oda_status launch_one(oda_ctx* ctx, const AttnArgs& a, int ctas, cudaStream_t st) {
  auto k = kernel_ptr<T, D, G, RING>();
  const size_t sm = smem_bytes<T, D, G, RING>(ctx->cfg.max_batch);
  if (RING) ctx->local_last_smem = sm;
  return launch_pdl(k, dim3(ctas), dim3(Shape<T, D, G>::W * 32), sm, st, a) == cudaSuccess
             ? ODA_OK
             : ODA_ERR_CUDA;
}

template <bool RING, typename F>
oda_status dispatch(const oda_config& c, F&& f) {
  const int G = c.hq / c.hkv;
#define ODA_CASE(TT, DD, GG)                                                     \
  if (c.head_dim == DD && G == GG) return f.template operator()<TT, DD, GG, RING>();
#ifdef ODA_ATTN_HOT_ONLY  // measurement builds: only the bf16, d = 128, G = 2 kernels
  if (c.dtype == ODA_BF16) {
    ODA_CASE(__nv_bfloat16, 128, 2)
  }
#else
  if (c.dtype == ODA_BF16) {
    ODA_CASE(__nv_bfloat16, 128, 2) ODA_CASE(__nv_bfloat16, 128, 1) ODA_CASE(__nv_bfloat16, 128, 4)
    ODA_CASE(__nv_bfloat16, 64, 2) ODA_CASE(__nv_bfloat16, 64, 1) ODA_CASE(__nv_bfloat16, 64, 4)
  } else {
    ODA_CASE(float, 128, 2) ODA_CASE(float, 128, 1) ODA_CASE(float, 128, 4)
    ODA_CASE(float, 64, 2) ODA_CASE(float, 64, 1) ODA_CASE(float, 64, 4)
  }
#endif
#undef ODA_CASE
  return ODA_ERR_SHAPE;
}

struct SetupRing {
  oda_ctx* ctx;
  int* out;
  template <typename T, int D, int G, bool RING>
  oda_status operator()() {
    return setup_one<T, D, G, RING>(ctx, *out);
  }
};

struct Launch {
  oda_ctx* ctx;
  const AttnArgs* a;
  cudaStream_t st;
  bool ring;
  template <typename T, int D, int G, bool RING>
  oda_status operator()() {
    AttnArgs b = *a;
    b.min_tiles_per_cta = RING ? Shape<T, D, G>::MIN_TILES_RING : Shape<T, D, G>::MIN_TILES_FULL;
    if (RING) {
      // few segments: one cluster of cs CTAs per (row, KV head) segment,
      // merged through distributed shared memory instead of global partials
      const int S = b.B * b.hkv;
      int cs = ctx->local_cluster_max;
      while (cs >= 2 && S * cs > ctx->attn_ctas_local) cs >>= 1;
      if (cs >= 2) {
        b.cluster = cs;
        // one tile per warp even for a full ring: the wide shape
        if (cs <= ctx->local_wide_cluster_max && S * cs <= ctx->local_wide_ctas &&
            (b.ring_blocks + cs - 1) / cs <= ShapeWide::W)
          return launch_cluster<T, D, G, ShapeWide::W, ShapeWide::NS>(ctx, b, S * cs, cs, st);
        return launch_cluster<T, D, G, Shape<T, D, G>::W, Shape<T, D, G>::NS>(ctx, b, S * cs, cs,
                                                                             st);
      }
    }
    return launch_one<T, D, G, RING>(ctx, b, RING ? ctx->attn_ctas_local : ctx->attn_ctas_full,
                                     st);
  }
};

}  // namespace

namespace oda_impl {

oda_status attn_setup(oda_ctx* ctx) {
  int ring_ctas = 0, full_ctas = 0;
  oda_status s = dispatch<true>(ctx->cfg, SetupRing{ctx, &ring_ctas});
  if (s != ODA_OK) return s;
  s = dispatch<false>(ctx->cfg, SetupRing{ctx, &full_ctas});
  if (s != ODA_OK) return s;
  ctx->attn_ctas_local = ring_ctas;
  ctx->attn_ctas_full = full_ctas;
  return ODA_OK;
}

oda_status launch_attn(oda_ctx* ctx, bool ring_mode, int layer, const void* q,
                       const int32_t* seq_lens, const void* kv, const int32_t* block_table,
                       const int32_t* idx, const int32_t* count, void* out, float* lse, int B,
                       cudaStream_t st, const int* plan, bool early, const int32_t* range_lo,
                       const int32_t* range_hi) {
  const oda_config& c = ctx->cfg;
  AttnArgs a;
  a.q = q;
  a.out = out;
  a.lse = lse;
  a.seq_lens = seq_lens;
  const size_t eb = (size_t)ctx->lay.elem_bytes;
  const int64_t lstride = ring_mode ? ctx->lay.ring_layer_elems : ctx->lay.cache_layer_elems;
  a.kv = static_cast<const unsigned char*>(kv) + (size_t)layer * (size_t)lstride * eb;
  a.block_table = block_table;
  a.idx = idx;
  a.count = count;
  a.num_blocks = c.num_blocks;
  a.max_blocks = c.max_blocks_per_seq;
  a.B = B;
  a.hkv = c.hkv;
  a.sink = c.sink;
  a.window = c.window;
  a.ring_blocks = (int)ctx->lay.ring_blocks;
  a.max_batch = c.max_batch;
  a.qscale = 1.4426950408889634f / sqrtf((float)c.head_dim);
  a.partials = ctx->partials;
  a.max_parts = ctx->max_parts;
  a.tickets = ctx->tickets;
  a.dyn = ctx->tickets + (size_t)c.max_batch * c.hkv;
  a.plan = plan;
  a.cluster = 0;
  a.early = early ? 1 : 0;
  a.range_lo = ring_mode ? nullptr : range_lo;
  a.range_hi = ring_mode ? nullptr : range_hi;
  a.err = ctx->err;
  if (ring_mode) return dispatch<true>(c, Launch{ctx, &a, st, true});
  return dispatch<false>(c, Launch{ctx, &a, st, false});
}

struct MinTiles {
  int* out;
  template <typename T, int D, int G, bool RING>
  oda_status operator()() {
    *out = RING ? Shape<T, D, G>::MIN_TILES_RING : Shape<T, D, G>::MIN_TILES_FULL;
    return ODA_OK;
  }
};

int attn_min_tiles(oda_ctx* ctx, bool ring_mode) {
  int v = 1;
  if (ring_mode) dispatch<true>(ctx->cfg, MinTiles{&v});
  else dispatch<false>(ctx->cfg, MinTiles{&v});
  return v;
}

}  // namespace oda_impl

// ---------------------------------------------------------------------------
// Full attention without any device allocation.
//
// Some callers cannot call cudaMalloc: inference engines that hand the whole
// GPU to their own pool allocator at start-up (a later cudaMalloc fails once
// the pool holds the memory, or silently breaks the engine's accounting), and
// host code on a latency-critical decode loop where a cudaMalloc would
// synchronize the device. oda_full_attn_gated_static serves them: it needs no
// context, and the split partials, segment tickets and fallback error word
// live in the file-scope __device__ arrays below, which every GPU that loads
// liboda holds until the process exits.
//
// In host code these names are host-side stand-ins, not device addresses;
// the device address of each is fetched once per device with
// cudaGetSymbolAddress (with that device current) on the first call there.
// ---------------------------------------------------------------------------

namespace {

constexpr int kStaticPartialFloats = 1 << 18;  // 1 MiB of split partials
constexpr int kStaticMaxSegments = 512;        // rows x KV heads per call
constexpr int kStaticMaxCtas = 512;            // persistent grid cap
constexpr int kStaticMaxDevices = 64;

static __device__ __align__(256) float g_static_partials[kStaticPartialFloats];
static __device__ __align__(256) int g_static_tickets[2 * kStaticMaxSegments];
static __device__ __align__(256) int g_static_err[1];

struct StaticDevice {
  bool ready;
  float* partials;
  int* tickets;
  int* err;
  int num_sms;
};
StaticDevice g_static_dev[kStaticMaxDevices];
std::mutex g_static_mu;

// Once per device, with that device current: resolve the device addresses.
oda_status static_setup(int dev, StaticDevice** out) {
  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticDevice& s = g_static_dev[dev];
  if (!s.ready) {
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&s.partials), g_static_partials) !=
            cudaSuccess ||
        cudaGetSymbolAddress(reinterpret_cast<void**>(&s.tickets), g_static_tickets) !=
            cudaSuccess ||
        cudaGetSymbolAddress(reinterpret_cast<void**>(&s.err), g_static_err) != cudaSuccess ||
        cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ODA_ERR_CUDA;
    s.ready = true;
  }
  *out = &s;
  return ODA_OK;
}

struct LaunchStatic {
  const AttnArgs* a;
  int num_sms;
  int max_batch;
  int B;
  cudaStream_t st;
  template <typename T, int D, int G, bool RING>
  oda_status operator()() {
    auto k = kernel_ptr<T, D, G, RING>();
    const size_t sm = smem_bytes<T, D, G, RING>(max_batch);
    // the limit only ever rises (a context sized for more rows keeps working),
    // and the occupancy is asked of the runtime once per size
    if (raise_smem_limit(reinterpret_cast<const void*>(k), sm) != cudaSuccess)
      return ODA_ERR_CUDA;
    int occ = 0;
    if (occupancy_cached(&occ, reinterpret_cast<const void*>(k), Shape<T, D, G>::W * 32, sm) !=
            cudaSuccess ||
        occ < 1)
      return ODA_ERR_CUDA;
    int ctas = num_sms * occ;
    if (ctas > kStaticMaxCtas) ctas = kStaticMaxCtas;
    // every partial index (CTA + segment) must fit the static array
    const long long need = (long long)(ctas + B * a->hkv) * G * (D + 2);
    if (need > kStaticPartialFloats) return ODA_ERR_SHAPE;
    AttnArgs b = *a;
    b.max_parts = kStaticPartialFloats / (G * (D + 2));
    b.min_tiles_per_cta = Shape<T, D, G>::MIN_TILES_FULL;
    b.max_batch = max_batch;
    return launch_pdl(k, dim3(ctas), dim3(Shape<T, D, G>::W * 32), sm, st, b) == cudaSuccess
               ? ODA_OK
               : ODA_ERR_CUDA;
  }
};

}  // namespace

extern "C" oda_status oda_full_attn_gated_static(const oda_config* cfg, int layer, const void* q,
                                                 const int32_t* seq_lens,
                                                 const int32_t* block_table, const void* kv_cache,
                                                 const int32_t* idx, const int32_t* count,
                                                 void* out, float* lse, int B, int32_t* err,
                                                 oda_stream stream) {
  oda_layout_info lay;
  const oda_status ls = oda_layout(cfg, &lay);
  if (ls != ODA_OK) return ls;
  if (layer < 0 || layer >= cfg->layers || B < 0) return ODA_ERR_ARG;
  if (B > cfg->max_batch) return ODA_ERR_SHAPE;
  if (B == 0) return ODA_OK;
  if (!q || !seq_lens || !block_table || !kv_cache || !idx || !count || !out) return ODA_ERR_ARG;
  if ((long long)B * cfg->hkv > kStaticMaxSegments) return ODA_ERR_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ODA_ERR_CUDA;
  if (dev < 0 || dev >= kStaticMaxDevices) return ODA_ERR_SHAPE;
  StaticDevice* sd = nullptr;
  oda_status s = static_setup(dev, &sd);
  if (s != ODA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // tickets and the dynamic tile counters must start at zero; a call that
  // gave up early may have left some set
  if (cudaMemsetAsync(sd->tickets, 0, sizeof(int) * 2 * (size_t)kStaticMaxSegments, st) !=
      cudaSuccess)
    return ODA_ERR_CUDA;
  AttnArgs a;
  a.q = q;
  a.out = out;
  a.lse = lse;
  a.seq_lens = seq_lens;
  a.kv = static_cast<const unsigned char*>(kv_cache) +
         (size_t)layer * (size_t)lay.cache_layer_elems * (size_t)lay.elem_bytes;
  a.block_table = block_table;
  a.idx = idx;
  a.count = count;
  a.num_blocks = cfg->num_blocks;
  a.max_blocks = cfg->max_blocks_per_seq;
  a.B = B;
  a.hkv = cfg->hkv;
  a.sink = cfg->sink;
  a.window = cfg->window;
  a.ring_blocks = (int)lay.ring_blocks;
  a.max_batch = cfg->max_batch;
  a.qscale = 1.4426950408889634f / sqrtf((float)cfg->head_dim);
  a.partials = sd->partials;
  a.tickets = sd->tickets;
  a.dyn = sd->tickets + kStaticMaxSegments;
  a.plan = nullptr;
  a.cluster = 0;
  a.early = 0;
  a.range_lo = nullptr;
  a.range_hi = nullptr;
  a.err = err ? err : sd->err;
  return dispatch<false>(*cfg, LaunchStatic{&a, sd->num_sms, cfg->max_batch, B, st});
}
