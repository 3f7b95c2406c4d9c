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
//     The total is split evenly over a persistent grid sized to the SMs, so a
//     batch-1 128K request and a 32-request mixed batch both fill the GPU.
//   * Each warp streams its own tiles through NS shared-memory stages with
//     cp.async.bulk (TMA bulk copies) completing on mbarriers; waits are
//     bounded and a timeout is recorded, never trapped.
//   * q.k: every lane owns d/32 dimensions; the 16*G partial dot products of
//     a tile are reduced across the warp with a transposing butterfly, leaving
//     one score per lane. Online softmax in base 2 (q pre-scaled by
//     log2(e)/sqrt(d)), fp32 accumulation on the CUDA cores: with G = 2 query
//     heads per KV head the contraction is too thin for tensor cores.
//   * Warps of a CTA merge their states in shared memory; CTAs sharing a
//     segment write (m, l, acc) partials and the last one to take the
//     segment's ticket merges them and writes the output.
#include <mutex>

#include "oda_internal.cuh"

using namespace oda;

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
  float* partials;
  int* tickets;
  int* err;
};

template <typename T>
struct Vec;

// Loads of DPL consecutive elements of one row, widened to float.
template <>
struct Vec<__nv_bfloat16> {
  template <int DPL>
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[DPL]) {
    static_assert(DPL == 2 || DPL == 4, "bf16 lanes own 2 or 4 dims");
    if constexpr (DPL == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(p);
      bf16x2_to_f32(w.x, x[0], x[1]);
      bf16x2_to_f32(w.y, x[2], x[3]);
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
      bf16x2_to_f32(w, x[0], x[1]);
    }
  }
  template <int DPL>
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&x)[DPL]) {
    for (int i = 0; i < DPL; ++i) p[i] = __float2bfloat16_rn(x[i]);
  }
};

template <>
struct Vec<float> {
  template <int DPL>
  static __device__ __forceinline__ void load(const float* p, float (&x)[DPL]) {
    static_assert(DPL == 2 || DPL == 4, "f32 lanes own 2 or 4 dims");
    if constexpr (DPL == 4) {
      const float4 w = *reinterpret_cast<const float4*>(p);
      x[0] = w.x; x[1] = w.y; x[2] = w.z; x[3] = w.w;
    } else {
      const float2 w = *reinterpret_cast<const float2*>(p);
      x[0] = w.x; x[1] = w.y;
    }
  }
  template <int DPL>
  static __device__ __forceinline__ void store(float* p, const float (&x)[DPL]) {
    for (int i = 0; i < DPL; ++i) p[i] = x[i];
  }
};

// Bits [lo, hi) of a 16-bit tile mask whose bit 0 is slot `base`.
__device__ __forceinline__ uint32_t range_bits(int lo, int hi, int base) {
  int l = min(max(lo - base, 0), 16);
  int h = min(max(hi - base, 0), 16);
  if (h <= l) return 0u;
  return ((1u << h) - 1u) & ~((1u << l) - 1u);
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

template <typename T, int D, int G, int W, int NS, bool RING>
__global__ void __launch_bounds__(W * 32)
attn_kernel(const AttnArgs a) {
  constexpr int TILE_ELEMS = 2 * ODA_TILE * D;
  constexpr int TILE_BYTES = TILE_ELEMS * (int)sizeof(T);
  constexpr int DPL = D / 32;
  constexpr int NV16 = 16 * G;                 // partial dot products per lane per tile
  constexpr int NV = NV16 >= 32 ? NV16 / 32 : 1;   // scores per lane after the butterfly
  constexpr int DUP = NV16 >= 32 ? 1 : 32 / NV16;  // lanes holding the same score
  constexpr int LPH = 16 * DUP / NV;           // lanes per query head after the butterfly

  extern __shared__ __align__(128) unsigned char smem[];
  T* tiles = reinterpret_cast<T*>(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)W * NS * TILE_BYTES);
  float* pbuf = reinterpret_cast<float*>(bars + W * NS);          // [W][NV16]
  float* wstate = pbuf + W * NV16;                                 // [W][G][D+2]
  int* rowstart = reinterpret_cast<int*>(wstate + W * G * (D + 2));  // [max_batch+1]
  int* rowb = rowstart + (a.max_batch + 1);
  int* rowt = rowb + a.max_batch;
  int* sflag = rowt + a.max_batch;
  unsigned char* badst = reinterpret_cast<unsigned char*>(sflag + 4);  // [W][NS]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int hq = a.hkv * G;

  // ---------------------------------------------------------------- rows
  int nrows;
  if (RING) {
    nrows = a.B;
  } else {
    nrows = *reinterpret_cast<const volatile int32_t*>(a.count);
    if (nrows < 0 || nrows > a.B) {
      if (tid == 0 && blockIdx.x == 0) record_error(a.err, ODA_ERR_BOUNDS);
      nrows = nrows < 0 ? 0 : a.B;
    }
  }
  if (nrows == 0) return;
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < nrows; base += 32) {
      const int i = base + lane;
      int nt = 0;
      if (i < nrows) {
        const int b = RING ? i : a.idx[i];
        const bool okb = b >= 0 && b < a.B;
        const int t = okb ? a.seq_lens[b] : 0;
        if (!okb || t < 1) {
          if (blockIdx.x == 0) record_error(a.err, ODA_ERR_BOUNDS);
        } else if (RING) {
          nt = (a.sink + min(t, a.window) + ODA_TILE - 1) / ODA_TILE;
        } else {
          nt = (t + ODA_TILE - 1) / ODA_TILE;
          if (nt > a.max_blocks) {
            if (blockIdx.x == 0) record_error(a.err, ODA_ERR_BOUNDS);
            nt = 0;
          }
        }
        rowb[i] = okb ? b : 0;
        rowt[i] = t;
      }
      int v = nt * a.hkv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
      }
      if (i < nrows) rowstart[i + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) rowstart[0] = 0;
  }
  __syncthreads();
  const int total = rowstart[nrows];
  if (total == 0) return;
  int P = (int)gridDim.x;
  {
    const int want = max(1, (total + a.min_tiles_per_cta - 1) / a.min_tiles_per_cta);
    P = min(P, want);
  }
  const int cta = (int)blockIdx.x;
  if (cta >= P) return;
  const int lo = (int)(((long long)cta * total) / P);
  const int hi = (int)(((long long)(cta + 1) * total) / P);
  if (lo >= hi) return;

  if (tid < W * NS) mbar_init(smem_addr(&bars[tid]), 1);
  fence_mbar_init();
  __syncthreads();

  const uint64_t policy = RING ? l2_policy_evict_last() : l2_policy_evict_first();
  const T* kvbase = reinterpret_cast<const T*>(a.kv);

  // -------------------------------------------------------- tile producer
  Cursor prod;
  prod.k = lo;
  locate(rowstart, nrows, a.hkv, lo, prod);
  prod.k = lo + warp;
  normalize(rowstart, a.hkv, hi, warp, prod);
  Cursor cons = prod;

  auto issue = [&](const Cursor& c, int stage) {
    if (lane == 0) {
      const uint32_t bar = smem_addr(&bars[warp * NS + stage]);
      const uint32_t dst = smem_addr(tiles + (size_t)(warp * NS + stage) * TILE_ELEMS);
      const int b = rowb[c.i];
      const int jt = c.k - (c.s1 - c.nt);
      const T* src;
      bool bad = false;
      if (RING) {
        src = kvbase + (((long long)b * a.hkv + c.g) * a.ring_blocks + jt) * TILE_ELEMS;
      } else {
        const int blk = a.block_table[(long long)b * a.max_blocks + jt];
        bad = blk < 0 || (long long)blk >= a.num_blocks;
        src = kvbase + ((long long)blk * a.hkv + c.g) * TILE_ELEMS;
      }
      badst[warp * NS + stage] = bad ? 1 : 0;
      if (bad) {
        record_error(a.err, ODA_ERR_BOUNDS);
        mbar_arrive(bar);
      } else {
        mbar_arrive_expect_tx(bar, TILE_BYTES);
        bulk_g2s(dst, src, TILE_BYTES, bar, policy);
      }
    }
  };

  int issued = 0;
#pragma unroll 1
  for (int s = 0; s < NS; ++s) {
    if (prod.k >= hi) break;
    issue(prod, s);
    ++issued;
    prod.k += W;
    normalize(rowstart, a.hkv, hi, warp, prod);
  }
  int consumed = 0;
  int waited = 0;        // tiles whose copy is known to have landed
  bool aborted = false;

  // ------------------------------------------------------- segment loop
  Cursor seg;
  seg.k = lo;
  locate(rowstart, nrows, a.hkv, lo, seg);
  while (true) {
    const int b = rowb[seg.i];
    const int t = rowt[seg.i];
    const int s0 = seg.s1 - seg.nt;

    float qv[G][DPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const T* qp = reinterpret_cast<const T*>(a.q) +
                    ((long long)b * hq + seg.g * G + h) * D + lane * DPL;
      float x[DPL];
      Vec<T>::template load<DPL>(qp, x);
#pragma unroll
      for (int e = 0; e < DPL; ++e) qv[h][e] = x[e] * a.qscale;
    }
    float m_run[G], l_run[G], acc[G][DPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_run[h] = -INFINITY;
      l_run[h] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
    }

    // ring validity constants of this row
    const int mw = min(t, a.window);
    const int nsv = min(max(t - a.window, 0), a.sink);

#pragma unroll 1
    while (cons.k < hi && cons.i == seg.i && cons.g == seg.g) {
      const int stage = consumed % NS;
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
      const int jt = cons.k - s0;
      uint32_t mask;
      if (RING) {
        const int base = jt * ODA_TILE;
        mask = range_bits(a.sink, a.sink + mw, base) | range_bits(0, nsv, base);
      } else {
        const int nvalid = min(ODA_TILE, t - jt * ODA_TILE);
        mask = nvalid >= 16 ? 0xFFFFu : ((1u << nvalid) - 1u);
      }
      if (badst[warp * NS + stage] || aborted) mask = 0;

      if (mask) {
        const T* tk = tiles + (size_t)(warp * NS + stage) * TILE_ELEMS;
        const T* tv = tk + ODA_TILE * D;
        // ---- q.k partial sums: x[h*16 + j]
        float x[NV16];
#pragma unroll
        for (int j = 0; j < ODA_TILE; ++j) {
          float kf[DPL];
          Vec<T>::template load<DPL>(tk + j * D + lane * DPL, kf);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) s = fmaf(qv[h][e], kf[e], s);
            x[h * 16 + j] = s;
          }
        }
        // ---- transposing butterfly: lane ends with full sums of its slots
        {
          int c = NV16;
#pragma unroll
          for (int r = 0; r < 5; ++r) {
            const int off = 16 >> r;
            if (c > 1) {
              const bool upper = (lane & off) != 0;
              const int half = c >> 1;
#pragma unroll
              for (int i2 = 0; i2 < NV16 / 2; ++i2) {
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
        // slot index of x[e] on this lane
        float sc[NV];
        int myh;
#pragma unroll
        for (int e = 0; e < NV; ++e) {
          const int v = NV16 >= 32 ? lane * NV + e : lane / DUP;
          const int j = v & 15;
          myh = v >> 4;
          sc[e] = ((mask >> j) & 1u) ? x[e] : -INFINITY;
        }
        // ---- per-head tile max
        float mx = sc[0];
#pragma unroll
        for (int e = 1; e < NV; ++e) mx = fmaxf(mx, sc[e]);
#pragma unroll
        for (int o = DUP; o < LPH; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float m_new[G], alpha[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float th = __shfl_sync(0xffffffffu, mx, h * LPH);
          m_new[h] = fmaxf(m_run[h], th);
          alpha[h] = (m_run[h] == -INFINITY) ? 0.f : fast_exp2(m_run[h] - m_new[h]);
        }
        float mine = m_new[0];
#pragma unroll
        for (int h = 1; h < G; ++h) if (myh == h) mine = m_new[h];
        float p[NV];
        float ps = 0.f;
#pragma unroll
        for (int e = 0; e < NV; ++e) {
          p[e] = (sc[e] == -INFINITY) ? 0.f : fast_exp2(sc[e] - mine);
          ps += p[e];
        }
#pragma unroll
        for (int o = DUP; o < LPH; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float tsum = __shfl_sync(0xffffffffu, ps, h * LPH);
          l_run[h] = l_run[h] * alpha[h] + tsum;
          m_run[h] = m_new[h];
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[h][e] *= alpha[h];
        }
        // ---- probabilities to shared memory, then P.V
        float* pw = pbuf + warp * NV16;
#pragma unroll
        for (int e = 0; e < NV; ++e) {
          const int v = NV16 >= 32 ? lane * NV + e : lane / DUP;
          if (NV16 >= 32 || (lane % DUP) == 0) pw[v] = p[e];
        }
        __syncwarp();
        if (mask == 0xFFFFu) {
#pragma unroll
          for (int j4 = 0; j4 < ODA_TILE; j4 += 4) {
            float4 pj[G];
#pragma unroll
            for (int h = 0; h < G; ++h) pj[h] = *reinterpret_cast<const float4*>(pw + h * 16 + j4);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              float vf[DPL];
              Vec<T>::template load<DPL>(tv + (j4 + jj) * D + lane * DPL, vf);
#pragma unroll
              for (int h = 0; h < G; ++h) {
                const float pp = jj == 0 ? pj[h].x : jj == 1 ? pj[h].y : jj == 2 ? pj[h].z : pj[h].w;
#pragma unroll
                for (int e = 0; e < DPL; ++e) acc[h][e] = fmaf(pp, vf[e], acc[h][e]);
              }
            }
          }
        } else {
#pragma unroll 1
          for (int j = 0; j < ODA_TILE; ++j) {
            if (!((mask >> j) & 1u)) continue;   // masked slots may hold garbage
            float vf[DPL];
            Vec<T>::template load<DPL>(tv + j * D + lane * DPL, vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float pp = pw[h * 16 + j];
#pragma unroll
              for (int e = 0; e < DPL; ++e) acc[h][e] = fmaf(pp, vf[e], acc[h][e]);
            }
          }
        }
      }
      __syncwarp();
      // refill the stage just consumed
      if (prod.k < hi && !aborted) {
        issue(prod, stage);
        ++issued;
        prod.k += W;
        normalize(rowstart, a.hkv, hi, warp, prod);
      }
      ++consumed;
      cons.k += W;
      normalize(rowstart, a.hkv, hi, warp, cons);
    }

    // ---------------------------------------------- merge warps of the CTA
    float* ws = wstate + (size_t)warp * G * (D + 2);
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int e = 0; e < DPL; ++e) ws[h * (D + 2) + lane * DPL + e] = acc[h][e];
      if (lane == 0) {
        ws[h * (D + 2) + D] = m_run[h];
        ws[h * (D + 2) + D + 1] = l_run[h];
      }
    }
    __syncthreads();

    const int sigma = seg.i * a.hkv + seg.g;
    const long long Pll = P;
    const int c_first = (int)(((long long)(s0 + 1) * Pll - 1) / total);
    const int c_last = (int)(((long long)seg.s1 * Pll - 1) / total);
    const int nparts = c_last - c_first + 1;
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
        float* pp = a.partials + ((long long)(cta + sigma) * G + h) * (D + 2);
        pp[dd] = at;
        if (dd == 0) { pp[D] = mt; pp[D + 1] = lt; }
      }
    }
    if (nparts > 1) {
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        const int prev = atomicAdd(&a.tickets[sigma], 1);
        sflag[0] = (prev == nparts - 1) ? 1 : 0;
      }
      __syncthreads();
      if (sflag[0]) {
        __threadfence();
        for (int o = tid; o < G * D; o += W * 32) {
          const int h = o / D, dd = o % D;
          float mt = -INFINITY;
          for (int c2 = c_first; c2 <= c_last; ++c2)
            mt = fmaxf(mt, __ldcg(a.partials + ((long long)(c2 + sigma) * G + h) * (D + 2) + D));
          float lt = 0.f, at = 0.f;
          if (mt != -INFINITY) {
            for (int c2 = c_first; c2 <= c_last; ++c2) {
              const float* pp = a.partials + ((long long)(c2 + sigma) * G + h) * (D + 2);
              const float pm = __ldcg(pp + D);
              if (pm == -INFINITY) continue;
              const float sc2 = fast_exp2(pm - mt);
              lt += __ldcg(pp + D + 1) * sc2;
              at += __ldcg(pp + dd) * sc2;
            }
          }
          const long long orow = ((long long)b * hq + hglob0 + h) * D;
          outp[orow + dd] = (T)(lt > 0.f ? at / lt : 0.f);
          if (dd == 0 && a.lse)
            a.lse[(long long)b * hq + hglob0 + h] =
                lt > 0.f ? (mt + fast_log2(lt)) * 0.69314718055994531f : -INFINITY;
        }
        if (tid == 0) a.tickets[sigma] = 0;
      }
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
}

template <typename T, int D, int G>
struct Shape {
  static constexpr int W = (sizeof(T) * D >= 512) ? 4 : 6;   // warps per CTA
  static constexpr int NS = 2;                                // stages per warp
};

template <typename T, int D, int G, bool RING>
size_t smem_bytes(int max_batch) {
  constexpr int W = Shape<T, D, G>::W, NS = Shape<T, D, G>::NS;
  constexpr size_t TILE_BYTES = 2 * ODA_TILE * D * sizeof(T);
  size_t s = (size_t)W * NS * TILE_BYTES;
  s += (size_t)W * NS * 8;
  s += (size_t)W * 16 * G * 4;
  s += (size_t)W * G * (D + 2) * 4;
  s += (size_t)(3 * max_batch + 1) * 4;
  s += 16;
  s += (size_t)W * NS;
  return (s + 127) & ~(size_t)127;
}

template <typename T, int D, int G, bool RING>
auto kernel_ptr() {
  return attn_kernel<T, D, G, Shape<T, D, G>::W, Shape<T, D, G>::NS, RING>;
}

template <typename T, int D, int G, bool RING>
oda_status setup_one(oda_ctx* ctx, int& ctas) {
  auto k = kernel_ptr<T, D, G, RING>();
  const size_t sm = smem_bytes<T, D, G, RING>(ctx->cfg.max_batch);
  ODA_CUDA_TRY(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
  int occ = 0;
  ODA_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, Shape<T, D, G>::W * 32, sm));
  if (occ < 1) return ODA_ERR_SHAPE;
  ctas = ctx->num_sms * occ;
  return ODA_OK;
}

template <typename T, int D, int G, bool RING>
oda_status launch_one(oda_ctx* ctx, const AttnArgs& a, int ctas, cudaStream_t st) {
  auto k = kernel_ptr<T, D, G, RING>();
  const size_t sm = smem_bytes<T, D, G, RING>(ctx->cfg.max_batch);
  k<<<ctas, Shape<T, D, G>::W * 32, sm, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? ODA_OK : ODA_ERR_CUDA;
}

template <bool RING, typename F>
oda_status dispatch(const oda_config& c, F&& f) {
  const int G = c.hq / c.hkv;
#define ODA_CASE(TT, DD, GG)                                                     \
  if (c.head_dim == DD && G == GG) return f.template operator()<TT, DD, GG, RING>();
  if (c.dtype == ODA_BF16) {
    ODA_CASE(__nv_bfloat16, 128, 2) ODA_CASE(__nv_bfloat16, 128, 1) ODA_CASE(__nv_bfloat16, 128, 4)
    ODA_CASE(__nv_bfloat16, 64, 2) ODA_CASE(__nv_bfloat16, 64, 1) ODA_CASE(__nv_bfloat16, 64, 4)
  } else {
    ODA_CASE(float, 128, 2) ODA_CASE(float, 128, 1) ODA_CASE(float, 128, 4)
    ODA_CASE(float, 64, 2) ODA_CASE(float, 64, 1) ODA_CASE(float, 64, 4)
  }
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
    b.min_tiles_per_cta = Shape<T, D, G>::W;
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
                       cudaStream_t st) {
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
  a.tickets = ctx->tickets;
  a.err = ctx->err;
  if (ring_mode) return dispatch<true>(c, Launch{ctx, &a, st, true});
  return dispatch<false>(c, Launch{ctx, &a, st, false});
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
static __device__ __align__(256) int g_static_tickets[kStaticMaxSegments];
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
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
        cudaSuccess)
      return ODA_ERR_CUDA;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, Shape<T, D, G>::W * 32, sm) !=
            cudaSuccess ||
        occ < 1)
      return ODA_ERR_CUDA;
    int ctas = num_sms * occ;
    if (ctas > kStaticMaxCtas) ctas = kStaticMaxCtas;
    // every partial index (CTA + segment) must fit the static array
    const long long need = (long long)(ctas + B * a->hkv) * G * (D + 2);
    if (need > kStaticPartialFloats) return ODA_ERR_SHAPE;
    AttnArgs b = *a;
    b.min_tiles_per_cta = Shape<T, D, G>::W;
    b.max_batch = max_batch;
    k<<<ctas, Shape<T, D, G>::W * 32, sm, st>>>(b);
    return cudaGetLastError() == cudaSuccess ? ODA_OK : ODA_ERR_CUDA;
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
  // tickets must start at zero; a call that gave up early may have left some set
  if (cudaMemsetAsync(sd->tickets, 0, sizeof(int) * (size_t)B * cfg->hkv, st) != cudaSuccess)
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
  a.err = err ? err : sd->err;
  return dispatch<false>(*cfg, LaunchStatic{&a, sd->num_sms, cfg->max_batch, B, st});
}
