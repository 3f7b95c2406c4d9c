// Recall head on the tensor cores.
//
// [SUM] Methodology: after Local, a recall score q_t = R_psi(h_{t-1}, E(x_t),
// h^L_t) is computed from three states; [EXPL] Jargon / Recall head: a small
// trained module (about 1.7 % of the backbone). The pages fix the inputs and
// their order only; this library's head is
//     score = w2 . GELU(W1 [h_{t-1}; E(x_t); h^L_t] + b1) + b2.
//
// Shape of the work: D[m][n] = sum_k W1[m][k] X[n][k] with M = hidden (4096),
// N = batch (16), K = 3H (6144). The weight read (50 MB) bounds it; the MMA
// only has to keep up, which CUDA-core FMAs at 16 rows per weight do not.
//
// B200 design:
//   * the (m-tile, k-block) units are spread evenly over one CTA per SM
//     (split-K, "stream-K" style), so 32 m-tiles still fill 148 SMs;
//   * warp 0 streams 128x64 W1 tiles and N x64 X tiles with TMA (tensor maps,
//     128-byte swizzle) into a ring of shared-memory stages; X is read from
//     the three input tensors in place (three tensor maps, no concat copy);
//   * warp 1 issues tcgen05.mma (kind::f16, bf16 in, f32 accumulate in TMEM,
//     M = 128, N = batch rounded up to 16) and releases stages with
//     tcgen05.commit;
//   * warps 2..5 read the accumulator with tcgen05.ld. CTAs sharing an m-tile
//     write partials; the last to take the m-tile's ticket sums them in a
//     fixed order, adds b1, applies GELU and the w2 dot product; the last
//     m-tile sums the per-tile dot products in order and adds b2. The result
//     is deterministic run to run.
#include <cooperative_groups.h>
#include <cuda.h>

#include "gate.cuh"
#include "oda_internal.cuh"

using namespace oda;

namespace {

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 bf16 = one 128-byte swizzle row
constexpr int A_STAGE_BYTES = BM * BK * 2;
constexpr int MAX_N = 256;
constexpr int MAX_MT = 64;             // hidden <= 8192
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct RecallArgs {
  const float* b1;
  const float* w2;
  float b2;
  float* scores;
  float* partials;   // [P + MT][N][128]
  float* spart;      // [MT][N]
  int* tickets;      // [MT] per m-tile, [MAX_MT] for the final sum
  int* err;
  int B, N, MT, KB, H, stages;
  // Cluster kernel only: stage the first W1 tiles before the dependency wait
  // (the weights were written before the previous kernel started), and gate
  // the scores in the last CTA (gate_scores non-null).
  int early;
  const float* gate_scores;     // the scores the gate compares (the head's own or given)
  float theta;
  uint8_t* flags;
  int32_t* idx;
  int32_t* count;
  unsigned long long cond;      // conditional-node handle set from the count, if set_cond
  int set_cond;
  // Cluster kernel after the step's prefix kernel (pre non-null): K starts at
  // k-block kb_begin, and pre [KS][hidden][N] (float32) holds the first
  // layer over k-blocks [0, kb_begin), split in KS quarters, rank r's share
  // being [r*kb_begin/KS, (r+1)*kb_begin/KS). The prefix's CTAs count
  // themselves in *pre_done once written; *pre_seen counts those of the
  // steps before (the last CTA adds MT). A rank that finds this step's
  // prefix incomplete computes its quarter itself; its owners then add no
  // prefix for it (nothing waits on the other kernel).
  int kb_begin;
  const float* pre;
  int* pre_done;
  int* pre_seen;
  int pre_expected;             // 0: no prefix ran for this call (every rank computes its quarter)
};

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// L2 prefetch of one tile of a tensor map (no completion to wait for).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y)
               : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), leading offset unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Instruction descriptor: kind::f16, bf16 A and B (K-major), f32 D, M=128.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void epi_bar() {  // named barrier over the 4 epilogue warps
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ float gelu_erf(float u) {
  return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f));
}

__global__ void __launch_bounds__(192, 1)
recall_kernel(const __grid_constant__ CUtensorMap tm_w1, const __grid_constant__ CUtensorMap tm_x0,
              const __grid_constant__ CUtensorMap tm_x1, const __grid_constant__ CUtensorMap tm_x2,
              const RecallArgs a) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  unsigned char* smem = smem_raw + pad;
  const int S = a.stages;
  const int N = a.N;
  const uint32_t b_stage_bytes = (uint32_t)N * BK * 2;
  unsigned char* sa = smem;
  unsigned char* sb = sa + (size_t)S * A_STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sb + (size_t)S * b_stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* acc_full = bars + 2 * S;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* done_bar = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 3);
  int* sflag = reinterpret_cast<int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(sflag + 4);  // [4][MAX_N]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int U = a.MT * a.KB;
  const int P = (int)gridDim.x;
  const int c = (int)blockIdx.x;
  const int u0 = (int)(((long long)c * U) / P);
  const int u1 = (int)(((long long)(c + 1) * U) / P);
  uint32_t ncols = 32;
  while ((int)ncols < N) ncols <<= 1;

  pdl_wait();
  pdl_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_addr(&full[s]), 1);
      mbar_init(smem_addr(&empty[s]), 1);
    }
    mbar_init(smem_addr(acc_full), 1);
    mbar_init(smem_addr(acc_empty), 4);
    mbar_init(smem_addr(done_bar), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (u0 < u1) {
    if (warp == 0) {
      // ------------------------------------------------------ TMA producer
      if (lane == 0) {
        const uint32_t tx = A_STAGE_BYTES + b_stage_bytes;
        for (int u = u0, i = 0; u < u1; ++u, ++i) {
          const int s = i % S;
          const uint32_t par = (uint32_t)(((i / S) & 1) ^ 1);
          if (!mbar_wait_bounded(smem_addr(&empty[s]), par, kWaitLimitNs)) {
            record_error(a.err, ODA_ERR_TIMEOUT);
            break;
          }
          const int mt = u / a.KB, kb = u % a.KB;
          const uint32_t fb = smem_addr(&full[s]);
          mbar_arrive_expect_tx(fb, tx);
          tma_load_2d(smem_addr(sa + (size_t)s * A_STAGE_BYTES), &tm_w1, kb * BK, mt * BM, fb);
          const int kglob = kb * BK;
          const int seg = kglob / a.H;
          const int kin = kglob - seg * a.H;
          const CUtensorMap* xm = seg == 0 ? &tm_x0 : (seg == 1 ? &tm_x1 : &tm_x2);
          tma_load_2d(smem_addr(sb + (size_t)s * b_stage_bytes), xm, kin, 0, fb);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------- MMA issuer
      if (lane == 0) {
        const uint32_t idesc = umma_idesc_bf16(N);
        int i = 0, j = 0;
        bool ok = true;
        for (int u = u0; u < u1 && ok; ++j) {
          const int mt = u / a.KB;
          const int uend = min(u1, (mt + 1) * a.KB);
          if (j > 0 && !mbar_wait_bounded(smem_addr(acc_empty), (uint32_t)((j - 1) & 1),
                                          kWaitLimitNs)) {
            record_error(a.err, ODA_ERR_TIMEOUT);
            break;
          }
          fence_after_sync();
          for (; u < uend; ++u, ++i) {
            const int s = i % S;
            if (!mbar_wait_bounded(smem_addr(&full[s]), (uint32_t)((i / S) & 1), kWaitLimitNs)) {
              record_error(a.err, ODA_ERR_TIMEOUT);
              ok = false;
              break;
            }
            fence_after_sync();
            const uint64_t ad = umma_desc_sw128(smem_addr(sa + (size_t)s * A_STAGE_BYTES));
            const uint64_t bd = umma_desc_sw128(smem_addr(sb + (size_t)s * b_stage_bytes));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              // +32 bytes per 16-element K step inside the swizzled row
              umma_bf16(tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc,
                        (u == max(u0, mt * a.KB) && kk == 0) ? 0u : 1u);
            }
            umma_commit(smem_addr(&empty[s]));
          }
          if (ok) umma_commit(smem_addr(acc_full));
        }
        umma_commit(smem_addr(done_bar));
      }
    } else {
      // ------------------------------------------------------- epilogue
      const int q = warp & 3;              // TMEM lane quarter this warp may read
      const int m = q * 32 + lane;         // row of the m-tile
      const int ew = warp - 2;             // 0..3
      int j = 0;
      for (int u = u0; u < u1; ++j) {
        const int mt = u / a.KB;
        const int seg_lo = mt * a.KB, seg_hi = (mt + 1) * a.KB;
        const int uend = min(u1, seg_hi);
        u = uend;
        // one elected waiter so that all four epilogue warps agree on the outcome
        if (tid == 64) {
          const bool got = mbar_wait_bounded(smem_addr(acc_full), (uint32_t)(j & 1), kWaitLimitNs);
          if (!got) record_error(a.err, ODA_ERR_TIMEOUT);
          sflag[2] = got ? 1 : 0;
        }
        epi_bar();
        if (!sflag[2]) break;
        fence_after_sync();
        const int c_first = (int)(((long long)(seg_lo + 1) * P - 1) / U);
        const int c_last = (int)(((long long)seg_hi * P - 1) / U);
        const int nparts = c_last - c_first + 1;
        // partials are [CTA + m-tile][row m][N]: a row's N sums are contiguous
        float* mypart = a.partials + ((size_t)(c + mt) * BM + m) * N;
        // TMEM -> registers -> partials (always written; the merge reads them)
        for (int n0 = 0; n0 < N; n0 += 16) {
          float v[16];
          tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)n0, v);
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(mypart + n0 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
        fence_before_sync();
        if (lane == 0) mbar_arrive(smem_addr(acc_empty));
        epi_bar();
        bool last = true;
        if (nparts > 1) {
          if (tid == 64) {
            const int prev = ticket_add(&a.tickets[mt], 1);   // releases this partial
            sflag[0] = (prev == nparts - 1) ? 1 : 0;
          }
          epi_bar();
          last = sflag[0] != 0;
          epi_bar();
        }
        if (last) {
          // (the last ticket acquired every other CTA's partial)
          const float bias = a.b1[mt * BM + m];
          const float wo = a.w2[mt * BM + m];
          for (int n0 = 0; n0 < N; n0 += 16) {
            // row m's 16 sums of every partial: all loads in flight together
            float4 s4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) s4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            constexpr int PB = 4;
            for (int c0 = c_first; c0 <= c_last; c0 += PB) {
              float4 v4[PB][4];
#pragma unroll
              for (int u = 0; u < PB; ++u)
                if (c0 + u <= c_last) {
                  const float4* src = reinterpret_cast<const float4*>(
                      a.partials + ((size_t)(c0 + u + mt) * BM + m) * N + n0);
#pragma unroll
                  for (int e = 0; e < 4; ++e) v4[u][e] = __ldcg(src + e);
                }
#pragma unroll
              for (int u = 0; u < PB; ++u)
                if (c0 + u <= c_last) {
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    s4[e].x += v4[u][e].x; s4[e].y += v4[u][e].y;
                    s4[e].z += v4[u][e].z; s4[e].w += v4[u][e].w;
                  }
                }
            }
            float contrib[16];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              contrib[4 * e + 0] = wo * gelu_erf(s4[e].x + bias);
              contrib[4 * e + 1] = wo * gelu_erf(s4[e].y + bias);
              contrib[4 * e + 2] = wo * gelu_erf(s4[e].z + bias);
              contrib[4 * e + 3] = wo * gelu_erf(s4[e].w + bias);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
              for (int e = 0; e < 16; ++e) contrib[e] += __shfl_xor_sync(0xffffffffu, contrib[e], o);
            if (lane == 0) {
#pragma unroll
              for (int e = 0; e < 16; ++e) red[ew * MAX_N + n0 + e] = contrib[e];
            }
          }
          epi_bar();
          for (int n = tid - 64; n < N; n += 128) {
            // fixed order over the four row quarters: rows 0-31, 32-63, 64-95, 96-127
            float s = 0.f;
            for (int qq = 0; qq < 4; ++qq) s += red[((qq + 2) & 3) * MAX_N + n];
            a.spart[(size_t)mt * N + n] = s;
          }
          if (tid == 64) a.tickets[mt] = 0;
          epi_bar();
          if (tid == 64) {
            const int prev = ticket_add(&a.tickets[MAX_MT], 1);   // releases the row sums
            sflag[1] = (prev == a.MT - 1) ? 1 : 0;
          }
          epi_bar();
          if (sflag[1]) {
            // (the last ticket acquired every m-tile's row sums)
            // every (m-tile, row) dot product loaded at once, summed in a
            // fixed order: thread j takes row j % Bc and m-tiles j / Bc + k*step
            const int j = tid - 64;
            const int Bc = a.B < 128 ? a.B : 128;
            const int step = 128 / Bc;
            float* red2 = red;                         // [128] partial sums
            for (int n0 = 0; n0 < a.B; n0 += Bc) {     // same trip count on every thread
              const int n = n0 + j % Bc;
              float s = 0.f;
              if (j / Bc < step && n < a.B) {
                float v[8];
                int t2 = j / Bc;
                for (; t2 + 7 * step < a.MT; t2 += 8 * step) {
#pragma unroll
                  for (int u = 0; u < 8; ++u) v[u] = __ldcg(a.spart + (size_t)(t2 + u * step) * N + n);
#pragma unroll
                  for (int u = 0; u < 8; ++u) s += v[u];
                }
                for (; t2 < a.MT; t2 += step) s += __ldcg(a.spart + (size_t)t2 * N + n);
              }
              epi_bar();
              if (j / Bc < step) red2[j] = s;
              epi_bar();
              if (j < Bc && n < a.B) {
                float tsum = 0.f;
                for (int k = 0; k < step; ++k) tsum += red2[k * Bc + j];
                a.scores[n] = tsum + a.b2;
              }
              epi_bar();
            }
            if (tid == 64) a.tickets[MAX_MT] = 0;
          }
          epi_bar();
        }
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    // all MMAs of this CTA must have completed before TMEM is released
    if (u0 < u1) {
      if (!mbar_wait_bounded(smem_addr(done_bar), 0u, kWaitLimitNs) && lane == 0)
        record_error(a.err, ODA_ERR_TIMEOUT);
    }
    __syncwarp();
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols)
                 : "memory");
  }
}

// Split-K over a thread-block cluster. For the common shape (hidden / 128
// m-tiles times KS fit the SMs, batch <= 64) the K range of each m-tile is
// split evenly over a cluster of KS CTAs instead of the stream-K order above:
// no CTA spans two m-tiles, and the split is reduced in distributed shared
// memory. Rank r owns rows [r*128/KS, (r+1)*128/KS) of the m-tile: every rank
// pushes its accumulator rows to their owners with remote stores, one cluster
// barrier publishes them, each owner sums its rows' KS parts in rank order,
// adds b1, applies GELU and w2 and reduces over its rows, and writes one
// partial dot product per batch row; the last CTA of the grid (ticket) sums
// those in a fixed order and adds b2. Deterministic, like the stream-K path.
constexpr int CL_MAX_N = 64;                             // batch rows (16, 32 or 64 columns)

__global__ void __launch_bounds__(192, 1)
recall_cluster_kernel(const __grid_constant__ CUtensorMap tm_w1,
                      const __grid_constant__ CUtensorMap tm_x0,
                      const __grid_constant__ CUtensorMap tm_x1,
                      const __grid_constant__ CUtensorMap tm_x2, const RecallArgs a, int KS) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  unsigned char* smem = smem_raw + pad;
  const int S = a.stages;
  const int N = a.N;
  const uint32_t b_stage_bytes = (uint32_t)N * BK * 2;
  unsigned char* sa = smem;
  unsigned char* sb = sa + (size_t)S * A_STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sb + (size_t)S * b_stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* acc_full = bars + 2 * S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  int* sflag = reinterpret_cast<int*>(tmem_slot + 1);
  float* rbuf = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(sflag + 4) + 15) & ~uintptr_t(15));   // [KS][128/KS][N]
  float* red = rbuf + BM * N;                             // [192] partial sums

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int rank = (int)blockIdx.x % KS;
  const int mt = (int)blockIdx.x / KS;
  const int kspan = a.KB - a.kb_begin;
  const int kb0 = a.kb_begin + (rank * kspan) / KS, kb1 = a.kb_begin + ((rank + 1) * kspan) / KS;
  // this rank's quarter of the prefix's K range (computed here only if the
  // prefix kernel had not finished)
  const int qb0 = (rank * a.kb_begin) / KS, qb1 = ((rank + 1) * a.kb_begin) / KS;
  const int RP = BM / KS;                                 // rows each rank owns
  uint32_t ncols = 32;
  while ((int)ncols < N) ncols <<= 1;

  cluster_arrive_relaxed();                               // "started": waited for before any push
  // Early mode: the first stages' W1 tiles are requested before the
  // dependency wait (each stage's barrier expects the W1 and the state tile;
  // the state tile, which a preceding kernel may write, follows after the
  // wait). The owner rows' b1 and w2 are read with them.
  const int pre = a.early ? min(S, kb1 - kb0) : 0;
  float* sb1 = red + 192;                                 // [RP] b1 of the owned rows
  float* sw2 = sb1 + BM;                                  // [RP] w2 of the owned rows
  float* sp1 = sw2 + BM;                                  // [KS][RP][N] prefix of the owned rows
  int* pflag = reinterpret_cast<int*>(sp1 + BM * N);      // [KS] rank r used the prefix
  if (tid == 0) {
    sflag[3] = 0;                                         // the prefix decision is not made yet
    for (int s2 = 0; s2 < S; ++s2) {
      mbar_init(smem_addr(&full[s2]), 1);
      mbar_init(smem_addr(&empty[s2]), 1);
    }
    mbar_init(smem_addr(acc_full), 1);
    fence_mbar_init();
    const uint32_t tx = A_STAGE_BYTES + b_stage_bytes;
    for (int i = 0; i < pre; ++i) {
      const uint32_t fb = smem_addr(&full[i]);
      mbar_arrive_expect_tx(fb, tx);
      tma_load_2d(smem_addr(sa + (size_t)i * A_STAGE_BYTES), &tm_w1, (kb0 + i) * BK, mt * BM, fb);
    }
    // the share's W1 tiles beyond the stages go to L2, so that the loads
    // which refill the stages after the wait find them there
    if (a.early)
      for (int i = pre; i < kb1 - kb0; ++i) tma_prefetch_2d(&tm_w1, (kb0 + i) * BK, mt * BM);
  }
  auto load_owner_weights = [&]() {
    for (int rl = tid - 64; rl >= 0 && rl < RP; rl += 128) {
      const int row = mt * BM + rank * RP + rl;
      sb1[rl] = a.b1[row];
      sw2[rl] = a.w2[row];
    }
  };
  if (a.early && warp >= 2) load_owner_weights();
  pdl_wait();
  pdl_launch_dependents();
  if (!a.early && warp >= 2) load_owner_weights();
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // k-blocks: this rank's share of the head's range, then (prefix
  // incomplete) its quarter of the prefix's range
  const int n2 = kb1 - kb0;
  auto kb_at = [&](int i) { return i < n2 ? kb0 + i : qb0 + (i - n2); };
  // With a prefix, the epilogue warps decide (off the dependency wait's
  // path; the weights already stream) whether this step's prefix is complete:
  // once MT more of its CTAs have counted themselves than in the steps before
  // (acquire: its rows are then visible). If so they load every quarter of the
  // owned rows' prefix with 16-byte asynchronous copies (each thread waits
  // for its own before the cluster barrier that precedes their use). The
  // producer and the MMA issuer read the decision when their share of the
  // head's range is done (sflag[3] says it is made).
  bool use_pre = false;
  if (a.pre && warp >= 2) {
    if (tid == 64) {
      int done;
      asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(done) : "l"(a.pre_done) : "memory");
      sflag[2] = (a.pre_expected && done - __ldcg(a.pre_seen) >= a.MT) ? 1 : 0;
      __threadfence_block();
      *reinterpret_cast<volatile int*>(&sflag[3]) = 1;
    }
    epi_bar();
    use_pre = sflag[2] != 0;
    if (use_pre) {
      for (int c = tid - 64; c < BM * N / 4; c += 128) {
        const int i = 4 * c;
        const int r2 = i / (RP * N), rem = i - r2 * RP * N;
        cp_async16(smem_addr(sp1 + i),
                   a.pre + ((size_t)r2 * a.MT * BM + (size_t)mt * BM + (size_t)rank * RP) * N + rem);
      }
    }
  }
  // producer / MMA issuer (lane 0): k-blocks after the head's share
  auto more_kb = [&]() -> int {
    if (!a.pre) return 0;
    for (long it = 0; *reinterpret_cast<volatile int*>(&sflag[3]) == 0; ++it) {
      if (it > (1L << 26)) {                              // bounded: never reached in practice
        record_error(a.err, ODA_ERR_TIMEOUT);
        return 0;
      }
    }
    __threadfence_block();
    return sflag[2] ? 0 : qb1 - qb0;
  };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t tx = A_STAGE_BYTES + b_stage_bytes;
      int nkb = n2;
      for (int i = 0; i < nkb; ++i) {
        if (i == n2 - 1) nkb += more_kb();
        const int kb = kb_at(i);
        const int s2 = i % S;
        const uint32_t fb = smem_addr(&full[s2]);
        if (i >= pre) {                                   // else W1 was requested early
          const uint32_t par = (uint32_t)(((i / S) & 1) ^ 1);
          if (!mbar_wait_bounded(smem_addr(&empty[s2]), par, kWaitLimitNs)) {
            record_error(a.err, ODA_ERR_TIMEOUT);
            break;
          }
          mbar_arrive_expect_tx(fb, tx);
          tma_load_2d(smem_addr(sa + (size_t)s2 * A_STAGE_BYTES), &tm_w1, kb * BK, mt * BM, fb);
        }
        const int kglob = kb * BK;
        const int seg = kglob / a.H;
        const int kin = kglob - seg * a.H;
        const CUtensorMap* xm = seg == 0 ? &tm_x0 : (seg == 1 ? &tm_x1 : &tm_x2);
        tma_load_2d(smem_addr(sb + (size_t)s2 * b_stage_bytes), xm, kin, 0, fb);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(N);
      int nkb = n2;
      for (int i = 0; i < nkb; ++i) {
        if (i == n2 - 1) nkb += more_kb();
        const int s2 = i % S;
        if (!mbar_wait_bounded(smem_addr(&full[s2]), (uint32_t)((i / S) & 1), kWaitLimitNs)) {
          record_error(a.err, ODA_ERR_TIMEOUT);
          break;
        }
        fence_after_sync();
        const uint64_t ad = umma_desc_sw128(smem_addr(sa + (size_t)s2 * A_STAGE_BYTES));
        const uint64_t bd = umma_desc_sw128(smem_addr(sb + (size_t)s2 * b_stage_bytes));
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_bf16(tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc,
                    (i == 0 && kk == 0) ? 0u : 1u);
        umma_commit(smem_addr(&empty[s2]));
      }
      umma_commit(smem_addr(acc_full));                   // after every MMA above
    }
  }

  // ------------------------------------------------- push rows to owners
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  if (tid == 64) {
    const bool got = n2 > 0 &&
                     mbar_wait_bounded(smem_addr(acc_full), 0u, kWaitLimitNs);
    if (!got && n2 > 0) record_error(a.err, ODA_ERR_TIMEOUT);
    sflag[0] = got ? 1 : 0;
  }
  __syncthreads();
  fence_after_sync();
  cluster_wait();                                         // every rank has started
  if (warp >= 2) {
    const int q = warp & 3;                               // TMEM lane quarter of this warp
    const int m = q * 32 + lane;                          // row of the m-tile
    const int owner = m / RP;
    float* dst = cl.map_shared_rank(rbuf, owner) + ((size_t)rank * RP + (m - owner * RP)) * N;
    for (int n0 = 0; n0 < N; n0 += 16) {
      float v[16];
      if (sflag[0]) {
        tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)n0, v);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 16; e += 4)
        *reinterpret_cast<float4*>(dst + n0 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
    }
    // every owner learns whether this rank's rows include its prefix quarter
    if (a.pre && tid - 64 < KS) cl.map_shared_rank(pflag, tid - 64)[rank] = use_pre ? 1 : 0;
    if (use_pre) cp_async_wait_all();                     // this thread's prefix copies
  }
  fence_before_sync();
  cluster_arrive();                                       // release: the pushes
  cluster_wait();                                         // acquire: every rank's pushes

  // ------------------------------------- owner: b1, GELU, w2 over its rows
  if (a.pre && !use_pre && warp >= 2) {
    // (rare) this rank found the prefix incomplete but another did: that
    // rank's quarter of the owned rows is read now (the barrier ordered it
    // after that rank's acquire)
    for (int i = tid - 64; i < BM * N; i += 128) {
      const int r2 = i / (RP * N), rem = i - r2 * RP * N;
      if (pflag[r2])
        sp1[i] = __ldcg(a.pre + ((size_t)r2 * a.MT * BM + (size_t)mt * BM + (size_t)rank * RP) * N +
                        rem);
    }
    epi_bar();
  }
  // Only the batch's columns are reduced (B rounded up to a power of two, at
  // most N, itself a power of two here; the tile's other columns are
  // padding): TPN threads per column, each taking rows t0, t0 + TPN, ... of
  // the owned ones.
  int NB = 1;
  while (NB < a.B) NB <<= 1;
  const int TPN = BM / NB;                                // threads per batch column
  const int TPR = TPN < RP ? TPN : RP;                    // of which hold rows
  if (warp >= 2) {
    const int j = tid - 64;                               // 0..127
    const int n = j % NB, t0 = j / NB;
    float s = 0.f;
    // fixed order; unrolled so that the rows' GELU chains overlap
#pragma unroll 4
    for (int rl = t0; rl < RP; rl += TPN) {
      float u = 0.f;
#pragma unroll 4
      for (int r2 = 0; r2 < KS; ++r2) {
        float v = rbuf[((size_t)r2 * RP + rl) * N + n];
        if (a.pre) {
          const float p = sp1[((size_t)r2 * RP + rl) * N + n];
          v += pflag[r2] ? p : 0.f;                       // rank r2's prefix quarter
        }
        u += v;
      }
      s += sw2[rl] * gelu_erf(u + sb1[rl]);
    }
    red[j] = s;
  }
  __syncthreads();
  if (warp >= 2) {
    const int j = tid - 64;
    if (j < NB) {
      float s = 0.f;
#pragma unroll 8
      for (int t2 = 0; t2 < TPR; ++t2) s += red[t2 * NB + j];
      a.spart[(size_t)blockIdx.x * N + j] = s;
    }
  }
  __syncthreads();
  if (tid == 64) {
    const int prev = ticket_add(&a.tickets[MAX_MT], 1);   // releases this CTA's partials
    sflag[1] = (prev == (int)gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (sflag[1]) {
    // (the ticket acquired every CTA's partial) thread (n, sub) of a group of
    // TPR lanes, a power of two within one warp, adds CTAs sub, sub + TPR, ...
    // of batch row n in CTA order; xor shuffles then add the group's lanes in
    // a fixed order
    int TPR = 32;
    while (TPR > 1 && TPR * a.B > 192) TPR >>= 1;
    const int n = tid / TPR, sub = tid % TPR;
    const bool row = n < a.B;
    // With at most 32 rows warp 0 gates alone; scores given to the gate from
    // outside are requested together with the partials.
    const bool warp_gate = a.gate_scores != nullptr && a.B <= 32;
    const bool own = a.gate_scores == a.scores;
    float gval = 0.f;
    if (warp_gate && !own && tid < a.B) gval = __ldcg(a.gate_scores + tid);
    float v = 0.f;
    if (row) {
      // eight partials requested at a time, added in CTA order
      for (int c2 = sub; c2 < (int)gridDim.x; c2 += 8 * TPR) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int cc = c2 + u * TPR;
          x[u] = cc < (int)gridDim.x ? __ldcg(a.spart + (size_t)cc * N + n) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) v += x[u];
      }
    }
    for (int o = 1; o < TPR; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (row && sub == 0) {
      a.scores[n] = v + a.b2;
      red[n] = v + a.b2;
    }
    __syncthreads();
    if (warp_gate && own && tid < a.B) gval = red[tid];
    if (tid == 0) {
      a.tickets[MAX_MT] = 0;
      if (a.pre && a.pre_expected) *a.pre_seen += a.MT;   // this step's prefix is accounted for
    }
    if (warp_gate) {
      if (warp == 0)
        gate_warp(gval, a.B, a.theta, a.flags, a.idx, a.count, (cudaGraphConditionalHandle)a.cond,
                  a.set_cond);
    } else if (a.gate_scores) {
      __syncthreads();                                    // the scores above are visible
      gate_block(a.gate_scores, a.theta, a.B, a.flags, a.idx, a.count,
                 (cudaGraphConditionalHandle)a.cond, a.set_cond, reinterpret_cast<int*>(red));
    }
  }
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    // every MMA must have completed before TMEM is released
    if (n2 > 0 && !mbar_wait_bounded(smem_addr(acc_full), 0u, kWaitLimitNs) && lane == 0)
      record_error(a.err, ODA_ERR_TIMEOUT);
    __syncwarp();
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols)
                 : "memory");
  }
}

// The first layer over the K range of h_{t-1} and E(x_t), which are known
// when a decode step starts (h^L_t only after its last Local launch): one
// m-tile per CTA over k-blocks [0, kb_end), in KS quarters (the cluster
// kernel's ranks' shares), each accumulated on its own in TMEM and written
// to pre [KS][hidden][N] in float32; then the CTA counts itself in
// *pre_done (release). Sized to run beside the Local launches: four warps
// (producer, MMA issuer, then all four read one TMEM lane quarter each), two
// stages, at most 80 registers, so that it fits an SM that holds two Local
// CTAs.
__global__ void __launch_bounds__(128, 6)
recall_prefix_kernel(const __grid_constant__ CUtensorMap tm_w1,
                     const __grid_constant__ CUtensorMap tm_x0,
                     const __grid_constant__ CUtensorMap tm_x1, const RecallArgs a, float* pre,
                     int kb_end, int KS) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  unsigned char* smem = smem_raw + pad;
  const int S = a.stages;
  const int N = a.N;
  const uint32_t b_stage_bytes = (uint32_t)N * BK * 2;
  unsigned char* sa = smem;
  unsigned char* sb = sa + (size_t)S * A_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sb + (size_t)S * b_stage_bytes);
  uint64_t* empty = full + S;
  uint64_t* acc_full = full + 2 * S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int mt = (int)blockIdx.x;
  uint32_t ncols = 32;
  while ((int)ncols < KS * N) ncols <<= 1;
  if (tid == 0) {
    for (int s2 = 0; s2 < S; ++s2) {
      mbar_init(smem_addr(&full[s2]), 1);
      mbar_init(smem_addr(&empty[s2]), 1);
    }
    mbar_init(smem_addr(acc_full), 1);
    fence_mbar_init();
  }
  pdl_wait();
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int m = warp * 32 + lane;                         // row of the m-tile (TMEM lane)

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    const uint32_t tx = A_STAGE_BYTES + b_stage_bytes;
    for (int kb = 0; kb < kb_end; ++kb) {
      const int s2 = kb % S;
      if (!mbar_wait_bounded(smem_addr(&empty[s2]), (uint32_t)(((kb / S) & 1) ^ 1),
                             kWaitLimitNs)) {
        record_error(a.err, ODA_ERR_TIMEOUT);
        break;
      }
      const uint32_t fb = smem_addr(&full[s2]);
      mbar_arrive_expect_tx(fb, tx);
      tma_load_2d(smem_addr(sa + (size_t)s2 * A_STAGE_BYTES), &tm_w1, kb * BK, mt * BM, fb);
      const int kglob = kb * BK;
      const int seg = kglob / a.H;
      tma_load_2d(smem_addr(sb + (size_t)s2 * b_stage_bytes), seg == 0 ? &tm_x0 : &tm_x1,
                  kglob - seg * a.H, 0, fb);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------- MMA issuer
    const uint32_t idesc = umma_idesc_bf16(N);
    int q = 0, qstart = 0, qnext = kb_end / KS;           // quarter q: [q*kb_end/KS, (q+1)*kb_end/KS)
    for (int kb = 0; kb < kb_end; ++kb) {
      while (kb >= qnext) {
        ++q;
        qstart = qnext;
        qnext = ((q + 1) * kb_end) / KS;
      }
      const int s2 = kb % S;
      if (!mbar_wait_bounded(smem_addr(&full[s2]), (uint32_t)((kb / S) & 1), kWaitLimitNs)) {
        record_error(a.err, ODA_ERR_TIMEOUT);
        break;
      }
      fence_after_sync();
      const uint64_t ad = umma_desc_sw128(smem_addr(sa + (size_t)s2 * A_STAGE_BYTES));
      const uint64_t bd = umma_desc_sw128(smem_addr(sb + (size_t)s2 * b_stage_bytes));
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        umma_bf16(tmem + (uint32_t)(q * N), ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk),
                  idesc, (kb == qstart && kk == 0) ? 0u : 1u);
      umma_commit(smem_addr(&empty[s2]));
    }
    umma_commit(smem_addr(acc_full));                     // after every MMA above
  }
  __syncwarp();
  // ---------------------------------------- epilogue: one lane quarter per warp
  const bool got = __all_sync(0xffffffffu, kb_end > 0 && mbar_wait_bounded(smem_addr(acc_full),
                                                                              0u, kWaitLimitNs));
  if (!got && kb_end > 0 && lane == 0) record_error(a.err, ODA_ERR_TIMEOUT);
  fence_after_sync();
  for (int q = 0; q < KS; ++q) {
    float* dst = pre + ((size_t)q * a.MT * BM + (size_t)mt * BM + m) * N;
    for (int n0 = 0; n0 < N; n0 += 16) {
      float v[16];
      if (got) {
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(q * N + n0), v);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 16; e += 4)
        *reinterpret_cast<float4*>(dst + n0 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
    }
  }
  fence_before_sync();
  __syncthreads();
  // every row written: count this CTA (release; a timed-out CTA does not)
  if (tid == 0 && got)
    asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(a.pre_done) : "memory");
  if (warp == 0) {
    // every MMA must have completed before TMEM is released
    if (kb_end > 0 && !got && !mbar_wait_bounded(smem_addr(acc_full), 0u, kWaitLimitNs) &&
        lane == 0)
      record_error(a.err, ODA_ERR_TIMEOUT);
    __syncwarp();
    fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols)
                 : "memory");
  }
}

// ------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool encode_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_in,
               uint32_t box_out) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_in, box_out};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int stages_for(int n) {
  const int per = A_STAGE_BYTES + n * BK * 2;
  int s = (200 * 1024) / per;
  if (s > 8) s = 8;
  if (s < 2) s = 2;
  return s;
}

size_t smem_for(int n, int s) {
  return 1024 + (size_t)s * (A_STAGE_BYTES + n * BK * 2) + (size_t)(2 * s + 3) * 8 + 4 + 16 +
         4 * MAX_N * 4 + 64;
}

// Shared memory of the cluster kernel with s stages (its row buffer comes first).
size_t cl_smem_for(int n, int s, size_t extra = 0) {
  return 1024 + (size_t)s * (A_STAGE_BYTES + n * BK * 2) + (size_t)(2 * s + 1) * 8 + 4 + 16 + 16 +
         (size_t)(BM * n + 192 + 2 * BM) * 4 + extra + 64;
}

// `extra` after the prefix kernel: every quarter of the owned rows' prefix
// (KS * 128/KS * n floats) and the ranks' flags
size_t cl_pre_bytes(int n) { return (size_t)BM * n * 4 + 64; }

// The cluster kernel's shared-memory limit: the most one CTA may have.
constexpr size_t kClusterSmemMax = 227 * 1024;

// Stages of the cluster kernel within `budget` bytes of shared memory.
int cl_stages_within(int n, size_t budget, size_t extra) {
  int s = 8;
  while (s > 2 && cl_smem_for(n, s, extra) > budget) --s;
  return s;
}

// The prefix kernel: two stages (it runs beside two Local CTAs).
#ifndef ODA_PREFIX_STAGES
#define ODA_PREFIX_STAGES 2
#endif
constexpr int kPrefixStages = ODA_PREFIX_STAGES;
size_t prefix_smem_for(int n) {
  return 1024 + (size_t)kPrefixStages * (A_STAGE_BYTES + n * BK * 2) +
         (size_t)(2 * kPrefixStages + 1) * 8 + 4 + 64;
}

// Cluster size of the split-K kernel for batch width N, or 0 for the
// stream-K kernel: every m-tile gets a whole cluster within one wave.
int cluster_ks(const oda_ctx* ctx, int N, int MT, int KB) {
  if (N != 16 && N != 32 && N != 64) return 0;
  for (int ks = ctx->recall_cluster_max; ks >= 2; ks >>= 1)
    if (MT * ks <= ctx->num_sms && KB >= ks) return ks;
  return 0;
}

bool shape_ok(int B, int H, int hidden) {
  return B >= 1 && B <= MAX_N && H >= BK && H % BK == 0 && hidden >= BM && hidden % BM == 0 &&
         hidden / BM <= MAX_MT;
}

}  // namespace

namespace oda_impl {

oda_status recall_setup(oda_ctx* ctx) {
  const size_t max_smem = smem_for(MAX_N, stages_for(MAX_N));
  size_t best = max_smem;
  for (int n = 16; n <= MAX_N; n += 16) best = best > smem_for(n, stages_for(n)) ? best : smem_for(n, stages_for(n));
  ODA_CUDA_TRY(raise_smem_limit(reinterpret_cast<const void*>(recall_kernel), best));
  const size_t pfl = (size_t)(ctx->num_sms + MAX_MT) * MAX_N * BM + (size_t)MAX_MT * MAX_N;
  ODA_CUDA_TRY(cudaMalloc(&ctx->recall_partials, pfl * sizeof(float)));
  ctx->recall_parts_cap = (int)((size_t)(ctx->num_sms + MAX_MT) * MAX_N * BM);
  // tickets: [MAX_MT] per m-tile, [MAX_MT] the final sum, then the prefix's
  // done and seen counters
  ODA_CUDA_TRY(cudaMalloc(&ctx->recall_tickets, (MAX_MT + 3) * sizeof(int)));
  ODA_CUDA_TRY(cudaMemset(ctx->recall_tickets, 0, (MAX_MT + 3) * sizeof(int)));
  // the prefix: [KS][hidden][N] with KS * hidden / 128 <= SMs
  ODA_CUDA_TRY(cudaMalloc(&ctx->recall_pre,
                          (size_t)ctx->num_sms * BM * CL_MAX_N * sizeof(float)));
  ODA_CUDA_TRY(raise_smem_limit(reinterpret_cast<const void*>(recall_prefix_kernel),
                                prefix_smem_for(CL_MAX_N)));
  // the cluster split-K kernel: the largest cluster (8, 4, 2) the GPU holds
  ctx->recall_cluster_max = 0;
  const size_t csm = kClusterSmemMax;
  if (raise_smem_limit(reinterpret_cast<const void*>(recall_cluster_kernel), csm) ==
      cudaSuccess) {
    for (int ks = 8; ks >= 2; ks >>= 1) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(ks);
      cfg.blockDim = dim3(192);
      cfg.dynamicSmemBytes = csm;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = ks;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int ncl = 0;
      if (cudaOccupancyMaxActiveClusters(&ncl, recall_cluster_kernel, &cfg) == cudaSuccess &&
          ncl > 0) {
        ctx->recall_cluster_max = ks;
        break;
      }
    }
  }
  cudaGetLastError();
  return ODA_OK;
}

oda_status launch_recall(oda_ctx* ctx, const void* h_prev, const void* emb, const void* h_local,
                         int H, const void* W1, const float* b1, const float* w2, float b2,
                         int hidden, float* scores, int B, cudaStream_t st, bool early,
                         const RecallGate* gate, bool* gate_fused, bool after_prefix) {
  if (gate_fused) *gate_fused = false;
  if (!shape_ok(B, H, hidden)) return ODA_ERR_SHAPE;
  const bool split = recall_split(ctx, B, H, hidden);
  if (after_prefix && !split) return ODA_ERR_SHAPE;
  const int N = ((B + 15) / 16) * 16;
  CUtensorMap tw, t0, t1, t2;
  const uint64_t K = 3ull * (uint64_t)H;
  if (!encode_2d(&tw, W1, K, (uint64_t)hidden, BK, BM)) return ODA_ERR_CUDA;
  if (!encode_2d(&t0, h_prev, (uint64_t)H, (uint64_t)B, BK, (uint32_t)N)) return ODA_ERR_CUDA;
  if (!encode_2d(&t1, emb, (uint64_t)H, (uint64_t)B, BK, (uint32_t)N)) return ODA_ERR_CUDA;
  if (!encode_2d(&t2, h_local, (uint64_t)H, (uint64_t)B, BK, (uint32_t)N)) return ODA_ERR_CUDA;
  RecallArgs a;
  a.b1 = b1;
  a.w2 = w2;
  a.b2 = b2;
  a.scores = scores;
  a.partials = ctx->recall_partials;
  a.spart = ctx->recall_partials + ctx->recall_parts_cap;
  a.tickets = ctx->recall_tickets;
  a.err = ctx->err;
  a.B = B;
  a.N = N;
  a.MT = hidden / BM;
  a.KB = (int)(K / BK);
  a.H = H;
  a.early = 0;
  a.gate_scores = nullptr;
  a.theta = 0.f;
  a.flags = nullptr;
  a.idx = nullptr;
  a.count = nullptr;
  a.cond = 0ull;
  a.set_cond = 0;
  // Where the step splits the head, every call runs the split layout: after
  // the step's prefix kernel, or alone with every rank computing its quarter
  // of the prefix's range itself.
  a.kb_begin = split ? 2 * H / BK : 0;
  a.pre = split ? ctx->recall_pre : nullptr;
  a.pre_done = ctx->recall_tickets + MAX_MT + 1;
  a.pre_seen = ctx->recall_tickets + MAX_MT + 2;
  a.pre_expected = after_prefix ? 1 : 0;
  // cluster split-K when every m-tile gets a whole cluster within one wave
  const int KS = cluster_ks(ctx, N, a.MT, a.KB - a.kb_begin);
  if (KS >= 2) {
    const size_t extra = split ? cl_pre_bytes(N) : 0;
    a.stages = cl_stages_within(N, kClusterSmemMax, extra);
    if (early) {
      // The CTAs are to become resident beside the preceding Local launch's
      // CTAs (one per SM) and request W1 while it runs: fewer stages, so both
      // fit one SM's shared memory (1 KB of it is reserved per CTA).
      const size_t sm_total = 228 * 1024;
      const size_t beside = ctx->local_last_smem + 2 * 1024;
      if (ctx->local_last_smem > 0 && beside + cl_smem_for(N, 2, extra) <= sm_total)
        a.stages = cl_stages_within(N, sm_total - beside, extra);
      a.early = 1;
    }
    if (gate && B <= 192) {
      a.gate_scores = gate->scores ? gate->scores : scores;
      a.theta = gate->theta;
      a.flags = gate->flags;
      a.idx = gate->idx;
      a.count = gate->count;
      a.cond = gate->cond;
      a.set_cond = gate->set_cond ? 1 : 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.MT * KS);
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = cl_smem_for(N, a.stages, extra);
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = KS;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, recall_cluster_kernel, tw, t0, t1, t2, a, KS) != cudaSuccess)
      return ODA_ERR_CUDA;
    if (gate_fused) *gate_fused = a.gate_scores != nullptr;
    return ODA_OK;
  }
  a.stages = stages_for(N);
  const int U = a.MT * a.KB;
  const int grid = U < ctx->num_sms ? U : ctx->num_sms;
  return launch_pdl(recall_kernel, dim3(grid), dim3(192), smem_for(N, a.stages), st, tw, t0, t1,
                    t2, a) == cudaSuccess
             ? ODA_OK
             : ODA_ERR_CUDA;
}

bool recall_split(const oda_ctx* ctx, int B, int H, int hidden) {
  if (!shape_ok(B, H, hidden)) return false;
  const int N = ((B + 15) / 16) * 16;
  const int MT = hidden / BM;
  const int ks = cluster_ks(ctx, N, MT, H / BK);         // the cluster kernel's K: h^L_t
  return ks >= 2 && cluster_ks(ctx, N, MT, 3 * H / BK) == ks;
}

oda_status launch_recall_prefix(oda_ctx* ctx, const void* h_prev, const void* emb, int H,
                                const void* W1, const float* b1, int hidden, int B,
                                cudaStream_t st) {
  if (!recall_split(ctx, B, H, hidden)) return ODA_ERR_SHAPE;
  const int N = ((B + 15) / 16) * 16;
  CUtensorMap tw, t0, t1;
  if (!encode_2d(&tw, W1, 3ull * (uint64_t)H, (uint64_t)hidden, BK, BM)) return ODA_ERR_CUDA;
  if (!encode_2d(&t0, h_prev, (uint64_t)H, (uint64_t)B, BK, (uint32_t)N)) return ODA_ERR_CUDA;
  if (!encode_2d(&t1, emb, (uint64_t)H, (uint64_t)B, BK, (uint32_t)N)) return ODA_ERR_CUDA;
  RecallArgs a = {};
  a.b1 = b1;
  a.err = ctx->err;
  a.B = B;
  a.N = N;
  a.MT = hidden / BM;
  a.KB = 3 * H / BK;
  a.H = H;
  a.stages = kPrefixStages;
  a.pre_done = ctx->recall_tickets + MAX_MT + 1;
  const int KS = cluster_ks(ctx, N, a.MT, H / BK);       // the cluster kernel's ranks
  return launch_pdl(recall_prefix_kernel, dim3(a.MT), dim3(128), prefix_smem_for(N), st, tw, t0,
                    t1, a, ctx->recall_pre, 2 * H / BK, KS) == cudaSuccess
             ? ODA_OK
             : ODA_ERR_CUDA;
}

}  // namespace oda_impl
