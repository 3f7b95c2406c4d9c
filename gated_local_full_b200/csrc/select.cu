// Selection at a call budget on the device.
//
// [SUM] State-Dependent Access Effectiveness: at a fixed call budget (40 %),
// how much net gain a policy captures per reference position, against the
// expected gain of random selection; [SUM] Conclusion: the offline Oracle,
// which knows each position's true gain, selects better than the recall head.
// A policy spends k = floor(budget * n) Full calls on the k positions with the
// largest scores (the recall head's q_t, or the gain itself for the Oracle):
// equal scores (+0 and -0 included) go to the earlier position and NaN ranks
// below every number, so the selected set is unique. The net gain is the sum
// of the gains of the selected positions over n.
//
// Device work: an exact radix select of the k-th largest score key (four
// passes, one 8-bit digit each, MSB first; the last block of each pass picks
// the digit and updates the search state), a count of the keys equal to that
// threshold per contiguous chunk with an exclusive scan over the chunks, then
// one pass that marks key > threshold, or key == threshold with an
// index-ordered rank below the number of equal keys still to take, and sums
// the selected gains in float64 in a fixed order (deterministic). Each pass
// reads the scores once (4 B per position); the mark pass also reads the gain
// and writes one byte per position: bound by HBM.
#include "oda_internal.cuh"

using namespace oda;

namespace {

constexpr int kThreads = 256;
constexpr int kTile = kThreads;          // positions per block iteration of the ordered passes

// Order-preserving key of a float32 score: a larger key is a larger value;
// +0 and -0 share a key, and NaN takes key 0, below every number.
__device__ __forceinline__ uint32_t score_key(float f) {
  if (f != f) return 0u;
  const uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Search state in the context's selection scratch.
struct SelState {
  uint32_t prefix;       // digits of the threshold key fixed so far
  uint32_t mask;         // their bits
  long long k_rem;       // positions still to take among keys matching the prefix
  int ticket;            // last-block ticket of the current pass
  int pad[3];
};

struct SelScratch {
  SelState* st;
  uint32_t* hist;        // [256]
  int* bcnt;             // [kSelectMaxBlocks] equal keys per chunk, then exclusive prefix
  double* bsum;          // [kSelectMaxBlocks] selected gain per chunk
};

__global__ void sel_init_kernel(SelState* st, uint32_t* hist, long long k) {
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x;
  if (tid == 0) {
    // k == 0: a threshold above every key with nothing equal left to take
    st->prefix = k > 0 ? 0u : 0xFFFFFFFFu;
    st->mask = k > 0 ? 0u : 0xFFFFFFFFu;
    st->k_rem = k;
    st->ticket = 0;
  }
  for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0u;
}

// One radix pass: histogram of digit `round` (MSB first) among the keys that
// match the prefix; the last block picks the digit holding the k_rem-th
// largest key and updates the state.
__global__ void __launch_bounds__(kThreads)
sel_round_kernel(const float* __restrict__ scores, long long n, int round, SelScratch s) {
  __shared__ uint32_t h[256];
  __shared__ int last;
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x;
  for (int i = tid; i < 256; i += kThreads) h[i] = 0u;
  __syncthreads();
  const uint32_t prefix = s.st->prefix, mask = s.st->mask;
  const int shift = 24 - 8 * round;
  for (long long i = blockIdx.x * (long long)kThreads + tid; i < n;
       i += (long long)gridDim.x * kThreads) {
    const uint32_t key = score_key(__ldcs(scores + i));
    if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
  }
  __syncthreads();
  for (int i = tid; i < 256; i += kThreads)
    if (h[i]) atomicAdd(&s.hist[i], h[i]);
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(&s.st->ticket, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (tid < 32) {
    // lane L holds bins 8L .. 8L+7; suffix sums over the lanes find the bin
    // where the count from the top first reaches k_rem
    const int lane = tid;
    uint32_t b[8];
    unsigned long long own = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      b[e] = __ldcg(s.hist + 8 * lane + e);
      own += b[e];
    }
    unsigned long long suf = own;                    // sum over lanes >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += y;
    }
    const unsigned long long above = suf - own;       // keys in bins of higher lanes
    const long long k_rem = s.st->k_rem;
    if ((long long)above < k_rem && (long long)suf >= k_rem) {
      unsigned long long cum = above;
      int d = 8 * lane;
      for (int e = 7; e >= 0; --e) {
        if ((long long)(cum + b[e]) >= k_rem) { d = 8 * lane + e; break; }
        cum += b[e];
      }
      s.st->prefix = prefix | ((uint32_t)d << shift);
      s.st->mask = mask | (255u << shift);
      s.st->k_rem = k_rem - (long long)cum;
    }
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 8; ++e) s.hist[8 * lane + e] = 0u;
    if (lane == 0) s.st->ticket = 0;
  }
}

// Block-wide exclusive prefix of one flag per thread (kThreads threads), in
// thread order; returns the prefix and writes the block total to *total.
__device__ __forceinline__ int block_exclusive(bool f, int* warp_sums, int* total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, f);
  if (lane == 0) warp_sums[warp] = __popc(bal);
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) {
    const int c = warp_sums[w];
    before += w < warp ? c : 0;
    all += c;
  }
  __syncthreads();
  *total = all;
  return before + __popc(bal & ((1u << lane) - 1u));
}

// Keys equal to the threshold per contiguous chunk; the last block turns the
// counts into an exclusive prefix over the chunks (in chunk order).
__global__ void __launch_bounds__(kThreads)
sel_count_kernel(const float* __restrict__ scores, long long n, long long chunk, SelScratch s) {
  __shared__ int red[kThreads / 32];
  __shared__ int last;
  __shared__ int carry[kThreads];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t T = s.st->prefix;
  const long long c0 = blockIdx.x * chunk, c1 = min(n, c0 + chunk);
  int cnt = 0;
  for (long long i = c0 + tid; i < c1; i += kThreads) cnt += score_key(__ldcs(scores + i)) == T;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) red[warp] = cnt;
  __syncthreads();
  if (tid == 0) {
    int t = 0;
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
    s.bcnt[blockIdx.x] = t;
    __threadfence();
    last = atomicAdd(&s.st->ticket, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  // exclusive scan of gridDim.x <= 4 * kThreads counts: each thread owns four
  // consecutive chunks
  const int nb = (int)gridDim.x;
  int v[4], own = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int b = 4 * tid + e;
    v[e] = b < nb ? __ldcg(s.bcnt + b) : 0;
    own += v[e];
  }
  carry[tid] = own;
  __syncthreads();
  for (int o = 1; o < kThreads; o <<= 1) {          // inclusive scan (Hillis-Steele)
    const int y = tid >= o ? carry[tid - o] : 0;
    __syncthreads();
    carry[tid] += y;
    __syncthreads();
  }
  int run = carry[tid] - own;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int b = 4 * tid + e;
    if (b < nb) s.bcnt[b] = run;
    run += v[e];
  }
  if (tid == 0) s.st->ticket = 0;
}

// Marks the selected positions in index order and sums their gains.
__global__ void __launch_bounds__(kThreads)
sel_mark_kernel(const float* __restrict__ scores, const float* __restrict__ gain, long long n,
                long long chunk, uint8_t* __restrict__ selected, double* net_gain,
                SelScratch s) {
  __shared__ int warp_sums[kThreads / 32];
  __shared__ double dred[kThreads];
  __shared__ int last;
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x;
  const uint32_t T = s.st->prefix;
  const long long k_eq = s.st->k_rem;
  const long long c0 = blockIdx.x * chunk, c1 = min(n, c0 + chunk);
  long long rank0 = s.bcnt[blockIdx.x];               // equal keys in earlier chunks
  double acc = 0.0;
  for (long long base = c0; base < c1; base += kTile) {
    const long long i = base + tid;
    const bool in = i < c1;
    const uint32_t key = in ? score_key(__ldcs(scores + i)) : 0u;
    const bool eq = in && key == T;
    int tile_eq = 0;
    const int r = block_exclusive(eq, warp_sums, &tile_eq);
    const bool sel = in && (key > T || (eq && rank0 + r < k_eq));
    if (in) {
      selected[i] = sel ? 1 : 0;
      if (sel && gain) acc += (double)__ldcs(gain + i);
    }
    rank0 += tile_eq;
  }
  if (!net_gain) return;
  // fixed-order tree: threads, then the chunks in chunk order
  dred[tid] = acc;
  __syncthreads();
  for (int o = kThreads / 2; o > 0; o >>= 1) {
    if (tid < o) dred[tid] += dred[tid + o];
    __syncthreads();
  }
  if (tid == 0) {
    s.bsum[blockIdx.x] = dred[0];
    __threadfence();
    last = atomicAdd(&s.st->ticket, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  double v = 0.0;
  for (int b = tid; b < (int)gridDim.x; b += kThreads) v += __ldcg(s.bsum + b);
  dred[tid] = v;
  __syncthreads();
  for (int o = kThreads / 2; o > 0; o >>= 1) {
    if (tid < o) dred[tid] += dred[tid + o];
    __syncthreads();
  }
  if (tid == 0) {
    *net_gain = dred[0] / (double)n;
    s.st->ticket = 0;
  }
}

}  // namespace

namespace oda_impl {

size_t select_scratch_bytes() {
  return sizeof(SelState) + 256 * sizeof(uint32_t) + kSelectMaxBlocks * sizeof(int) +
         kSelectMaxBlocks * sizeof(double) + 64;
}

oda_status launch_select(oda_ctx* ctx, const float* scores, const float* gain, long long n,
                         long long k, uint8_t* selected, double* net_gain, cudaStream_t st) {
  unsigned char* base = static_cast<unsigned char*>(ctx->select_scratch);
  SelScratch s;
  s.bsum = reinterpret_cast<double*>(base);
  s.st = reinterpret_cast<SelState*>(s.bsum + kSelectMaxBlocks);
  s.hist = reinterpret_cast<uint32_t*>(s.st + 1);
  s.bcnt = reinterpret_cast<int*>(s.hist + 256);
  // chunks of whole tiles, at least 16 tiles each, one block per chunk
  long long blocks = (n + 16LL * kTile - 1) / (16LL * kTile);
  const long long cap = (long long)ctx->num_sms * 4 < kSelectMaxBlocks
                            ? (long long)ctx->num_sms * 4
                            : kSelectMaxBlocks;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  long long chunk = (n + blocks - 1) / blocks;
  chunk = (chunk + kTile - 1) / kTile * kTile;
  blocks = (n + chunk - 1) / chunk;
  const dim3 grid((unsigned)blocks), block(kThreads);
  if (launch_pdl(sel_init_kernel, dim3(1), dim3(kThreads), 0, st, s.st, s.hist, k) !=
      cudaSuccess)
    return ODA_ERR_CUDA;
  if (k > 0) {
    for (int round = 0; round < 4; ++round)
      if (launch_pdl(sel_round_kernel, grid, block, 0, st, scores, n, round, s) != cudaSuccess)
        return ODA_ERR_CUDA;
  }
  if (launch_pdl(sel_count_kernel, grid, block, 0, st, scores, n, chunk, s) != cudaSuccess ||
      launch_pdl(sel_mark_kernel, grid, block, 0, st, scores, gain, n, chunk, selected, net_gain,
                 s) != cudaSuccess)
    return ODA_ERR_CUDA;
  return ODA_OK;
}

}  // namespace oda_impl
