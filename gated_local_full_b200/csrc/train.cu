// The recall head's training objective on the device.
//
// [SUM] Methodology / training the recall head: the access gain of a
// position is g_t = log p^F_t(x_{t+1}) - log p^L_t(x_{t+1}) (how much Full
// attention raises the next token's log-probability); the head regresses
// y_t = T(g_t - lambda) with T(u) = sign(u) log(1 + |u|), under a Huber loss
// with transition point 1; a step pays for Full exactly when g_t > lambda.
// For n positions this kernel returns the mean loss and that count.
//
// The work is one pass over three float arrays (12 bytes per position), so it
// is bound by HBM: six CTAs per SM stream them with 16-byte loads. The gain
// f - l, its comparison with lambda (which decides the count) and the Huber
// term are formed in float64; T's logarithm is taken in float32 (relative
// error below 2^-22; float64 logarithms would make the pass compute-bound on
// this GPU). Each thread keeps a float64 sum, blocks reduce in a fixed order,
// and the last block to take the ticket adds the block sums with a
// fixed-order tree, so the result is the same run to run.
#include "oda_internal.cuh"

using namespace oda;

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ double signed_log1p(double u) {
  return copysign((double)log1pf((float)fabs(u)), u);
}

__device__ __forceinline__ double huber1(double r) {
  const double a = fabs(r);
  return a <= 1.0 ? 0.5 * a * a : a - 0.5;
}

// One position: the count of g > lambda and the Huber term.
__device__ __forceinline__ void position(float qv, float f, float l, double lam, double& s,
                                         int& c) {
  const double g = (double)f - (double)l;            // access gain
  c += g > lam ? 1 : 0;                              // Full pays off (strict)
  s += huber1((double)qv - signed_log1p(g - lam));
}

__global__ void __launch_bounds__(kThreads)
recall_loss_kernel(const float* __restrict__ q, const float* __restrict__ lpf,
                   const float* __restrict__ lpl, float lam, long long n, int vec,
                   double* __restrict__ bsum, int* __restrict__ bcnt, int* __restrict__ ticket,
                   float* __restrict__ loss, int32_t* __restrict__ n_full) {
  __shared__ double ssum[kThreads / 32];
  __shared__ int scnt[kThreads / 32];
  __shared__ double tsum[kThreads];
  __shared__ long long tcnt[kThreads];
  __shared__ int last;
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long stride = (long long)gridDim.x * kThreads;
  const long long first = blockIdx.x * (long long)kThreads + tid;
  const double dlam = (double)lam;
  double s = 0.0;
  int c = 0;
  // 16-byte loads of four positions of each array, streamed past L1/L2
  const long long n4 = vec ? n / 4 : 0;
  const float4* q4 = reinterpret_cast<const float4*>(q);
  const float4* f4 = reinterpret_cast<const float4*>(lpf);
  const float4* l4 = reinterpret_cast<const float4*>(lpl);
#pragma unroll 2
  for (long long i = first; i < n4; i += stride) {
    const float4 a = __ldcs(q4 + i), f = __ldcs(f4 + i), l = __ldcs(l4 + i);
    position(a.x, f.x, l.x, dlam, s, c);
    position(a.y, f.y, l.y, dlam, s, c);
    position(a.z, f.z, l.z, dlam, s, c);
    position(a.w, f.w, l.w, dlam, s, c);
  }
  for (long long i = n4 * 4 + first; i < n; i += stride) position(q[i], lpf[i], lpl[i], dlam, s, c);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
  }
  if (lane == 0) { ssum[warp] = s; scnt[warp] = c; }
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    int k = 0;
    for (int w = 0; w < kThreads / 32; ++w) { t += ssum[w]; k += scnt[w]; }
    bsum[blockIdx.x] = t;
    bcnt[blockIdx.x] = k;
    __threadfence();
    last = atomicAdd(ticket, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  // the block sums: thread i adds blocks i, i + kThreads, ... in order, then a
  // fixed-order tree over the threads
  double t = 0.0;
  long long k = 0;
  for (int b = tid; b < (int)gridDim.x; b += kThreads) {
    t += __ldcg(bsum + b);
    k += __ldcg(bcnt + b);
  }
  tsum[tid] = t;
  tcnt[tid] = k;
  __syncthreads();
  for (int o = kThreads / 2; o > 0; o >>= 1) {
    if (tid < o) {
      tsum[tid] += tsum[tid + o];
      tcnt[tid] += tcnt[tid + o];
    }
    __syncthreads();
  }
  if (tid == 0) {
    *loss = (float)(tsum[0] / (double)n);
    *n_full = (int32_t)tcnt[0];
    *ticket = 0;
  }
}

}  // namespace

namespace oda_impl {

oda_status launch_recall_loss(oda_ctx* ctx, const float* q, const float* lpf, const float* lpl,
                              float lam, long long n, float* loss, int32_t* n_full,
                              cudaStream_t st) {
  long long grid = (n + kThreads * 8 - 1) / (kThreads * 8);   // >= 8 positions per thread
  const long long cap = (long long)ctx->num_sms * 6;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  double* bsum = reinterpret_cast<double*>(ctx->train_scratch);
  int* bcnt = reinterpret_cast<int*>(bsum + kTrainMaxBlocks);
  int* ticket = bcnt + kTrainMaxBlocks;
  if (grid > kTrainMaxBlocks) grid = kTrainMaxBlocks;
  const int vec = ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(lpf) |
                    reinterpret_cast<uintptr_t>(lpl)) & 15u) == 0;
  return launch_pdl(recall_loss_kernel, dim3((unsigned)grid), dim3(kThreads), 0, st, q, lpf, lpl,
                    lam, n, vec, bsum, bcnt, ticket, loss, n_full) == cudaSuccess
             ? ODA_OK
             : ODA_ERR_CUDA;
}

}  // namespace oda_impl
