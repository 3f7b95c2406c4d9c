// Threshold gate with device-side compaction.
//
// [SUM] Methodology / Local-First Decoding: when q_t > theta the step is
// recomputed with Full, otherwise Local is accepted; the default theta is 0.
// [SUM] Efficient Execution: the decision stays on the GPU (conditional CUDA
// graphs), so the flagged rows are compacted here and their count is written
// to device memory; inside a step graph the same kernel also sets the
// conditional node that guards the Full launches.
//
// The comparison is strict and in float32 (no flush-to-zero: a positive
// denormal score is above theta = 0); NaN never compares greater. Flagged ids
// are written in ascending order and the tail of idx is -1.
#include "oda_internal.cuh"

using namespace oda;

namespace {

__global__ void __launch_bounds__(1024)
gate_kernel(const float* __restrict__ scores, float theta, int B, uint8_t* __restrict__ flags,
            int32_t* __restrict__ idx, int32_t* __restrict__ count,
            cudaGraphConditionalHandle cond, int set_cond) {
  __shared__ int warp_counts[32];
  __shared__ int warp_base[33];
  pdl_wait();
  pdl_launch_dependents();
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  bool f = false;
  if (tid < B) {
    const float s = scores[tid];
    f = s > theta;                       // strict, float32, NaN -> false
  }
  const unsigned ballot = __ballot_sync(0xffffffffu, f);
  if (lane == 0) warp_counts[warp] = __popc(ballot);
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    const int nw = (blockDim.x + 31) / 32;
    for (int w = 0; w < nw; ++w) { warp_base[w] = acc; acc += warp_counts[w]; }
    warp_base[32] = acc;
  }
  __syncthreads();
  const int total = warp_base[32];
  if (tid < B) {
    flags[tid] = f ? 1 : 0;
    const int pos = warp_base[warp] + __popc(ballot & ((1u << lane) - 1u));
    if (f) idx[pos] = tid;
    if (tid >= total) idx[tid] = -1;
  }
  if (tid == 0) {
    *count = total;
    if (set_cond) cudaGraphSetConditional(cond, total > 0 ? 1u : 0u);
  }
}

}  // namespace

namespace oda_impl {

oda_status launch_gate(oda_ctx* ctx, const float* scores, float theta, int B, uint8_t* flags,
                       int32_t* idx, int32_t* count, cudaStream_t st,
                       unsigned long long cond_handle, bool set_cond) {
  (void)ctx;
  const int threads = ((B + 31) / 32) * 32 > 0 ? ((B + 31) / 32) * 32 : 32;
  return launch_pdl(gate_kernel, dim3(1), dim3(threads), 0, st, scores, theta, B, flags, idx,
                    count, (cudaGraphConditionalHandle)cond_handle, set_cond ? 1 : 0) ==
                 cudaSuccess
             ? ODA_OK
             : ODA_ERR_CUDA;
}

}  // namespace oda_impl
