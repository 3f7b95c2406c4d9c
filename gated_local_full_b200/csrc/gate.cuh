// Threshold gate with device-side compaction, as a block-level routine shared
// by the gate kernel and the recall head's last CTA (which gates inside the
// captured step, so the decision needs no separate launch).
//
// [SUM] Methodology / Local-First Decoding: when q_t > theta the step is
// recomputed with Full, otherwise Local is accepted; the default theta is 0.
// [SUM] Efficient Execution: the decision stays on the GPU (conditional CUDA
// graphs): the flagged rows are compacted and counted in device memory, and
// inside a step graph the same code sets the conditional node that guards the
// Full launches.
//
// The comparison is strict and in float32 (no flush-to-zero: a positive
// denormal score is above theta = 0); NaN never compares greater. Flagged ids
// are written in ascending order and the tail of idx is -1.
//
// The gate sets the step graph's condition on every launch (1 when a row is
// flagged, else 0): the handle carries no default, whose reset at each graph
// launch measured slower than this store.
#pragma once

#include "oda_internal.cuh"

namespace oda {

// Every thread of the block calls it (it holds __syncthreads); needs
// B <= blockDim.x, blockDim.x a multiple of 32 and at most 1024, and 65 ints
// of shared memory.
__device__ __forceinline__ void gate_block(const float* scores, float theta, int B, uint8_t* flags,
                                           int32_t* idx, int32_t* count,
                                           cudaGraphConditionalHandle cond, int set_cond,
                                           int* s_ints) {
  int* warp_counts = s_ints;        // [32]
  int* warp_base = s_ints + 32;     // [33]
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

// The same gate for B <= 32 rows by one warp (all 32 lanes call it; lane i
// holds row i's score in v, lanes >= B are ignored): no shared memory and no
// block barrier.
__device__ __forceinline__ void gate_warp(float v, int B, float theta, uint8_t* flags,
                                          int32_t* idx, int32_t* count,
                                          cudaGraphConditionalHandle cond, int set_cond) {
  const int lane = threadIdx.x & 31;
  const bool f = lane < B && v > theta;  // strict, float32, NaN -> false
  const unsigned ballot = __ballot_sync(0xffffffffu, f);
  const int total = __popc(ballot);
  if (lane < B) {
    flags[lane] = f ? 1 : 0;
    if (f) idx[__popc(ballot & ((1u << lane) - 1u))] = lane;
    if (lane >= total) idx[lane] = -1;
  }
  if (lane == 0) {
    *count = total;
    if (set_cond) cudaGraphSetConditional(cond, total > 0 ? 1u : 0u);
  }
}

}  // namespace oda
