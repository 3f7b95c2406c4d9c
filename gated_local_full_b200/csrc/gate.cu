// The threshold gate as a kernel of its own (oda_gate, and the step when the
// recall head does not gate in its last CTA); the routine is in gate.cuh.
#include "gate.cuh"

using namespace oda;

namespace {

__global__ void __launch_bounds__(1024)
gate_kernel(const float* __restrict__ scores, float theta, int B, uint8_t* __restrict__ flags,
            int32_t* __restrict__ idx, int32_t* __restrict__ count,
            cudaGraphConditionalHandle cond, int set_cond) {
  __shared__ int s_ints[65];
  pdl_wait();
  pdl_launch_dependents();
  gate_block(scores, theta, B, flags, idx, count, cond, set_cond, s_ints);
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
