// Internal definitions shared by liboda's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

#include "../../include/oda.h"

#define ODA_TILE 16  // tokens per paged block / ring tile

struct oda_ctx {
  oda_config cfg;
  oda_layout_info lay;
  int device;
  int num_sms;
  int attn_ctas_local;       // persistent grid of the Local attention kernel
  int attn_ctas_full;        // persistent grid of the Full attention kernel
  int max_parts;             // capacity of the partials buffer (in partials)
  float* partials;           // [max_parts][G][d+2]
  int* tickets;              // [2][max_batch * hkv]: merge tickets, dynamic tile counters;
                             // zero between launches
  int* err;                  // device sticky error word
  int* recall_tickets;       // recall-head split reduction counters
  float* recall_partials;    // recall-head split partials
  int recall_parts_cap;      // capacity of recall_partials in floats
  float* recall_pre;         // the step's first-layer prefix over h_{t-1}, E(x_t): [hidden][N]
  int recall_cluster_max;    // largest cluster for the recall head's split-K (0: none)
  void* train_scratch;       // recall-loss block sums [kTrainMaxBlocks] f64, counts, ticket
  int* plan_local;           // partition shared by a step's Local launches
  int local_cluster_max;     // largest cluster for the cluster-merge Local kernel (0: none)
  int local_wide_cluster_max;  // the same for its one-tile-per-warp shape
  int local_wide_ctas;       // CTAs of that shape one wave holds
  size_t local_last_smem;    // dynamic shared memory of the last Local launch issued
  void* select_scratch;      // budgeted selection: chunk sums, search state, histogram, counts
};

// The gate run by the recall head's last CTA inside a captured step.
struct RecallGate {
  const float* scores;       // scores to compare; null: the head's own output
  float theta;
  uint8_t* flags;
  int32_t* idx;
  int32_t* count;
  unsigned long long cond;   // conditional-node handle
  bool set_cond;
};

namespace oda {

constexpr int kTrainMaxBlocks = 1024;   // blocks of the recall-loss reduction
constexpr int kSelectMaxBlocks = 1024;  // blocks (chunks) of the budgeted selection

// ----------------------------------------------------------------- host utils
#define ODA_CUDA_TRY(expr)                                   \
  do {                                                       \
    cudaError_t _e = (expr);                                 \
    if (_e != cudaSuccess) return ODA_ERR_CUDA;              \
  } while (0)

inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// A kernel's dynamic shared-memory limit is one value per (function, device)
// for the whole process, shared by every context and by the allocation-free
// entry point. raise_smem_limit sets it to at least `bytes` on the current
// device and never lowers it, so one caller sized for a small batch cannot
// break another's launches. occupancy_cached returns the resident blocks per
// SM of `fn` at `threads` threads and `smem` bytes, asked of the runtime once
// per (device, function, threads, smem). Both are thread safe.
cudaError_t raise_smem_limit(const void* fn, size_t bytes);
cudaError_t occupancy_cached(int* occ, const void* fn, int threads, size_t smem);

// ------------------------------------------------------------ device helpers
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of barrier `bar` to complete, giving up after
// limit_ns nanoseconds of wall time. Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// One bulk (non-tensor) global->shared copy completing on an mbarrier.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// Thread-block-cluster barrier halves (every thread of every CTA of the
// cluster takes part). arrive: release by default, or relaxed; wait: acquire.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// Bulk prefetch of global memory into L2 (no completion to wait for).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Ticket increment with acquire-release semantics at GPU scope: the writes
// the block made before a __syncthreads are released with it, and a block
// that takes the last ticket acquires every earlier taker's writes (its other
// threads read them after a __syncthreads), with no separate fences.
__device__ __forceinline__ int ticket_add(int* p, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Asynchronous global -> shared copies that hold no registers (cp.async):
// 16 bytes through L2 only, or 4 bytes; wait_all waits for this thread's.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// bf16 pair (packed in a 32-bit word, low half first) -> two floats, exactly.
__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xFFFF0000u);
}

// Programmatic dependent launch: a kernel launched with
// launch_pdl may be scheduled while its predecessor in the stream is still
// running; pdl_wait() blocks until that predecessor has completed and its
// writes are visible, so every kernel calls it before reading any input.
// pdl_launch_dependents() lets the next kernel start being scheduled.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace oda

// Host-side entry points implemented per translation unit (C++ linkage).
namespace oda_impl {
oda_status launch_append(oda_ctx* ctx, int lb, int le, const void* k_new, const void* v_new,
                         const int32_t* seq_lens, const int32_t* block_table, void* kv_cache,
                         void* ring, int B, cudaStream_t st, int* local_plan = nullptr);
oda_status launch_ring_init(oda_ctx* ctx, int lb, int le, const int32_t* seq_lens,
                            const int32_t* block_table, const void* kv_cache, void* ring, int B,
                            cudaStream_t st);
oda_status launch_attn(oda_ctx* ctx, bool ring_mode, int layer, const void* q,
                       const int32_t* seq_lens, const void* kv, const int32_t* block_table,
                       const int32_t* idx, const int32_t* count, void* out, float* lse, int B,
                       cudaStream_t st, const int* plan = nullptr, bool early = false,
                       const int32_t* range_lo = nullptr, const int32_t* range_hi = nullptr);
int attn_min_tiles(oda_ctx* ctx, bool ring_mode);
oda_status attn_setup(oda_ctx* ctx);
oda_status launch_gate(oda_ctx* ctx, const float* scores, float theta, int B, uint8_t* flags,
                       int32_t* idx, int32_t* count, cudaStream_t st,
                       unsigned long long cond_handle, bool set_cond);
oda_status launch_recall(oda_ctx* ctx, const void* h_prev, const void* emb, const void* h_local,
                         int H, const void* W1, const float* b1, const float* w2, float b2,
                         int hidden, float* scores, int B, cudaStream_t st, bool early = false,
                         const RecallGate* gate = nullptr, bool* gate_fused = nullptr,
                         bool after_prefix = false);
// Whether a step splits the head's first layer: the prefix kernel over the
// K range of h_{t-1} and E(x_t) (launch_recall_prefix, free to run beside the
// Local launches) and then the cluster kernel over h^L_t only
// (launch_recall with after_prefix).
bool recall_split(const oda_ctx* ctx, int B, int H, int hidden);
oda_status launch_recall_prefix(oda_ctx* ctx, const void* h_prev, const void* emb, int H,
                                const void* W1, const float* b1, int hidden, int B,
                                cudaStream_t st);
oda_status recall_setup(oda_ctx* ctx);
oda_status launch_recall_loss(oda_ctx* ctx, const float* q, const float* lpf, const float* lpl,
                              float lam, long long n, float* loss, int32_t* n_full,
                              cudaStream_t st);
oda_status launch_wait_selftest(oda_ctx* ctx, uint64_t timeout_ns, cudaStream_t st);
size_t select_scratch_bytes();
oda_status launch_select(oda_ctx* ctx, const float* scores, const float* gain, long long n,
                         long long k, uint8_t* selected, double* net_gain, cudaStream_t st);
}  // namespace oda_impl
