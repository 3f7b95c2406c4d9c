// C ABI of liboda: argument checks, the context, the device error word.
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "oda_internal.cuh"
#include "plan.cuh"

using namespace oda;

namespace {

oda_status check_config(const oda_config* c) {
  if (!c) return ODA_ERR_ARG;
  if (c->dtype != ODA_BF16 && c->dtype != ODA_F32) return ODA_ERR_DTYPE;
  if (c->layers < 1 || c->max_batch < 1 || c->hq < 1 || c->hkv < 1 || c->sink < 0 ||
      c->window < 1 || c->max_blocks_per_seq < 1 || c->num_blocks < 1)
    return ODA_ERR_ARG;
  if (c->max_batch > ODA_MAX_BATCH) return ODA_ERR_SHAPE;
  if (c->block_size != ODA_TILE) return ODA_ERR_SHAPE;
  if (c->head_dim != 64 && c->head_dim != 128) return ODA_ERR_SHAPE;
  if (c->hq % c->hkv != 0) return ODA_ERR_SHAPE;
  const int g = c->hq / c->hkv;
  if (g != 1 && g != 2 && g != 4) return ODA_ERR_SHAPE;
  // tile indices are 32-bit inside the kernels
  const long long ring_blocks = ((long long)c->sink + c->window + ODA_TILE - 1) / ODA_TILE;
  const long long max_tiles = (long long)c->max_batch * c->hkv *
                              (c->max_blocks_per_seq > ring_blocks ? c->max_blocks_per_seq : ring_blocks);
  if (max_tiles >= (1ll << 31) || (long long)c->sink + c->window >= (1ll << 30)) return ODA_ERR_SHAPE;
  return ODA_OK;
}

oda_status check_batch(const oda_ctx* ctx, int B) {
  if (B < 0) return ODA_ERR_ARG;
  if (B > ctx->cfg.max_batch) return ODA_ERR_SHAPE;
  return ODA_OK;
}

__global__ void wait_selftest_kernel(uint64_t timeout_ns, int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the bounded wait must give up
  if (threadIdx.x == 0 && !mbar_wait_bounded(smem_addr(&bar), 0u, timeout_ns))
    record_error(err, ODA_ERR_TIMEOUT);
}

}  // namespace

namespace oda {

namespace attr_cache {
struct SmemLimit {
  int dev;
  const void* fn;
  size_t bytes;
};
struct OccEntry {
  int dev;
  const void* fn;
  int threads;
  size_t smem;
  int occ;
};
std::mutex g_attr_mu;
std::vector<SmemLimit> g_smem_limits;
std::vector<OccEntry> g_occ;
}  // namespace attr_cache
using namespace attr_cache;

cudaError_t raise_smem_limit(const void* fn, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  for (SmemLimit& l : g_smem_limits) {
    if (l.dev == dev && l.fn == fn) {
      if (l.bytes >= bytes) return cudaSuccess;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
      if (e == cudaSuccess) l.bytes = bytes;
      return e;
    }
  }
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) g_smem_limits.push_back(SmemLimit{dev, fn, bytes});
  return e;
}

cudaError_t occupancy_cached(int* occ, const void* fn, int threads, size_t smem) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  for (const OccEntry& o : g_occ) {
    if (o.dev == dev && o.fn == fn && o.threads == threads && o.smem == smem) {
      *occ = o.occ;
      return cudaSuccess;
    }
  }
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ, fn, threads, smem);
  if (e == cudaSuccess) g_occ.push_back(OccEntry{dev, fn, threads, smem, *occ});
  return e;
}

}  // namespace oda

namespace oda_impl {
oda_status launch_wait_selftest(oda_ctx* ctx, uint64_t timeout_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(timeout_ns, ctx->err);
  return cudaGetLastError() == cudaSuccess ? ODA_OK : ODA_ERR_CUDA;
}
}  // namespace oda_impl

extern "C" {

const char* oda_version(void) { return "oda-b200 0.1 (sm_100a)"; }

oda_status oda_layout(const oda_config* cfg, oda_layout_info* out) {
  if (!out) return ODA_ERR_ARG;
  const oda_status s = check_config(cfg);
  if (s != ODA_OK) return s;
  const int64_t d = cfg->head_dim;
  out->elem_bytes = cfg->dtype == ODA_BF16 ? 2 : 4;
  out->tile_elems = 2 * ODA_TILE * d;
  out->cache_layer_elems = cfg->num_blocks * cfg->hkv * out->tile_elems;
  out->ring_blocks = ((int64_t)cfg->sink + cfg->window + ODA_TILE - 1) / ODA_TILE;
  out->ring_layer_elems = (int64_t)cfg->max_batch * cfg->hkv * out->ring_blocks * out->tile_elems;
  return ODA_OK;
}

oda_status oda_create(const oda_config* cfg, oda_ctx** out) {
  if (!out) return ODA_ERR_ARG;
  *out = nullptr;
  oda_layout_info lay;
  oda_status s = oda_layout(cfg, &lay);
  if (s != ODA_OK) return s;
  oda_ctx* ctx = static_cast<oda_ctx*>(calloc(1, sizeof(oda_ctx)));
  if (!ctx) return ODA_ERR_ARG;
  ctx->cfg = *cfg;
  ctx->lay = lay;
  if (cudaGetDevice(&ctx->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device) !=
          cudaSuccess) {
    free(ctx);
    return ODA_ERR_CUDA;
  }
  s = oda_impl::attn_setup(ctx);
  if (s == ODA_OK) {
    const int g = cfg->hq / cfg->hkv;
    const int ctas = ctx->attn_ctas_local > ctx->attn_ctas_full ? ctx->attn_ctas_local
                                                                : ctx->attn_ctas_full;
    ctx->max_parts = ctas + cfg->max_batch * cfg->hkv;
    const size_t pbytes = (size_t)ctx->max_parts * g * (cfg->head_dim + 2) * sizeof(float);
    if (cudaMalloc(&ctx->partials, pbytes) != cudaSuccess ||
        cudaMalloc(&ctx->tickets, 2 * (size_t)cfg->max_batch * cfg->hkv * sizeof(int)) !=
            cudaSuccess ||
        cudaMalloc(&ctx->err, sizeof(int)) != cudaSuccess ||
        cudaMemset(ctx->tickets, 0, 2 * (size_t)cfg->max_batch * cfg->hkv * sizeof(int)) !=
            cudaSuccess ||
        cudaMemset(ctx->err, 0, sizeof(int)) != cudaSuccess)
      s = ODA_ERR_CUDA;
  }
  if (s == ODA_OK &&
      cudaMalloc(&ctx->plan_local,
                 PlanLayout::ints(cfg->max_batch, ctx->attn_ctas_local) * sizeof(int)) !=
          cudaSuccess)
    s = ODA_ERR_CUDA;
  if (s == ODA_OK) s = oda_impl::recall_setup(ctx);
  if (s == ODA_OK) {
    // recall-loss reduction: block sums (f64), block counts (i32), one ticket
    const size_t tb = (size_t)oda::kTrainMaxBlocks * (sizeof(double) + sizeof(int)) + 16;
    if (cudaMalloc(&ctx->train_scratch, tb) != cudaSuccess ||
        cudaMemset(ctx->train_scratch, 0, tb) != cudaSuccess)
      s = ODA_ERR_CUDA;
  }
  if (s == ODA_OK) {
    const size_t sb = oda_impl::select_scratch_bytes();
    if (cudaMalloc(&ctx->select_scratch, sb) != cudaSuccess ||
        cudaMemset(ctx->select_scratch, 0, sb) != cudaSuccess)
      s = ODA_ERR_CUDA;
  }
  if (s == ODA_OK && cudaDeviceSynchronize() != cudaSuccess) s = ODA_ERR_CUDA;
  if (s != ODA_OK) {
    oda_destroy(ctx);
    return s;
  }
  *out = ctx;
  return ODA_OK;
}

oda_status oda_destroy(oda_ctx* ctx) {
  if (!ctx) return ODA_OK;
  cudaDeviceSynchronize();
  cudaFree(ctx->partials);
  cudaFree(ctx->tickets);
  cudaFree(ctx->err);
  cudaFree(ctx->recall_partials);
  cudaFree(ctx->recall_tickets);
  cudaFree(ctx->recall_pre);
  cudaFree(ctx->plan_local);
  cudaFree(ctx->train_scratch);
  cudaFree(ctx->select_scratch);
  free(ctx);
  return ODA_OK;
}

oda_status oda_append_kv(oda_ctx* ctx, int layer_begin, int layer_end, const void* k_new,
                         const void* v_new, const int32_t* seq_lens, const int32_t* block_table,
                         void* kv_cache, void* ring, int B, oda_stream stream) {
  if (!ctx) return ODA_ERR_ARG;
  oda_status s = check_batch(ctx, B);
  if (s != ODA_OK) return s;
  if (layer_begin < 0 || layer_end > ctx->cfg.layers || layer_begin > layer_end) return ODA_ERR_ARG;
  if (B == 0 || layer_begin == layer_end || (!kv_cache && !ring)) return ODA_OK;
  if (!k_new || !v_new || !seq_lens || (kv_cache && !block_table)) return ODA_ERR_ARG;
  return oda_impl::launch_append(ctx, layer_begin, layer_end, k_new, v_new, seq_lens, block_table,
                                 kv_cache, ring, B, static_cast<cudaStream_t>(stream));
}

oda_status oda_ring_init(oda_ctx* ctx, int layer_begin, int layer_end, const int32_t* seq_lens,
                         const int32_t* block_table, const void* kv_cache, void* ring, int B,
                         oda_stream stream) {
  if (!ctx) return ODA_ERR_ARG;
  oda_status s = check_batch(ctx, B);
  if (s != ODA_OK) return s;
  if (layer_begin < 0 || layer_end > ctx->cfg.layers || layer_begin > layer_end) return ODA_ERR_ARG;
  if (B == 0 || layer_begin == layer_end) return ODA_OK;
  if (!seq_lens || !block_table || !kv_cache || !ring) return ODA_ERR_ARG;
  return oda_impl::launch_ring_init(ctx, layer_begin, layer_end, seq_lens, block_table, kv_cache,
                                    ring, B, static_cast<cudaStream_t>(stream));
}

oda_status oda_local_attn(oda_ctx* ctx, int layer, const void* q, const int32_t* seq_lens,
                          const void* ring, void* out, float* lse, int B, unsigned flags,
                          oda_stream stream) {
  if (!ctx) return ODA_ERR_ARG;
  oda_status s = check_batch(ctx, B);
  if (s != ODA_OK) return s;
  if (layer < 0 || layer >= ctx->cfg.layers) return ODA_ERR_ARG;
  if (flags & ~ODA_ATTN_INPUTS_READY) return ODA_ERR_ARG;
  if (B == 0) return ODA_OK;
  if (!q || !seq_lens || !ring || !out) return ODA_ERR_ARG;
  return oda_impl::launch_attn(ctx, true, layer, q, seq_lens, ring, nullptr, nullptr, nullptr, out,
                               lse, B, static_cast<cudaStream_t>(stream), nullptr,
                               (flags & ODA_ATTN_INPUTS_READY) != 0);
}

oda_status oda_full_attn_gated(oda_ctx* ctx, int layer, const void* q, const int32_t* seq_lens,
                               const int32_t* block_table, const void* kv_cache,
                               const int32_t* idx, const int32_t* count, void* out, float* lse,
                               int B, unsigned flags, oda_stream stream) {
  if (!ctx) return ODA_ERR_ARG;
  oda_status s = check_batch(ctx, B);
  if (s != ODA_OK) return s;
  if (layer < 0 || layer >= ctx->cfg.layers) return ODA_ERR_ARG;
  if (flags & ~ODA_ATTN_INPUTS_READY) return ODA_ERR_ARG;
  if (B == 0) return ODA_OK;
  if (!q || !seq_lens || !block_table || !kv_cache || !idx || !count || !out) return ODA_ERR_ARG;
  return oda_impl::launch_attn(ctx, false, layer, q, seq_lens, kv_cache, block_table, idx, count,
                               out, lse, B, static_cast<cudaStream_t>(stream), nullptr,
                               (flags & ODA_ATTN_INPUTS_READY) != 0);
}

oda_status oda_range_attn(oda_ctx* ctx, int layer, const void* q, const int32_t* seq_lens,
                          const int32_t* range_lo, const int32_t* range_hi,
                          const int32_t* block_table, const void* kv_cache, const int32_t* idx,
                          const int32_t* count, void* out, float* lse, int B, unsigned flags,
                          oda_stream stream) {
  if (!ctx) return ODA_ERR_ARG;
  oda_status s = check_batch(ctx, B);
  if (s != ODA_OK) return s;
  if (layer < 0 || layer >= ctx->cfg.layers) return ODA_ERR_ARG;
  if (flags & ~ODA_ATTN_INPUTS_READY) return ODA_ERR_ARG;
  if (B == 0) return ODA_OK;
  if (!q || !seq_lens || !range_lo || !range_hi || !block_table || !kv_cache || !idx || !count ||
      !out)
    return ODA_ERR_ARG;
  return oda_impl::launch_attn(ctx, false, layer, q, seq_lens, kv_cache, block_table, idx, count,
                               out, lse, B, static_cast<cudaStream_t>(stream), nullptr,
                               (flags & ODA_ATTN_INPUTS_READY) != 0, range_lo, range_hi);
}

oda_status oda_recall_score(oda_ctx* ctx, const void* h_prev, const void* emb,
                            const void* h_local, int H, const void* W1, const float* b1,
                            const float* w2, float b2, int hidden, float* scores, int B,
                            oda_stream stream) {
  if (!ctx) return ODA_ERR_ARG;
  if (B < 0) return ODA_ERR_ARG;
  if (B == 0) return ODA_OK;
  if (!h_prev || !emb || !h_local || !W1 || !b1 || !w2 || !scores) return ODA_ERR_ARG;
  if (H < 1 || hidden < 1) return ODA_ERR_ARG;
  return oda_impl::launch_recall(ctx, h_prev, emb, h_local, H, W1, b1, w2, b2, hidden, scores, B,
                                 static_cast<cudaStream_t>(stream));
}

oda_status oda_recall_loss(oda_ctx* ctx, const float* q, const float* logp_full,
                           const float* logp_local, float lambda, int64_t n, float* loss,
                           int32_t* n_full, oda_stream stream) {
  if (!ctx || !q || !logp_full || !logp_local || !loss || !n_full || n < 1) return ODA_ERR_ARG;
  if (n > (int64_t)INT32_MAX) return ODA_ERR_SHAPE;
  return oda_impl::launch_recall_loss(ctx, q, logp_full, logp_local, lambda, (long long)n, loss,
                                      n_full, static_cast<cudaStream_t>(stream));
}

oda_status oda_select_budget(oda_ctx* ctx, const float* scores, const float* gain, int64_t n,
                             int64_t k, uint8_t* selected, double* net_gain, oda_stream stream) {
  if (!ctx || !scores || !selected || n < 1 || k < 0 || k > n) return ODA_ERR_ARG;
  if (net_gain && !gain) return ODA_ERR_ARG;
  if (n > (int64_t)INT32_MAX) return ODA_ERR_SHAPE;
  return oda_impl::launch_select(ctx, scores, gain, (long long)n, (long long)k, selected, net_gain,
                                 static_cast<cudaStream_t>(stream));
}

oda_status oda_gate(oda_ctx* ctx, const float* scores, float theta, int B, uint8_t* flags,
                    int32_t* idx, int32_t* count, oda_stream stream) {
  if (!ctx) return ODA_ERR_ARG;
  if (B < 0) return ODA_ERR_ARG;
  if (B > ODA_MAX_BATCH) return ODA_ERR_SHAPE;
  if (!count || (B > 0 && (!scores || !flags || !idx))) return ODA_ERR_ARG;
  return oda_impl::launch_gate(ctx, scores, theta, B, flags, idx, count,
                               static_cast<cudaStream_t>(stream), 0ull, false);
}

oda_status oda_get_device_error(oda_ctx* ctx, oda_stream stream, int* err) {
  if (!ctx || !err) return ODA_ERR_ARG;
  *err = ODA_OK;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ODA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ctx->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ODA_ERR_CUDA;
  if (v != 0 && cudaMemset(ctx->err, 0, sizeof(int)) != cudaSuccess) return ODA_ERR_CUDA;
  *err = v;
  return ODA_OK;
}

oda_status oda_selftest_wait_timeout(oda_ctx* ctx, uint64_t timeout_ns, oda_stream stream) {
  if (!ctx) return ODA_ERR_ARG;
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return ODA_ERR_ARG;
  return oda_impl::launch_wait_selftest(ctx, timeout_ns, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
