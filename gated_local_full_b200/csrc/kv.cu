// KV commit into the paged cache and the ring, and ring rebuild after prefill.
//
// [SUM] Methodology: the Local pass produces Delta C^L_t, the current token's
// K/V, which every later step can read. [SUM] Efficient Execution: a
// persistent ring KV workspace serves Local, and KV commits are fused across
// layers. Here one launch commits a whole range of layers: each thread moves
// 16 bytes, so a step at batch 1 with 28 layers is one small launch.
#include "oda_internal.cuh"
#include "plan.cuh"

using namespace oda;

namespace {

struct AppendArgs {
  const unsigned char* k_new;
  const unsigned char* v_new;
  const int32_t* seq_lens;
  const int32_t* block_table;
  unsigned char* cache;         // layer 0 base, or null
  unsigned char* ring;          // layer 0 base, or null
  long long cache_layer_bytes;
  long long ring_layer_bytes;
  long long num_blocks;
  int max_blocks;
  int lb, nl, B, hkv, row_bytes;  // row_bytes = d * elem_bytes
  int sink, window, ring_blocks;
  int* err;
  int nblk_append;              // blocks doing the copies; one more writes the plan
  int* plan;                    // Local partition of this step's rows, or null
  PlanIn pin;
  int max_batch;
};

// Byte offset of slot `slot`, K (kv=0) or V (kv=1), inside the (row, head)
// ring tile run; tiles are [2][16][d].
__device__ __forceinline__ long long ring_slot_off(int slot, int kv, int row_bytes) {
  const int tile = slot / ODA_TILE, within = slot % ODA_TILE;
  return ((long long)(tile * 2 + kv) * ODA_TILE + within) * row_bytes;
}

__global__ void append_kernel(const AppendArgs a) {
  extern __shared__ int plan_smem[];
  pdl_wait();
  pdl_launch_dependents();
  if ((int)blockIdx.x == a.nblk_append) {
    // The Local partition depends only on the rows' positions, so it is
    // worked out once here for every Local launch of the step.
    plan_write(a.pin, a.max_batch, a.plan, plan_smem);
    return;
  }
  const int chunks = a.row_bytes / 16;
  const long long total = (long long)a.nl * a.B * a.hkv * 2 * chunks;
  for (long long it = blockIdx.x * (long long)blockDim.x + threadIdx.x; it < total;
       it += (long long)a.nblk_append * blockDim.x) {
    long long r = it;
    const int ch = (int)(r % chunks); r /= chunks;
    const int kv = (int)(r % 2); r /= 2;
    const int g = (int)(r % a.hkv); r /= a.hkv;
    const int b = (int)(r % a.B); r /= a.B;
    const int l = (int)r;                      // 0 .. nl-1, layer lb + l
    const int t = a.seq_lens[b];
    if (t < 1) {
      record_error(a.err, ODA_ERR_BOUNDS);
      continue;
    }
    const unsigned char* src = (kv ? a.v_new : a.k_new) +
                               (((long long)l * a.B + b) * a.hkv + g) * a.row_bytes + ch * 16;
    const uint4 val = *reinterpret_cast<const uint4*>(src);
    if (a.cache) {
      const int bi = (t - 1) / ODA_TILE;
      const int blk = bi < a.max_blocks ? a.block_table[(long long)b * a.max_blocks + bi] : -1;
      if (blk < 0 || (long long)blk >= a.num_blocks) {
        record_error(a.err, ODA_ERR_BOUNDS);
      } else {
        unsigned char* dst = a.cache + (long long)(a.lb + l) * a.cache_layer_bytes +
                             (((long long)blk * a.hkv + g) * 2 + kv) * ODA_TILE * a.row_bytes +
                             (long long)((t - 1) % ODA_TILE) * a.row_bytes + ch * 16;
        *reinterpret_cast<uint4*>(dst) = val;
      }
    }
    if (a.ring) {
      unsigned char* base = a.ring + (long long)(a.lb + l) * a.ring_layer_bytes +
                            ((long long)b * a.hkv + g) * a.ring_blocks * 2 * ODA_TILE * a.row_bytes +
                            ch * 16;
      const int wslot = a.sink + (t - 1) % a.window;
      *reinterpret_cast<uint4*>(base + ring_slot_off(wslot, kv, a.row_bytes)) = val;
      if (t <= a.sink)
        *reinterpret_cast<uint4*>(base + ring_slot_off(t - 1, kv, a.row_bytes)) = val;
    }
  }
}

struct RingInitArgs {
  const int32_t* seq_lens;      // n = positions committed
  const int32_t* block_table;
  const unsigned char* cache;   // layer 0 base
  unsigned char* ring;          // layer 0 base
  long long cache_layer_bytes;
  long long ring_layer_bytes;
  long long num_blocks;
  int max_blocks;
  int lb, nl, B, hkv, row_bytes;
  int sink, window, ring_blocks;
  int* err;
};

// One thread per 16-byte chunk of every (layer, row, head, K/V, slot).
__global__ void ring_init_kernel(const RingInitArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int chunks = a.row_bytes / 16;
  const int slots = a.sink + a.window;
  const long long total = (long long)a.nl * a.B * a.hkv * 2 * slots * chunks;
  for (long long it = blockIdx.x * (long long)blockDim.x + threadIdx.x; it < total;
       it += (long long)gridDim.x * blockDim.x) {
    long long r = it;
    const int ch = (int)(r % chunks); r /= chunks;
    const int slot = (int)(r % slots); r /= slots;
    const int kv = (int)(r % 2); r /= 2;
    const int g = (int)(r % a.hkv); r /= a.hkv;
    const int b = (int)(r % a.B); r /= a.B;
    const int l = (int)r;
    const int n = a.seq_lens[b];
    int p;  // position held by this slot, 0 = none
    if (slot < a.sink) {
      p = (slot + 1 <= n) ? slot + 1 : 0;
    } else {
      const int rr = slot - a.sink;
      // latest position p <= n with (p-1) mod w == rr
      p = (n >= 1 && rr < n) ? n - ((n - 1 - rr) % a.window) : 0;
    }
    uint4 val = make_uint4(0, 0, 0, 0);
    if (p >= 1) {
      const int bi = (p - 1) / ODA_TILE;
      const int blk = bi < a.max_blocks ? a.block_table[(long long)b * a.max_blocks + bi] : -1;
      if (blk < 0 || (long long)blk >= a.num_blocks) {
        record_error(a.err, ODA_ERR_BOUNDS);
      } else {
        const unsigned char* src = a.cache + (long long)(a.lb + l) * a.cache_layer_bytes +
                                   (((long long)blk * a.hkv + g) * 2 + kv) * ODA_TILE * a.row_bytes +
                                   (long long)((p - 1) % ODA_TILE) * a.row_bytes + ch * 16;
        val = *reinterpret_cast<const uint4*>(src);
      }
    } else if (slot < a.sink) {
      continue;  // sink slots beyond n are left untouched
    }
    unsigned char* base = a.ring + (long long)(a.lb + l) * a.ring_layer_bytes +
                          ((long long)b * a.hkv + g) * a.ring_blocks * 2 * ODA_TILE * a.row_bytes +
                          ch * 16;
    *reinterpret_cast<uint4*>(base + ring_slot_off(slot, kv, a.row_bytes)) = val;
  }
}

int grid_for(long long work, int threads, int num_sms) {
  long long g = (work + threads - 1) / threads;
  const long long cap = (long long)num_sms * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

namespace oda_impl {

oda_status launch_append(oda_ctx* ctx, int lb, int le, const void* k_new, const void* v_new,
                         const int32_t* seq_lens, const int32_t* block_table, void* kv_cache,
                         void* ring, int B, cudaStream_t st, int* local_plan) {
  const oda_config& c = ctx->cfg;
  AppendArgs a;
  a.k_new = static_cast<const unsigned char*>(k_new);
  a.v_new = static_cast<const unsigned char*>(v_new);
  a.seq_lens = seq_lens;
  a.block_table = block_table;
  a.cache = static_cast<unsigned char*>(kv_cache);
  a.ring = static_cast<unsigned char*>(ring);
  a.cache_layer_bytes = ctx->lay.cache_layer_elems * ctx->lay.elem_bytes;
  a.ring_layer_bytes = ctx->lay.ring_layer_elems * ctx->lay.elem_bytes;
  a.num_blocks = c.num_blocks;
  a.max_blocks = c.max_blocks_per_seq;
  a.lb = lb;
  a.nl = le - lb;
  a.B = B;
  a.hkv = c.hkv;
  a.row_bytes = c.head_dim * (int)ctx->lay.elem_bytes;
  a.sink = c.sink;
  a.window = c.window;
  a.ring_blocks = (int)ctx->lay.ring_blocks;
  a.err = ctx->err;
  const long long work = (long long)a.nl * B * c.hkv * 2 * (a.row_bytes / 16);
  a.nblk_append = grid_for(work, 256, ctx->num_sms);
  a.plan = local_plan;
  a.max_batch = c.max_batch;
  size_t smem = 0;
  if (local_plan) {
    a.pin.B = B;
    a.pin.count = nullptr;
    a.pin.idx = nullptr;
    a.pin.seq_lens = seq_lens;
    a.pin.hkv = c.hkv;
    a.pin.sink = c.sink;
    a.pin.window = c.window;
    a.pin.max_blocks = c.max_blocks_per_seq;
    a.pin.min_tiles = attn_min_tiles(ctx, true);
    a.pin.grid = ctx->attn_ctas_local;
    a.pin.err = ctx->err;
    a.pin.report = true;
    a.pin.range_lo = nullptr;
    a.pin.range_hi = nullptr;
    smem = (size_t)(4 * c.max_batch + 2) * sizeof(int);
  }
  const int grid = a.nblk_append + (local_plan ? 1 : 0);
  return launch_pdl(append_kernel, dim3(grid), dim3(256), smem, st, a) == cudaSuccess
             ? ODA_OK
             : ODA_ERR_CUDA;
}

oda_status launch_ring_init(oda_ctx* ctx, int lb, int le, const int32_t* seq_lens,
                            const int32_t* block_table, const void* kv_cache, void* ring, int B,
                            cudaStream_t st) {
  const oda_config& c = ctx->cfg;
  RingInitArgs a;
  a.seq_lens = seq_lens;
  a.block_table = block_table;
  a.cache = static_cast<const unsigned char*>(kv_cache);
  a.ring = static_cast<unsigned char*>(ring);
  a.cache_layer_bytes = ctx->lay.cache_layer_elems * ctx->lay.elem_bytes;
  a.ring_layer_bytes = ctx->lay.ring_layer_elems * ctx->lay.elem_bytes;
  a.num_blocks = c.num_blocks;
  a.max_blocks = c.max_blocks_per_seq;
  a.lb = lb;
  a.nl = le - lb;
  a.B = B;
  a.hkv = c.hkv;
  a.row_bytes = c.head_dim * (int)ctx->lay.elem_bytes;
  a.sink = c.sink;
  a.window = c.window;
  a.ring_blocks = (int)ctx->lay.ring_blocks;
  a.err = ctx->err;
  const long long work =
      (long long)a.nl * B * c.hkv * 2 * (c.sink + c.window) * (a.row_bytes / 16);
  return launch_pdl(ring_init_kernel, dim3(grid_for(work, 256, ctx->num_sms)), dim3(256), 0, st,
                    a) == cudaSuccess
             ? ODA_OK
             : ODA_ERR_CUDA;
}

}  // namespace oda_impl
