/*
 * oda.h -- C ABI of the gated local/full decode-attention library (liboda.so).
 *
 * One decode step of On-Demand Attention (ODA) for a batch of requests:
 *   1. commit the new token's K/V (oda_append_kv),
 *   2. attention over the Local access set, in every layer (oda_local_attn),
 *   3. a recall score per request (oda_recall_score),
 *   4. the threshold gate, compacted on the device (oda_gate),
 *   5. attention over the Full access set for the flagged requests only
 *      (oda_full_attn_gated),
 * plus a captured CUDA graph of the whole step whose Full part sits behind a
 * device-side conditional node (oda_step_graph_*).
 *
 * Sources (web pages restated by this library):
 *   [SUM]  "On-Demand Attention (ODA)" summary, picx.dev
 *   [EXPL] "Let models trigger full attention only when recall helps --
 *          On-Demand Attention recall-head gating", learnaivisually explainer
 *
 * Conventions for every entry point
 *   - Positions are 1-indexed. t = seq_lens[b] is the position of the token
 *     being decoded; its K/V must be committed before either attention reads
 *     it, because t belongs to both access sets.
 *   - Pointers named as device pointers must point to device memory of the
 *     context's device; host pointers are marked "host". The caller owns every
 *     buffer it passes. The context owns only its scratch (split partials,
 *     tickets) and a device error word.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream). None synchronizes except
 *     oda_get_device_error, oda_create and oda_destroy.
 *   - One context serves one stream at a time: two calls on different streams
 *     with the same context race on its scratch.
 *   - A returned status covers argument checks and launch errors. Errors the
 *     device finds (an out-of-range block-table entry, a bounded wait that
 *     expired) are recorded in the context's sticky error word; the kernel
 *     skips the bad access and carries on, it never traps.
 *   - Element types: ODA_BF16 (storage bf16, arithmetic fp32) or ODA_F32.
 *     Queries, K/V, rings and outputs share the context's dtype.
 *   - Kernels are launched with programmatic dependent launch: a kernel may
 *     become resident while the previous one on the stream still runs, but
 *     nothing it computes or writes depends on memory read before that kernel
 *     has completed (griddepcontrol.wait), so stream order holds as for plain
 *     launches. Before the wait an attention kernel may read row ids,
 *     lengths and block-table entries (bypassing L1) only to choose which
 *     K/V lines to warm in L2 with bulk prefetches; these are read again
 *     after the wait, and a prefetch returns no value. With the flag
 *     ODA_ATTN_INPUTS_READY the caller states that those inputs and the K/V
 *     were complete earlier, and the kernel also stages its first K/V tiles
 *     before the wait (see that flag).
 */
#ifndef ODA_H
#define ODA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int oda_status;
#define ODA_OK            0
#define ODA_ERR_ARG       1  /* null pointer, negative size, layer out of range */
#define ODA_ERR_SHAPE     2  /* unsupported head_dim/group/batch, sizes over limits */
#define ODA_ERR_DTYPE     3  /* dtype not ODA_BF16 / ODA_F32 */
#define ODA_ERR_CUDA      4  /* a CUDA runtime call failed */
#define ODA_ERR_TIMEOUT   5  /* device: a bounded wait expired */
#define ODA_ERR_BOUNDS    6  /* device: block-table entry, row id or position out of range */
#define ODA_ERR_STATE     7  /* object in the wrong state for the call */

#define ODA_BF16 0
#define ODA_F32  1

#define ODA_MAX_BATCH 1024

typedef void* oda_stream;            /* cudaStream_t */
typedef struct oda_ctx oda_ctx;
typedef struct oda_graph oda_graph;

/* Static shape of one model's attention and its KV storage. */
typedef struct oda_config {
  int layers;              /* L: number of attention layers                          */
  int max_batch;           /* rows the ring and scratch are sized for (<= 1024)      */
  int hq;                  /* query heads                                            */
  int hkv;                 /* KV heads; hq / hkv in {1, 2, 4} (GQA group size)       */
  int head_dim;            /* d in {64, 128}                                         */
  int sink;                /* s: initial positions kept by Local ([SUM] s = 4)       */
  int window;              /* w: recent window of Local ([SUM] w = 2048)             */
  int block_size;          /* tokens per paged KV block; must be 16                  */
  int dtype;               /* ODA_BF16 or ODA_F32                                     */
  int max_blocks_per_seq;  /* columns of the block table                              */
  int64_t num_blocks;      /* physical blocks per layer in the paged cache           */
} oda_config;

/* Sizes and strides (in elements of the context dtype) of the caller-owned
 * KV storage, filled in by oda_layout. */
typedef struct oda_layout_info {
  int64_t tile_elems;          /* one (block, kv_head) tile: [2][16][d], K rows then V rows  */
  int64_t cache_layer_elems;   /* paged cache, one layer: [num_blocks][hkv][2][16][d]        */
  int64_t ring_blocks;         /* ceil((s + w) / 16) 16-slot tiles per (row, kv_head)         */
  int64_t ring_layer_elems;    /* ring, one layer: [max_batch][hkv][ring_blocks][2][16][d]    */
  int64_t elem_bytes;          /* 2 (bf16) or 4 (f32)                                          */
} oda_layout_info;

/*
 * KV layouts (row-major, innermost last), per layer, layers back to back:
 *   paged cache  [num_blocks][hkv][2][16][d]   position p of row b lives in
 *                block block_table[b][(p-1)/16], slot (p-1)%16; index 0 of
 *                the [2] axis is K, 1 is V.
 *   ring         [max_batch][hkv][ring_blocks][2][16][d] viewed as
 *                [ring_blocks*16] slots: slots 0..s-1 hold positions 1..s
 *                (the sinks); slot s + ((p-1) mod w) holds the latest
 *                position p of the recent window ([SUM] "persistent ring KV
 *                workspace for Local").
 *   block table  int32 [B][max_blocks_per_seq] (row stride max_blocks_per_seq).
 */

/* Validate a configuration and fill in the storage layout. Host only; no GPU
 * needed. Returns ODA_ERR_ARG / ODA_ERR_SHAPE / ODA_ERR_DTYPE on a bad config. */
oda_status oda_layout(const oda_config* cfg, oda_layout_info* out);

/* Create a context on the current CUDA device. Validates cfg, allocates the
 * context's scratch (split-KV partials, zeroed tickets, error word) and
 * synchronizes once. *out receives the context. */
oda_status oda_create(const oda_config* cfg, oda_ctx** out);

/* Synchronize the device and free the context's scratch. NULL is accepted. */
oda_status oda_destroy(oda_ctx* ctx);

/*
 * Commit the current token's K/V ([SUM] Methodology: the Local pass returns
 * Delta C^L_t; Efficient Execution: "fused KV commits across layers").
 * One launch covers layers [layer_begin, layer_end).
 *   k_new, v_new  device, [layer_end-layer_begin][B][hkv][d]
 *   seq_lens      device int32 [B], t = position of the token being committed
 *   block_table   device int32 [B][max_blocks_per_seq]
 *   kv_cache      device, paged cache of ALL layers (layer 0 base); NULL skips it
 *   ring          device, ring of ALL layers (layer 0 base); NULL skips it
 * Writes position t into the paged cache and into ring slot s+((t-1) mod w),
 * and also into sink slot t-1 when t <= s. 0 <= B <= max_batch.
 */
oda_status oda_append_kv(oda_ctx* ctx, int layer_begin, int layer_end,
                         const void* k_new, const void* v_new,
                         const int32_t* seq_lens, const int32_t* block_table,
                         void* kv_cache, void* ring, int B, oda_stream stream);

/*
 * Rebuild the ring of layers [layer_begin, layer_end) from the paged cache
 * after a prefill: with n = seq_lens[b] positions committed, the ring receives
 * positions 1..min(s, n) in the sink slots and max(1, n-w+1)..n in the window
 * slots; window slots with no position are zeroed.
 */
oda_status oda_ring_init(oda_ctx* ctx, int layer_begin, int layer_end,
                         const int32_t* seq_lens, const int32_t* block_table,
                         const void* kv_cache, void* ring, int B, oda_stream stream);

/*
 * Flags of oda_local_attn and oda_full_attn_gated.
 *
 * ODA_ATTN_INPUTS_READY: the caller guarantees that the K/V source (ring or
 * paged cache), seq_lens, block_table, idx and count of this call were
 * complete before the previous kernel on `stream` reached its dependency wait
 * -- for example because that kernel is another Local or Full launch of this
 * library, which writes none of them and, like every kernel of this library,
 * waits for its own predecessor before it lets the next launch start. The
 * launch then works out its split and issues its first K/V tile copies into
 * shared memory while the previous kernel is still running; it still reads
 * the queries and writes its outputs and scratch only after that kernel has
 * completed. Without the flag (0) the call makes no assumption beyond stream
 * order. The captured step uses it for every Local and Full launch except the
 * first of each kind.
 */
#define ODA_ATTN_INPUTS_READY 1u

/*
 * Local attention F^L of one layer ([SUM] Methodology / Local-First Decoding):
 * for every row b and query head h,
 *   out[b][h] = sum_{j in S^L_t} softmax_j(q[b][h] . k_j / sqrt(d)) v_j,
 *   S^L_t = {1..min(s,t)} U {max(1,t-w+1)..t},  t = seq_lens[b],
 * with KV head floor(h / (hq/hkv)). Reads only the ring.
 *   q     device [B][hq][d];  ring: all layers (layer 0 base)
 *   out   device [B][hq][d];  lse: device float [B][hq] or NULL
 *         (lse = log sum_j exp(q.k_j / sqrt d), natural log)
 * When B*hkv segments times a cluster size fit one wave of CTAs, each
 * (row, KV head) segment is split over one thread-block cluster and merged in
 * distributed shared memory; otherwise the split is merged through the
 * context's partials. The environment variable ODA_LOCAL_CLUSTER, read by
 * oda_create, caps the cluster size (0: always the partials merge).
 * flags: 0 or ODA_ATTN_INPUTS_READY (see above); other bits: ODA_ERR_ARG.
 */
oda_status oda_local_attn(oda_ctx* ctx, int layer, const void* q,
                          const int32_t* seq_lens, const void* ring,
                          void* out, float* lse, int B, unsigned flags, oda_stream stream);

/*
 * Recall score ([SUM] Methodology, q_t = R_psi(h_{t-1}, E(x_t), h^L_t)):
 *   scores[b] = w2 . GELU(W1 [h_prev[b]; emb[b]; h_local[b]] + b1) + b2,
 * GELU in its erf form. The pages fix the three inputs and their order, not
 * the head's architecture; this library's head is one hidden layer.
 *   h_prev, emb, h_local  device bf16 [B][H]       (H % 64 == 0)
 *   W1                    device bf16 [hidden][3H] row-major (hidden % 128 == 0)
 *   b1, w2                device float [hidden];  b2 by value
 *   scores                device float [B]
 * Runs on the tensor cores (tcgen05, TMEM accumulator). 1 <= B <= 256.
 */
oda_status oda_recall_score(oda_ctx* ctx, const void* h_prev, const void* emb,
                            const void* h_local, int H, const void* W1,
                            const float* b1, const float* w2, float b2, int hidden,
                            float* scores, int B, oda_stream stream);

/*
 * Training objective of the recall head ([SUM] Methodology, training the
 * recall head; an offline step, not part of a decode step). For n positions:
 *   g_t = logp_full[t] - logp_local[t]          access gain (float32),
 *   y_t = T(g_t - lambda),  T(u) = sign(u) log(1 + |u|),
 *   *loss   = (1/n) sum_t Huber_1(q[t] - y_t)   (Huber with transition 1),
 *   *n_full = #{t : g_t > lambda}               (steps where Full pays off).
 *   q, logp_full, logp_local  device float [n] (recall scores; next-token
 *                             log-probabilities under Full and under Local)
 *   loss     device float [1];  n_full  device int32 [1]
 * The gain, its comparison with lambda and the Huber term are formed in
 * float64 from the float32 inputs, T's logarithm in float32 (relative error
 * below 2^-22); the sum is kept in float64 and reduced in a fixed order
 * (deterministic).
 * 1 <= n <= 2^31 - 1, else ODA_ERR_ARG / ODA_ERR_SHAPE. Uses the context's
 * scratch: calls on one context must not overlap.
 */
oda_status oda_recall_loss(oda_ctx* ctx, const float* q, const float* logp_full,
                           const float* logp_local, float lambda, int64_t n, float* loss,
                           int32_t* n_full, oda_stream stream);

/*
 * Selection at a call budget ([SUM] State-Dependent Access Effectiveness: the
 * net gain a policy captures per reference position at a fixed Full-call
 * budget, against random selection; Conclusion: the offline Oracle selects by
 * the true gain). An offline analysis step, not part of a decode step:
 *   selected[t] = 1 for the k positions with the largest scores, else 0;
 *     scores compare as float32, equal scores (+0 and -0 alike) go to the
 *     earlier position, NaN ranks below every number, so the set is unique;
 *     k = floor(budget * n) is the caller's (0 <= k <= n);
 *   *net_gain = (1/n) * sum of gain[t] over the selected t (float64, summed
 *     in a fixed order: the same bits run to run on one GPU).
 *   scores    device float [n]: the recall head's q_t, or the gain itself for
 *             the offline Oracle
 *   gain      device float [n] (access gains g_t), or NULL when net_gain is NULL
 *   selected  device uint8 [n];  net_gain: device double [1] or NULL
 * 1 <= n <= 2^31 - 1, else ODA_ERR_ARG / ODA_ERR_SHAPE. Uses the context's
 * scratch: calls on one context must not overlap.
 */
oda_status oda_select_budget(oda_ctx* ctx, const float* scores, const float* gain, int64_t n,
                             int64_t k, uint8_t* selected, double* net_gain, oda_stream stream);

/*
 * Threshold gate ([SUM] Methodology: recompute with Full iff q_t > theta;
 * default theta = 0) with device-side compaction ([SUM] Efficient Execution:
 * GPU-side conditional execution, no host round trip):
 *   flags[b] = scores[b] > theta (float32, strict; NaN is not flagged),
 *   idx[0..count) = flagged row ids ascending, idx[count..B) = -1,
 *   *count = number of flagged rows.
 * All pointers are device pointers. 0 <= B <= 1024.
 */
oda_status oda_gate(oda_ctx* ctx, const float* scores, float theta, int B,
                    uint8_t* flags, int32_t* idx, int32_t* count, oda_stream stream);

/*
 * Full attention F over S^F_t = {1..t} for the rows idx[0..*count) only
 * ([SUM] Methodology: "if q_t > theta, ODA recomputes with Full"), split
 * over the KV sequence across the whole GPU and merged by log-sum-exp.
 * Rows not listed keep whatever `out` holds (normally the Local output).
 *   q, out       device [B][hq][d];  lse: device float [B][hq] or NULL
 *   kv_cache     paged cache of all layers;  idx, count: device (from oda_gate)
 * *count and idx are read on the device: no host synchronization.
 * flags: 0 or ODA_ATTN_INPUTS_READY (see above); other bits: ODA_ERR_ARG.
 */
oda_status oda_full_attn_gated(oda_ctx* ctx, int layer, const void* q,
                               const int32_t* seq_lens, const int32_t* block_table,
                               const void* kv_cache, const int32_t* idx,
                               const int32_t* count, void* out, float* lse, int B,
                               unsigned flags, oda_stream stream);

/*
 * Range-restricted ("focus") attention: for the rows idx[0..*count), softmax
 * attention over the positions of one region [lo, hi) of the paged history
 * only, reading only that region's K/V. The Declarative Attention pages
 * describe this mode ("<focus>: narrowed to a specific region, reading only
 * that region's KV cache", zhichai.net post, section "Three Attention
 * Modes"; kongchang.com article, section "<focus> Mode: Precise Region
 * Targeting"). For row b with t = seq_lens[b]:
 *   out[b][h] = sum_{j = lo..hi-1} softmax_j(q[b][h] . k_j / sqrt(d)) v_j,
 *   lo = range_lo[b], hi = range_hi[b],  1 <= lo < hi <= t + 1
 * (hi = t + 1 includes the current token; lo = 1, hi = t + 1 is Full).
 * A region outside those bounds records ODA_ERR_BOUNDS and the row is left
 * as `out` holds it. Arguments, layouts and flags as for oda_full_attn_gated;
 * range_lo, range_hi: device int32 [B], indexed by row id like seq_lens.
 */
oda_status oda_range_attn(oda_ctx* ctx, int layer, const void* q, const int32_t* seq_lens,
                          const int32_t* range_lo, const int32_t* range_hi,
                          const int32_t* block_table, const void* kv_cache, const int32_t* idx,
                          const int32_t* count, void* out, float* lse, int B, unsigned flags,
                          oda_stream stream);

/*
 * Full attention for callers that cannot allocate device memory (the pages
 * have no counterpart; this is an interface for integrators). Engines that
 * hand the whole GPU to their own pool allocator at start-up cannot have a
 * library call cudaMalloc later (it fails once the pool holds the memory, or
 * breaks the pool's accounting), and a cudaMalloc on a latency-critical decode
 * loop synchronizes the device. This entry point computes the same function
 * as oda_full_attn_gated, with the same arguments (less `flags`), within the
 * attention tolerance (its persistent grid is capped at 512 CTAs, so its
 * split of the sequence may differ from a context's), but needs no context
 * and allocates nothing: its split partials and tickets live in fixed
 * __device__ arrays inside liboda (1 MiB of partials, 512 segment tickets),
 * held by every GPU that loads the library until the process exits.
 *   cfg     host pointer to the model configuration (as for oda_create)
 *   err     device int32 that receives device-detected errors (ODA_ERR_BOUNDS,
 *           ODA_ERR_TIMEOUT; first error wins), or NULL to drop them into an
 *           internal word
 *   others  as for oda_full_attn_gated
 * Limits: B * hkv <= 512 segments, and (persistent grid + B * hkv) *
 * (hq/hkv) * (head_dim + 2) floats within the 1 MiB partials array; larger
 * calls return ODA_ERR_SHAPE without launching.
 * The first call on a device resolves the arrays' device addresses
 * (cudaGetSymbolAddress, with that device current): make that first call
 * before any stream capture. Every call shares the arrays, which keep the last
 * call's contents; the tickets are cleared on `stream` before each launch.
 * Calls that overlap on the GPU (different streams, or another thread's call
 * in flight) race on the shared arrays and must be serialized by the caller.
 */
oda_status oda_full_attn_gated_static(const oda_config* cfg, int layer, const void* q,
                                      const int32_t* seq_lens, const int32_t* block_table,
                                      const void* kv_cache, const int32_t* idx,
                                      const int32_t* count, void* out, float* lse, int B,
                                      int32_t* err, oda_stream stream);

/* Synchronize `stream`, then return and clear the sticky device error word
 * (ODA_OK if none). Call outside the hot loop. */
oda_status oda_get_device_error(oda_ctx* ctx, oda_stream stream, int* err);

/*
 * Test hook for the bounded-wait path: launches one CTA that waits on a
 * shared-memory barrier nothing will complete, with a limit of timeout_ns.
 * The kernel gives up, records ODA_ERR_TIMEOUT in the error word and returns;
 * the context stays usable.
 */
oda_status oda_selftest_wait_timeout(oda_ctx* ctx, uint64_t timeout_ns, oda_stream stream);

/* ----------------------------------------------------------------------- */
/* One whole decode step                                                    */
/* ----------------------------------------------------------------------- */

typedef struct oda_step_desc {
  int B;                         /* rows this step (<= max_batch)                     */
  const void* q;                 /* [L][B][hq][d] queries (Local and Full)            */
  const void* k_new;             /* [L][B][hkv][d] current token's keys              */
  const void* v_new;             /* [L][B][hkv][d] current token's values            */
  const int32_t* seq_lens;       /* [B] t                                              */
  const int32_t* block_table;    /* [B][max_blocks_per_seq]                            */
  void* kv_cache;                /* paged cache, all layers                            */
  void* ring;                    /* ring, all layers                                   */
  void* out;                     /* [L][B][hq][d] final attention output              */
  float* lse;                    /* [L][B][hq] or NULL                                 */
  /* recall head: set W1 = NULL to skip it */
  const void* h_prev; const void* emb; const void* h_local; int H;
  const void* W1; const float* b1; const float* w2; float b2; int hidden;
  float* scores;                 /* [B] written by the recall head                    */
  const float* gate_scores;      /* [B] scores the gate reads; NULL = `scores`        */
  float theta;
  uint8_t* flags; int32_t* idx; int32_t* count;   /* gate outputs                  */
} oda_step_desc;

/* Issue one step with plain launches: append (all layers, one launch), Local
 * per layer, recall head, gate, then Full per layer (those kernels exit at
 * once when *count == 0). With 8 layers or more, where the head's shape
 * allows (batch <= 64 and its m-tiles times a cluster fit the SMs), its
 * first layer over h_prev and emb,
 * inputs of the step, runs as a kernel of its own before the append; the
 * rest of the head, after the last Local launch, streams the weights of
 * h_local only. */
oda_status oda_step_run(oda_ctx* ctx, const oda_step_desc* d, oda_stream stream);

/* Capture the same step as a CUDA graph in which the Full launches sit in the
 * body of a conditional IF node that the gate kernel sets from *count, so a
 * step with no flagged row launches no Full kernel ([SUM] Efficient
 * Execution: GPU-side conditional CUDA Graphs). The head's first-layer part
 * over h_prev and emb is a branch of its own that starts with the graph and
 * runs beside the Local launches; the rest of the head does not wait for it
 * (a rank of it that finds that part unfinished computes its own share of it
 * instead), so scores can differ between launches in float32 rounding only.
 * The descriptor's pointers are baked in: refill the same buffers between
 * launches. */
oda_status oda_step_graph_create(oda_ctx* ctx, const oda_step_desc* d, oda_graph** out);
oda_status oda_step_graph_launch(oda_graph* g, oda_stream stream);

/* One step of a host-driven decode loop in a single call: copy in_bytes from
 * host memory h_in to device memory d_in (the step's packed inputs), launch
 * the step graph, copy out_bytes from device memory d_out to host memory
 * h_out (the step's results), then wait for the stream. Each copy is one
 * cudaMemcpyAsync on `stream`; host buffers should be pinned for the copies
 * to be asynchronous. in_bytes or out_bytes may be 0 (that copy is skipped).
 * Returns after h_out holds the results; a CUDA error returns ODA_ERR_CUDA.
 * Device-detected errors still go to the context's error word. */
oda_status oda_step_graph_run_io(oda_graph* g, const void* h_in, void* d_in, size_t in_bytes,
                                 const void* d_out, void* h_out, size_t out_bytes,
                                 oda_stream stream);
oda_status oda_step_graph_destroy(oda_graph* g);

/* Library version string. */
const char* oda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ODA_H */
