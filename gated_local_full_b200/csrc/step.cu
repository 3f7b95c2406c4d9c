// One decode step: plain launches, or a CUDA graph with a device-side IF node.
//
// [SUM] Methodology / Local-First Decoding gives the order: commit the token,
// run Local, score, and recompute with Full only if q_t > theta.
// [SUM] Efficient Execution: the runtime uses GPU-side conditional CUDA
// graphs, so the decision never returns to the host. Here the gate kernel
// writes the IF node's condition (count > 0); with no flagged row the graph
// launches no Full kernel at all.
#include <stdlib.h>

#include "oda_internal.cuh"

struct oda_graph {
  oda_ctx* ctx;
  cudaGraph_t graph;
  cudaGraphExec_t exec;
};

namespace {

oda_status check_desc(const oda_ctx* ctx, const oda_step_desc* d) {
  if (!ctx || !d) return ODA_ERR_ARG;
  if (d->B < 1) return ODA_ERR_ARG;
  if (d->B > ctx->cfg.max_batch) return ODA_ERR_SHAPE;
  if (!d->q || !d->k_new || !d->v_new || !d->seq_lens || !d->block_table || !d->kv_cache ||
      !d->ring || !d->out || !d->flags || !d->idx || !d->count)
    return ODA_ERR_ARG;
  if (d->W1 && (!d->h_prev || !d->emb || !d->h_local || !d->b1 || !d->w2 || !d->scores))
    return ODA_ERR_ARG;
  if (!d->W1 && !d->gate_scores && !d->scores) return ODA_ERR_ARG;
  return ODA_OK;
}

size_t layer_elems(const oda_ctx* ctx, int B, int heads) {
  return (size_t)B * heads * ctx->cfg.head_dim;
}

// The step splits the recall head only above this many layers.
constexpr int kRecallSplitMinLayers = 8;

// Early staging (launch_attn's `early`): the append kernel writes the ring
// and the paged cache of every layer, the record copy before it holds the
// lengths, and the gate writes the compacted ids. Every Local launch after the
// first follows another Local launch, and every Full launch after the first
// another Full launch; none of them writes those inputs, and each waits for
// its predecessor before it lets the next launch start. So from the second
// launch of each kind on, the inputs a launch stages before its own
// dependency wait were complete before it started.
//
// The recall head reads h_{t-1} and E(x_t), inputs of the step, and h^L_t,
// known only after the last Local launch. Where the head splits (recall_split),
// its first layer over the first two runs as a kernel of its own that starts
// with the step: on `side` (a captured graph), forked from `st` at the start,
// so that its weight stream overlaps the Local launches (which leave most of
// the memory bandwidth unused); without a side stream it runs first. The rest
// of the head then streams only the weights of h^L_t. No graph edge joins the
// prefix to the head: an edge from another branch would hold the head's
// launch past the last Local launch's completion, and its first weight tiles
// could no longer be requested while that launch runs. The prefix counts its
// finished CTAs instead, and each rank of the head that finds it incomplete
// computes its own share of the prefix's range. The side stream rejoins
// `st` after the head (before the conditional node).
oda_status pre_part(oda_ctx* ctx, const oda_step_desc* d, cudaStream_t st, cudaStream_t side,
                    cudaEvent_t fork, cudaEvent_t join, unsigned long long cond, bool set_cond) {
  const oda_config& c = ctx->cfg;
  const size_t eb = (size_t)ctx->lay.elem_bytes;
  oda_status s = ODA_OK;
  // (the prefix takes ~40 us beside the Local launches; with fewer layers the
  // head would find it unfinished and both would stream its weights)
  const bool split = d->W1 && c.layers >= kRecallSplitMinLayers &&
                     oda_impl::recall_split(ctx, d->B, d->H, d->hidden);
  if (split) {
    if (side) {
      if (cudaEventRecord(fork, st) != cudaSuccess || cudaStreamWaitEvent(side, fork, 0) != cudaSuccess)
        return ODA_ERR_CUDA;
    }
    s = oda_impl::launch_recall_prefix(ctx, d->h_prev, d->emb, d->H, d->W1, d->b1, d->hidden,
                                       d->B, side ? side : st);
    if (s != ODA_OK) return s;
    if (side && cudaEventRecord(join, side) != cudaSuccess) return ODA_ERR_CUDA;
  }
  s = oda_impl::launch_append(ctx, 0, c.layers, d->k_new, d->v_new, d->seq_lens, d->block_table,
                              d->kv_cache, d->ring, d->B, st, ctx->plan_local);
  if (s != ODA_OK) return s;
  for (int l = 0; l < c.layers; ++l) {
    const size_t qo = (size_t)l * layer_elems(ctx, d->B, c.hq) * eb;
    float* lse = d->lse ? d->lse + (size_t)l * d->B * c.hq : nullptr;
    s = oda_impl::launch_attn(ctx, true, l, static_cast<const char*>(d->q) + qo, d->seq_lens,
                              d->ring, nullptr, nullptr, nullptr,
                              static_cast<char*>(d->out) + qo, lse, d->B, st, ctx->plan_local,
                              /*early=*/l > 0);
    if (s != ODA_OK) return s;
  }
  const float* gs = d->gate_scores ? d->gate_scores : d->scores;
  bool gated = false;
  if (d->W1) {
    // The recall head follows the last Local launch, which writes none of its
    // weights: it requests its first W1 tiles before its dependency wait, and
    // its last CTA gates the scores, so the step needs no gate launch.
    RecallGate g;
    g.scores = gs;
    g.theta = d->theta;
    g.flags = d->flags;
    g.idx = d->idx;
    g.count = d->count;
    g.cond = cond;
    g.set_cond = set_cond;
    s = oda_impl::launch_recall(ctx, d->h_prev, d->emb, d->h_local, d->H, d->W1, d->b1, d->w2,
                                d->b2, d->hidden, d->scores, d->B, st, /*early=*/true, &g, &gated,
                                /*after_prefix=*/split);
    if (s != ODA_OK) return s;
    if (split && side && cudaStreamWaitEvent(st, join, 0) != cudaSuccess) return ODA_ERR_CUDA;
  }
  if (gated) return ODA_OK;
  return oda_impl::launch_gate(ctx, gs, d->theta, d->B, d->flags, d->idx, d->count, st, cond,
                               set_cond);
}

oda_status full_part(oda_ctx* ctx, const oda_step_desc* d, cudaStream_t st) {
  const oda_config& c = ctx->cfg;
  const size_t eb = (size_t)ctx->lay.elem_bytes;
  for (int l = 0; l < c.layers; ++l) {
    const size_t qo = (size_t)l * layer_elems(ctx, d->B, c.hq) * eb;
    float* lse = d->lse ? d->lse + (size_t)l * d->B * c.hq : nullptr;
    oda_status s = oda_impl::launch_attn(ctx, false, l, static_cast<const char*>(d->q) + qo,
                                         d->seq_lens, d->kv_cache, d->block_table, d->idx,
                                         d->count, static_cast<char*>(d->out) + qo, lse, d->B, st,
                                         nullptr, /*early=*/l > 0);
    if (s != ODA_OK) return s;
  }
  return ODA_OK;
}

}  // namespace

extern "C" {

oda_status oda_step_run(oda_ctx* ctx, const oda_step_desc* d, oda_stream stream) {
  oda_status s = check_desc(ctx, d);
  if (s != ODA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = pre_part(ctx, d, st, nullptr, nullptr, nullptr, 0ull, false);
  if (s != ODA_OK) return s;
  return full_part(ctx, d, st);
}

oda_status oda_step_graph_create(oda_ctx* ctx, const oda_step_desc* d, oda_graph** out) {
  if (!out) return ODA_ERR_ARG;
  *out = nullptr;
  oda_status s = check_desc(ctx, d);
  if (s != ODA_OK) return s;
  cudaStream_t st = nullptr, st2 = nullptr, st3 = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  s = ODA_ERR_CUDA;
  do {
    if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&st2, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&st3, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess)
      break;
    if (cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal) != cudaSuccess) break;
    cudaStreamCaptureStatus cs;
    cudaGraph_t cap = nullptr;
    const cudaGraphNode_t* deps = nullptr;
    size_t ndeps = 0;
    // the gate sets the condition on every launch (1 when it flags a row,
    // else 0), so the handle needs no default applied at each launch
    cudaGraphConditionalHandle handle = 0;
    bool ok = cudaStreamGetCaptureInfo(st, &cs, nullptr, &cap, &deps, &ndeps) == cudaSuccess &&
              cs == cudaStreamCaptureStatusActive &&
              cudaGraphConditionalHandleCreate(&handle, cap, 0, 0) == cudaSuccess;
    oda_status ps =
        ok ? pre_part(ctx, d, st, st3, fork, join, (unsigned long long)handle, true) : ODA_ERR_CUDA;
    cudaGraphNode_t cond_node = nullptr;
    cudaGraph_t body = nullptr;
    if (ps == ODA_OK &&
        cudaStreamGetCaptureInfo(st, &cs, nullptr, &cap, &deps, &ndeps) == cudaSuccess) {
      cudaGraphNodeParams p = {};
      p.type = cudaGraphNodeTypeConditional;
      p.conditional.handle = handle;
      p.conditional.type = cudaGraphCondTypeIf;
      p.conditional.size = 1;
      if (cudaGraphAddNode(&cond_node, cap, deps, ndeps, &p) == cudaSuccess) {
        body = p.conditional.phGraph_out[0];
        ok = cudaStreamUpdateCaptureDependencies(st, &cond_node, 1,
                                                 cudaStreamSetCaptureDependencies) == cudaSuccess;
      } else {
        ok = false;
      }
    } else {
      ok = false;
    }
    if (ok) {
      ok = cudaStreamBeginCaptureToGraph(st2, body, nullptr, nullptr, 0,
                                         cudaStreamCaptureModeThreadLocal) == cudaSuccess;
      if (ok) {
        const oda_status fs = full_part(ctx, d, st2);
        cudaGraph_t body_out = nullptr;
        ok = cudaStreamEndCapture(st2, &body_out) == cudaSuccess && fs == ODA_OK;
      }
    }
    cudaGraph_t done = nullptr;
    const bool ended = cudaStreamEndCapture(st, &done) == cudaSuccess;
    if (!ok || !ended || ps != ODA_OK) {
      if (done) cudaGraphDestroy(done);
      s = ps != ODA_OK ? ps : ODA_ERR_CUDA;
      break;
    }
    graph = done;
    if (cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) {
      cudaGraphDestroy(graph);
      graph = nullptr;
      break;
    }
    // upload now, so that the first launch does not pay for it (its
    // branches then start together, like every later launch's)
    if (cudaGraphUpload(exec, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess) {
      cudaGraphExecDestroy(exec);
      cudaGraphDestroy(graph);
      graph = nullptr;
      exec = nullptr;
      break;
    }
    s = ODA_OK;
  } while (false);
  cudaGetLastError();
  if (join) cudaEventDestroy(join);
  if (fork) cudaEventDestroy(fork);
  if (st3) cudaStreamDestroy(st3);
  if (st2) cudaStreamDestroy(st2);
  if (st) cudaStreamDestroy(st);
  if (s != ODA_OK) return s;
  oda_graph* g = static_cast<oda_graph*>(calloc(1, sizeof(oda_graph)));
  if (!g) {
    cudaGraphExecDestroy(exec);
    cudaGraphDestroy(graph);
    return ODA_ERR_ARG;
  }
  g->ctx = ctx;
  g->graph = graph;
  g->exec = exec;
  *out = g;
  return ODA_OK;
}

oda_status oda_step_graph_launch(oda_graph* g, oda_stream stream) {
  if (!g || !g->exec) return ODA_ERR_ARG;
  ODA_CUDA_TRY(cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream)));
  return ODA_OK;
}

oda_status oda_step_graph_run_io(oda_graph* g, const void* h_in, void* d_in, size_t in_bytes,
                                 const void* d_out, void* h_out, size_t out_bytes,
                                 oda_stream stream) {
  if (!g || !g->exec) return ODA_ERR_ARG;
  if ((in_bytes && (!h_in || !d_in)) || (out_bytes && (!d_out || !h_out))) return ODA_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (in_bytes) ODA_CUDA_TRY(cudaMemcpyAsync(d_in, h_in, in_bytes, cudaMemcpyHostToDevice, st));
  ODA_CUDA_TRY(cudaGraphLaunch(g->exec, st));
  if (out_bytes)
    ODA_CUDA_TRY(cudaMemcpyAsync(h_out, d_out, out_bytes, cudaMemcpyDeviceToHost, st));
  ODA_CUDA_TRY(cudaStreamSynchronize(st));
  return ODA_OK;
}

oda_status oda_step_graph_destroy(oda_graph* g) {
  if (!g) return ODA_OK;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  free(g);
  return ODA_OK;
}

}  // extern "C"
