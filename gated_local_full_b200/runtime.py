"""Decode-step runtime: static buffers + one captured CUDA graph per step.

A serving loop writes each step's inputs (queries, the new token's K/V, the
positions, optionally the recall head's hidden states) into fixed device
buffers and replays the graph captured by oda_step_graph_create. The graph
holds every launch of the step; the Full launches sit behind the IF node the
gate sets on the device, so no decision travels to the host.

torch is used for memory and copies only.
"""

from __future__ import annotations

from typing import Optional

from . import oda


class DecodeStep:
    def __init__(self, ctx: oda.OdaContext, B: int, kv_cache, ring, block_table, *,
                 recall: Optional[dict] = None, external_scores: bool = False,
                 with_lse: bool = False, theta: float = 0.0, graph: bool = True):
        import torch
        c = ctx.cfg
        self.ctx, self.B = ctx, B
        dt = torch.bfloat16 if c.dtype == oda.BF16 else torch.float32
        dev = "cuda"
        L, hq, hkv, d = c.layers, c.hq, c.hkv, c.head_dim
        self.q = torch.zeros((L, B, hq, d), dtype=dt, device=dev)
        self.k_new = torch.zeros((L, B, hkv, d), dtype=dt, device=dev)
        self.v_new = torch.zeros((L, B, hkv, d), dtype=dt, device=dev)
        self.seq_lens = torch.ones(B, dtype=torch.int32, device=dev)
        self.out = torch.zeros((L, B, hq, d), dtype=dt, device=dev)
        self.lse = torch.zeros((L, B, hq), dtype=torch.float32, device=dev) if with_lse else None
        self.scores = torch.zeros(B, dtype=torch.float32, device=dev)
        self.gate_scores = torch.zeros(B, dtype=torch.float32, device=dev) if external_scores else None
        self.flags = torch.zeros(B, dtype=torch.uint8, device=dev)
        self.idx = torch.zeros(B, dtype=torch.int32, device=dev)
        self.count = torch.zeros(1, dtype=torch.int32, device=dev)
        self.kv_cache, self.ring, self.block_table = kv_cache, ring, block_table
        self.recall = recall
        rk = {}
        if recall is not None:
            H = recall["H"]
            self.h_prev = torch.zeros((B, H), dtype=torch.bfloat16, device=dev)
            self.emb = torch.zeros((B, H), dtype=torch.bfloat16, device=dev)
            self.h_local = torch.zeros((B, H), dtype=torch.bfloat16, device=dev)
            rk = dict(h_prev=self.h_prev, emb=self.emb, h_local=self.h_local, H=H,
                      W1=recall["W1"], b1=recall["b1"], w2=recall["w2"], b2=recall["b2"],
                      hidden=recall["hidden"])
        if recall is None and not external_scores:
            raise ValueError("without a recall head the gate needs external scores")
        self.desc = ctx.step_desc(B=B, q=self.q, k_new=self.k_new, v_new=self.v_new,
                                  seq_lens=self.seq_lens, block_table=block_table,
                                  kv_cache=kv_cache, ring=ring, out=self.out, lse=self.lse,
                                  scores=self.scores, gate_scores=self.gate_scores, theta=theta,
                                  flags=self.flags, idx=self.idx, count=self.count, **rk)
        self.graph = ctx.step_graph(self.desc) if graph else None

    def feed(self, q, k_new, v_new, seq_lens, gate_scores=None, h_prev=None, emb=None,
             h_local=None, non_blocking=True) -> None:
        """Copy one step's inputs into the static buffers (device or pinned host)."""
        self.q.copy_(q, non_blocking=non_blocking)
        self.k_new.copy_(k_new, non_blocking=non_blocking)
        self.v_new.copy_(v_new, non_blocking=non_blocking)
        self.seq_lens.copy_(seq_lens, non_blocking=non_blocking)
        if gate_scores is not None:
            self.gate_scores.copy_(gate_scores, non_blocking=non_blocking)
        if h_prev is not None:
            self.h_prev.copy_(h_prev, non_blocking=non_blocking)
            self.emb.copy_(emb, non_blocking=non_blocking)
            self.h_local.copy_(h_local, non_blocking=non_blocking)

    def run(self, stream=None) -> None:
        if self.graph is not None:
            self.graph.launch(stream)
        else:
            self.ctx.step_run(self.desc, stream)

    def close(self) -> None:
        if self.graph is not None:
            self.graph.close()
            self.graph = None
