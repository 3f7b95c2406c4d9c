"""Decode-step runtime: static buffers + one captured CUDA graph per step.

A serving loop writes each step's inputs (queries, the new token's K/V, the
positions, the gate scores and/or the recall head's hidden states) into fixed
device buffers and replays the graph captured by oda_step_graph_create. The
graph holds every launch of the step; the Full launches sit behind the IF
node the gate sets on the device, so no decision travels to the host.

All per-step inputs live in one contiguous "record" (256-byte aligned
fields), so a step is fed with a single copy, from device or pinned host
memory. torch is used for memory and copies only.
"""

from __future__ import annotations

from typing import Optional

from . import oda


def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


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
        if recall is None and not external_scores:
            raise ValueError("without a recall head the gate needs external scores")
        # ---- input record layout
        fields = [("q", (L, B, hq, d), dt), ("k_new", (L, B, hkv, d), dt),
                  ("v_new", (L, B, hkv, d), dt), ("seq_lens", (B,), torch.int32)]
        if external_scores:
            fields.append(("gate_scores", (B,), torch.float32))
        if recall is not None:
            H = recall["H"]
            fields += [("h_prev", (B, H), torch.bfloat16), ("emb", (B, H), torch.bfloat16),
                       ("h_local", (B, H), torch.bfloat16)]
        self.fields = {}
        off = 0
        for name, shape, fdt in fields:
            n = 1
            for s in shape:
                n *= s
            nbytes = n * torch.empty((), dtype=fdt).element_size()
            self.fields[name] = (off, shape, fdt, nbytes)
            off = _align(off + nbytes)
        self.record_bytes = off
        self.record = torch.zeros(self.record_bytes, dtype=torch.uint8, device=dev)
        for name, (o, shape, fdt, nbytes) in self.fields.items():
            setattr(self, name, self.record[o:o + nbytes].view(fdt).view(shape))
        if not external_scores:
            self.gate_scores = None
        # ---- outputs; the last layer's output and the count are contiguous
        # (the "result" a host loop reads back every step, in one copy)
        esz = torch.empty((), dtype=dt).element_size()
        out_bytes = L * B * hq * d * esz
        self._outbuf = torch.zeros(out_bytes + 16, dtype=torch.uint8, device=dev)
        self.out = self._outbuf[:out_bytes].view(dt).view(L, B, hq, d)
        self.count = self._outbuf[out_bytes:out_bytes + 4].view(torch.int32)
        self.result = self._outbuf[(L - 1) * B * hq * d * esz:out_bytes + 4]
        self.lse = torch.zeros((L, B, hq), dtype=torch.float32, device=dev) if with_lse else None
        self.scores = torch.zeros(B, dtype=torch.float32, device=dev)
        self.flags = torch.zeros(B, dtype=torch.uint8, device=dev)
        self.idx = torch.zeros(B, dtype=torch.int32, device=dev)
        self.kv_cache, self.ring, self.block_table = kv_cache, ring, block_table
        self.recall = recall
        rk = {}
        if recall is not None:
            rk = dict(h_prev=self.h_prev, emb=self.emb, h_local=self.h_local, H=recall["H"],
                      W1=recall["W1"], b1=recall["b1"], w2=recall["w2"], b2=recall["b2"],
                      hidden=recall["hidden"])
        self.desc = ctx.step_desc(B=B, q=self.q, k_new=self.k_new, v_new=self.v_new,
                                  seq_lens=self.seq_lens, block_table=block_table,
                                  kv_cache=kv_cache, ring=ring, out=self.out, lse=self.lse,
                                  scores=self.scores, gate_scores=self.gate_scores, theta=theta,
                                  flags=self.flags, idx=self.idx, count=self.count, **rk)
        self.graph = ctx.step_graph(self.desc) if graph else None

    # ------------------------------------------------------------- feeding
    def new_records(self, n: int, device="cuda", pin: bool = False):
        """Zeroed [n][record_bytes] buffer for pre-packed step records."""
        import torch
        r = torch.zeros((n, self.record_bytes), dtype=torch.uint8,
                        device=device if not pin else "cpu")
        return r.pin_memory() if pin else r

    def record_view(self, records, i: int, name: str):
        """View of field `name` inside record i of a records buffer."""
        o, shape, fdt, nbytes = self.fields[name]
        return records[i, o:o + nbytes].view(fdt).view(shape)

    def pack(self, records, i: int, **inputs) -> None:
        for name, val in inputs.items():
            if val is not None:
                self.record_view(records, i, name).copy_(val)

    def feed_record(self, records, i: int, non_blocking: bool = True) -> None:
        """One copy: record i (device or pinned host) -> the static inputs."""
        self.record.copy_(records[i], non_blocking=non_blocking)

    def feed(self, q, k_new, v_new, seq_lens, gate_scores=None, h_prev=None, emb=None,
             h_local=None, non_blocking=True) -> None:
        """Per-field copies into the static inputs (convenience)."""
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

    def new_result(self):
        """Pinned host buffer shaped like `result` (last layer's output, then the count)."""
        import torch
        return torch.empty(self.result.numel(), dtype=torch.uint8).pin_memory()

    def run_io(self, h_record, h_result, stream=None) -> None:
        """One host-driven step in one library call: the packed inputs from the
        host record h_record (pinned, record_bytes), the captured step, and
        the result back into h_result (see new_result); returns when h_result
        holds it. Needs the captured graph."""
        if self.graph is None:
            raise RuntimeError("run_io needs the captured step graph")
        self.graph.run_io(h_record, self.record, self.result, h_result, stream)

    def split_result(self, h_result):
        """(last layer's output, count) views of a result buffer."""
        import torch
        n = self.result.numel() - 4
        out = h_result[:n].view(self.out.dtype).view(self.out.shape[1:])
        return out, h_result[n:n + 4].view(torch.int32)

    def close(self) -> None:
        if self.graph is not None:
            self.graph.close()
            self.graph = None
