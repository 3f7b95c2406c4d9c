"""Materialise a synthetic workload in GPU memory.

Allocates the caller-owned buffers of the decode path (paged KV cache, ring,
block table, per-step inputs) as torch tensors and fills them with the same
values synth/gen.py defines, using libsynth.so for the large tensors. This is
input generation only: the ring is *not* built here (the library's
ring-init entry point does that), and no attention arithmetic happens.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import c_int, c_int64, c_void_p

import numpy as np

from .gen import KIND_HIDDEN, stream_key
from .workloads import Workload

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} missing: run `python -m gated_local_full_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.synth_fill_streams.argtypes = [c_void_p, c_int, c_void_p, c_void_p, c_int, c_int64,
                                         c_int64, c_void_p, c_void_p]
        L.synth_fill_streams.restype = c_int
        L.synth_fill_paged_kv.argtypes = [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_int,
                                          c_int, c_int, c_int, c_int, c_int, c_int64, c_int,
                                          c_void_p, c_void_p, c_void_p]
        L.synth_fill_paged_kv.restype = c_int
        _lib = L
    return _lib


def _torch():
    import torch
    return torch


def _table_tensor(table: np.ndarray, device):
    torch = _torch()
    if table.dtype == np.uint16:
        return torch.from_numpy(table.view(np.int16).copy()).to(device)
    return torch.from_numpy(table.astype(np.float32).copy()).to(device)


def storage_dtype(w: Workload):
    torch = _torch()
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def host_to_device(a: np.ndarray, w: Workload, device):
    """Storage-dtype numpy array (uint16 bf16 bits or float32) -> torch tensor."""
    torch = _torch()
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16).copy()).to(device).view(
            torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32).copy()).to(device)


def fill_streams(dst, keys, offs, n_outer: int, inner: int, table: np.ndarray, stream=None):
    """Device version of gen.fill_streams into a contiguous tensor `dst`."""
    torch = _torch()
    dev = dst.device
    k = torch.from_numpy(np.asarray(keys, np.uint64).view(np.int64).copy()).to(dev)
    o = torch.from_numpy(np.asarray(offs, np.uint64).view(np.int64).copy()).to(dev)
    t = _table_tensor(table, dev)
    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    r = lib().synth_fill_streams(dst.data_ptr(), dst.element_size(), k.data_ptr(), o.data_ptr(),
                                 int(k.numel()), int(n_outer), int(inner), t.data_ptr(), st)
    if r != 0:
        raise RuntimeError(f"synth_fill_streams failed ({r})")
    torch.cuda.current_stream().synchronize()


class DeviceWorkload:
    """All buffers of a workload on the GPU.

    extra_steps: steps beyond w.steps to provision (cache capacity and
    per-step inputs), e.g. for benchmark warm-up.
    host_q: build per-step queries on the host (needed when needles adjust
    them); otherwise the GPU fill writes them.
    """

    def __init__(self, w: Workload, lay: dict, max_batch: int, extra_steps: int = 0,
                 device: str = "cuda", host_q=None, fill_cache: bool = True):
        torch = _torch()
        self.w = w
        self.device = device
        self.steps = w.steps + extra_steps
        S, L, B, hq, hkv, d = self.steps, w.layers, w.batch, w.hq, w.hkv, w.d
        dt = storage_dtype(w)
        bt, nb = w.paging(extra_steps)
        self.num_blocks = nb
        self.max_blocks = bt.shape[1]
        self.block_table = torch.from_numpy(bt).to(device)
        self.cache = torch.empty(L * lay["cache_layer_elems"], dtype=dt, device=device)
        self.ring = torch.zeros(L * lay["ring_layer_elems"], dtype=dt, device=device)
        # history positions 1..t0-1
        if fill_cache:
            keys = torch.from_numpy(w.kv_keys().reshape(-1).view(np.int64).copy()).to(device)
            npos = torch.from_numpy((w.t0 - 1).astype(np.int32)).to(device)
            table = _table_tensor(w.kv_table(), device)
            bad = torch.zeros(1, dtype=torch.int32, device=device)
            r = lib().synth_fill_paged_kv(self.cache.data_ptr(), self.cache.element_size(),
                                          keys.data_ptr(), self.block_table.data_ptr(),
                                          npos.data_ptr(), L, B, hkv, d, w.block_size,
                                          self.max_blocks, nb, int((w.t0 - 1).max()),
                                          table.data_ptr(), bad.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
            if r != 0 or int(bad.item()) != 0:
                raise RuntimeError("synth_fill_paged_kv failed")
            for n in w.needles:
                self.write_cache_row(n.layer, n.row, n.kv_head, 0, n.position,
                                     host_to_device(n.key, w, device))
        # per-step queries [S][L][B][hq][d]
        if host_q is None:
            host_q = len(w.needles) > 0
        if host_q:
            q = np.stack([w.q_step(i) for i in range(S)])
            self.q = host_to_device(q, w, device)
        else:
            self.q = torch.empty((S, L, B, hq, d), dtype=dt, device=device)
            fill_streams(self.q, w.q_keys().reshape(-1), np.zeros(L * B * hq, np.uint64), S, d,
                         w.q_table())
        # per-step new K/V [S][L][B][hkv][d]: history streams at position t0+i
        kk = w.kv_keys()
        self.k_new = torch.empty((S, L, B, hkv, d), dtype=dt, device=device)
        self.v_new = torch.empty((S, L, B, hkv, d), dtype=dt, device=device)
        for kv, dst in ((0, self.k_new), (1, self.v_new)):
            keys = kk[:, :, :, kv].reshape(-1)
            offs = np.repeat(((w.t0 - 1) * d).astype(np.uint64)[None, :, None], L, axis=0)
            offs = np.repeat(offs, hkv, axis=2).reshape(-1)
            fill_streams(dst, keys, offs, S, d, w.kv_table())
        # step positions and gate scores
        t = (w.t0[None, :] + np.arange(S)[:, None]).astype(np.int32)
        self.seq_lens = torch.from_numpy(t).to(device)           # [S][B]
        sc = w.scores(extra_steps)
        self.scores = None if sc is None else torch.from_numpy(sc).to(device)
        # recall head
        self.recall = None
        if w.recall:
            W1, b1, w2, b2 = w.recall_weights()
            H = w.hidden
            hs = []
            tab = w.recall_tables()[0]
            for which in range(3):
                t_ = torch.empty((S, B, H), dtype=torch.bfloat16, device=device)
                keys = [stream_key(w.seed, KIND_HIDDEN, which, b) for b in range(B)]
                # counter = step*H + j  ->  outer = step, stream = row, inner = H
                fill_streams(t_, np.array(keys, np.uint64), np.zeros(B, np.uint64), S, H, tab)
                hs.append(t_)
            self.recall = dict(
                h_prev=hs[0], emb=hs[1], h_local=hs[2], H=H,
                W1=host_to_device(W1, w, device).view(torch.bfloat16),
                b1=torch.from_numpy(b1).to(device),
                w2=torch.from_numpy(
                    (w2.astype(np.uint32) << 16).view(np.float32).copy()).to(device),
                b2=float(b2), hidden=w.recall_hidden)
        torch.cuda.synchronize()

    def write_cache_row(self, layer, row, g, kv, position, values):
        """Write one [d] row at (layer, row, kv head, K/V, position) of the paged cache."""
        w = self.w
        bi = (position - 1) // w.block_size
        blk = int(self.block_table[row, bi].item())
        off = ((((layer * self.num_blocks + blk) * w.hkv + g) * 2 + kv) * w.block_size
               + (position - 1) % w.block_size) * w.d
        self.cache[off:off + w.d] = values

    def read_cache_row(self, layer, row, g, kv, position):
        w = self.w
        bi = (position - 1) // w.block_size
        blk = int(self.block_table[row, bi].item())
        off = ((((layer * self.num_blocks + blk) * w.hkv + g) * 2 + kv) * w.block_size
               + (position - 1) % w.block_size) * w.d
        return self.cache[off:off + w.d]
