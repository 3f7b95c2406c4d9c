"""Thin ctypes binding of liboda.so.

Argument marshalling only: tensors become raw device pointers and the current
torch stream becomes the cudaStream_t; every step of the decode path runs in
liboda's kernels. If the shared library is missing this module raises at
load time -- there is no fallback implementation.

Method names follow the C entry points in include/oda.h (without the
``oda_`` prefix).
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_int32, c_int64, c_uint8, c_uint64, c_void_p
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboda.so")

OK, ERR_ARG, ERR_SHAPE, ERR_DTYPE, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS, ERR_STATE = range(8)
BF16, F32 = 0, 1
MAX_BATCH = 1024
ATTN_INPUTS_READY = 1     # oda_local_attn / oda_full_attn_gated flag (see oda.h)
# A step with at least this many layers runs the recall head's first layer over
# h_prev and emb as a kernel of its own (oda.h, oda_step_run): one launch more.
RECALL_SPLIT_MIN_LAYERS = 8
STATUS_NAMES = {0: "ODA_OK", 1: "ODA_ERR_ARG", 2: "ODA_ERR_SHAPE", 3: "ODA_ERR_DTYPE",
                4: "ODA_ERR_CUDA", 5: "ODA_ERR_TIMEOUT", 6: "ODA_ERR_BOUNDS", 7: "ODA_ERR_STATE"}

# Every symbol include/oda.h declares.
EXPORTS = (
    "oda_layout", "oda_create", "oda_destroy", "oda_append_kv", "oda_ring_init",
    "oda_local_attn", "oda_recall_score", "oda_recall_loss", "oda_gate", "oda_full_attn_gated",
    "oda_get_device_error", "oda_selftest_wait_timeout", "oda_step_run",
    "oda_step_graph_create", "oda_step_graph_launch", "oda_step_graph_run_io",
    "oda_step_graph_destroy", "oda_version",
    "oda_full_attn_gated_static", "oda_range_attn", "oda_select_budget",
)


class OdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class OdaConfig(ctypes.Structure):
    _fields_ = [("layers", c_int), ("max_batch", c_int), ("hq", c_int), ("hkv", c_int),
                ("head_dim", c_int), ("sink", c_int), ("window", c_int),
                ("block_size", c_int), ("dtype", c_int), ("max_blocks_per_seq", c_int),
                ("num_blocks", c_int64)]


class OdaLayoutInfo(ctypes.Structure):
    _fields_ = [("tile_elems", c_int64), ("cache_layer_elems", c_int64),
                ("ring_blocks", c_int64), ("ring_layer_elems", c_int64),
                ("elem_bytes", c_int64)]


class OdaStepDesc(ctypes.Structure):
    _fields_ = [("B", c_int), ("q", c_void_p), ("k_new", c_void_p), ("v_new", c_void_p),
                ("seq_lens", c_void_p), ("block_table", c_void_p), ("kv_cache", c_void_p),
                ("ring", c_void_p), ("out", c_void_p), ("lse", c_void_p),
                ("h_prev", c_void_p), ("emb", c_void_p), ("h_local", c_void_p), ("H", c_int),
                ("W1", c_void_p), ("b1", c_void_p), ("w2", c_void_p), ("b2", c_float),
                ("hidden", c_int), ("scores", c_void_p), ("gate_scores", c_void_p),
                ("theta", c_float), ("flags", c_void_p), ("idx", c_void_p), ("count", c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load liboda.so (built by gated_local_full_b200.build) once."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m gated_local_full_b200.build` (no fallback exists)")
    L = ctypes.CDLL(LIB_PATH)
    vp = c_void_p
    sig = {
        "oda_layout": [POINTER(OdaConfig), POINTER(OdaLayoutInfo)],
        "oda_create": [POINTER(OdaConfig), POINTER(c_void_p)],
        "oda_destroy": [vp],
        "oda_append_kv": [vp, c_int, c_int, vp, vp, vp, vp, vp, vp, c_int, vp],
        "oda_ring_init": [vp, c_int, c_int, vp, vp, vp, vp, c_int, vp],
        "oda_local_attn": [vp, c_int, vp, vp, vp, vp, vp, c_int, ctypes.c_uint, vp],
        "oda_recall_score": [vp, vp, vp, vp, c_int, vp, vp, vp, c_float, c_int, vp, c_int, vp],
        "oda_gate": [vp, vp, c_float, c_int, vp, vp, vp, vp],
        "oda_recall_loss": [vp, vp, vp, vp, c_float, c_int64, vp, vp, vp],
        "oda_full_attn_gated": [vp, c_int, vp, vp, vp, vp, vp, vp, vp, vp, c_int, ctypes.c_uint,
                                vp],
        "oda_get_device_error": [vp, vp, POINTER(c_int)],
        "oda_selftest_wait_timeout": [vp, c_uint64, vp],
        "oda_step_run": [vp, POINTER(OdaStepDesc), vp],
        "oda_step_graph_create": [vp, POINTER(OdaStepDesc), POINTER(c_void_p)],
        "oda_step_graph_launch": [vp, vp],
        "oda_step_graph_run_io": [vp, vp, vp, ctypes.c_size_t, vp, vp, ctypes.c_size_t, vp],
        "oda_step_graph_destroy": [vp],
        "oda_full_attn_gated_static": [POINTER(OdaConfig), c_int, vp, vp, vp, vp, vp, vp, vp,
                                       vp, c_int, vp, vp],
        "oda_range_attn": [vp, c_int, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, c_int,
                           ctypes.c_uint, vp],
        "oda_select_budget": [vp, vp, vp, c_int64, c_int64, vp, vp, vp],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = c_int
    L.oda_version.argtypes = []
    L.oda_version.restype = ctypes.c_char_p
    _lib = L
    return L


def _check(status: int, where: str) -> None:
    if status != OK:
        raise OdaError(status, where)


def ptr(x) -> Optional[int]:
    """Device pointer of a tensor (must be CUDA and contiguous), an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("tensor must live on the GPU")
    if not x.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return x.data_ptr()


def hptr(x) -> Optional[int]:
    """Host pointer of a contiguous CPU tensor (pin it for asynchronous copies), or None."""
    if x is None:
        return None
    if x.is_cuda:
        raise ValueError("tensor must live in host memory")
    if not x.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_config(*, layers, max_batch, hq, hkv, head_dim, sink, window, dtype,
                max_blocks_per_seq, num_blocks, block_size=16) -> OdaConfig:
    dt = {"bf16": BF16, "f32": F32}.get(dtype, dtype)
    return OdaConfig(layers, max_batch, hq, hkv, head_dim, sink, window, block_size, dt,
                     max_blocks_per_seq, num_blocks)


def layout(cfg: OdaConfig) -> dict:
    info = OdaLayoutInfo()
    _check(lib().oda_layout(ctypes.byref(cfg), ctypes.byref(info)), "oda_layout")
    return {k: int(getattr(info, k)) for k, _ in OdaLayoutInfo._fields_}


class OdaGraph:
    """A captured decode step (see oda_step_graph_create)."""

    def __init__(self, ctx: "OdaContext", desc: OdaStepDesc):
        self._desc = desc
        h = c_void_p()
        _check(lib().oda_step_graph_create(ctx.handle, ctypes.byref(desc), ctypes.byref(h)),
               "oda_step_graph_create")
        self.handle = h

    def launch(self, stream=None) -> None:
        _check(lib().oda_step_graph_launch(self.handle, _stream(stream)), "oda_step_graph_launch")

    def run_io(self, h_in, d_in, d_out, h_out, stream=None) -> None:
        """Copy h_in -> d_in, launch, copy d_out -> h_out, wait (one call)."""
        nin = h_in.numel() * h_in.element_size() if h_in is not None else 0
        nout = h_out.numel() * h_out.element_size() if h_out is not None else 0
        _check(lib().oda_step_graph_run_io(self.handle, hptr(h_in), ptr(d_in), nin, ptr(d_out),
                                           hptr(h_out), nout, _stream(stream)),
               "oda_step_graph_run_io")

    def close(self) -> None:
        if self.handle:
            lib().oda_step_graph_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class OdaContext:
    """One liboda context (config + scratch) on the current CUDA device."""

    def __init__(self, cfg: OdaConfig):
        self.cfg = cfg
        self.layout = layout(cfg)
        h = c_void_p()
        _check(lib().oda_create(ctypes.byref(cfg), ctypes.byref(h)), "oda_create")
        self.handle = h

    def close(self) -> None:
        if self.handle:
            lib().oda_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------- the path
    def append_kv(self, layer_begin, layer_end, k_new, v_new, seq_lens, block_table, kv_cache,
                  ring, B, stream=None):
        _check(lib().oda_append_kv(self.handle, layer_begin, layer_end, ptr(k_new), ptr(v_new),
                                   ptr(seq_lens), ptr(block_table), ptr(kv_cache), ptr(ring), B,
                                   _stream(stream)), "oda_append_kv")

    def ring_init(self, layer_begin, layer_end, seq_lens, block_table, kv_cache, ring, B,
                  stream=None):
        _check(lib().oda_ring_init(self.handle, layer_begin, layer_end, ptr(seq_lens),
                                   ptr(block_table), ptr(kv_cache), ptr(ring), B,
                                   _stream(stream)), "oda_ring_init")

    def local_attn(self, layer, q, seq_lens, ring, out, lse, B, stream=None,
                   inputs_ready=False):
        """inputs_ready sets ODA_ATTN_INPUTS_READY (the ring and seq_lens were
        complete before the previous kernel on the stream reached its wait)."""
        _check(lib().oda_local_attn(self.handle, layer, ptr(q), ptr(seq_lens), ptr(ring),
                                    ptr(out), ptr(lse), B,
                                    ATTN_INPUTS_READY if inputs_ready else 0,
                                    _stream(stream)), "oda_local_attn")

    def recall_score(self, h_prev, emb, h_local, H, W1, b1, w2, b2, hidden, scores, B,
                     stream=None):
        _check(lib().oda_recall_score(self.handle, ptr(h_prev), ptr(emb), ptr(h_local), H,
                                      ptr(W1), ptr(b1), ptr(w2), float(b2), hidden, ptr(scores),
                                      B, _stream(stream)), "oda_recall_score")

    def recall_loss(self, q, logp_full, logp_local, lam, loss, n_full, stream=None):
        """Mean Huber_1(q - T(g - lam)) and #{g > lam}, g = logp_full - logp_local."""
        n = q.numel()
        if logp_full.numel() != n or logp_local.numel() != n:
            raise ValueError("recall_loss: q, logp_full and logp_local differ in length")
        _check(lib().oda_recall_loss(self.handle, ptr(q), ptr(logp_full), ptr(logp_local),
                                     float(lam), n, ptr(loss), ptr(n_full), _stream(stream)),
               "oda_recall_loss")

    def select_budget(self, scores, gain, k, selected, net_gain=None, stream=None):
        """The k positions with the largest scores (oda_select_budget), and the
        net gain per position of that selection when gain is given."""
        n = scores.numel()
        if gain is not None and gain.numel() != n:
            raise ValueError("select_budget: scores and gain differ in length")
        _check(lib().oda_select_budget(self.handle, ptr(scores), ptr(gain), n, int(k),
                                       ptr(selected), ptr(net_gain), _stream(stream)),
               "oda_select_budget")

    def gate(self, scores, theta, B, flags, idx, count, stream=None):
        _check(lib().oda_gate(self.handle, ptr(scores), float(theta), B, ptr(flags), ptr(idx),
                              ptr(count), _stream(stream)), "oda_gate")

    def full_attn_gated(self, layer, q, seq_lens, block_table, kv_cache, idx, count, out, lse,
                        B, stream=None, inputs_ready=False):
        """inputs_ready sets ODA_ATTN_INPUTS_READY (cache, lengths, block table,
        idx and count were complete before the previous kernel on the stream
        reached its wait)."""
        _check(lib().oda_full_attn_gated(self.handle, layer, ptr(q), ptr(seq_lens),
                                         ptr(block_table), ptr(kv_cache), ptr(idx), ptr(count),
                                         ptr(out), ptr(lse), B,
                                         ATTN_INPUTS_READY if inputs_ready else 0,
                                         _stream(stream)), "oda_full_attn_gated")

    def range_attn(self, layer, q, seq_lens, range_lo, range_hi, block_table, kv_cache, idx,
                   count, out, lse, B, stream=None, inputs_ready=False):
        """Attention of the rows idx[0..count) over positions [lo, hi) only
        (oda_range_attn)."""
        _check(lib().oda_range_attn(self.handle, layer, ptr(q), ptr(seq_lens), ptr(range_lo),
                                    ptr(range_hi), ptr(block_table), ptr(kv_cache), ptr(idx),
                                    ptr(count), ptr(out), ptr(lse), B,
                                    ATTN_INPUTS_READY if inputs_ready else 0, _stream(stream)),
               "oda_range_attn")

    def get_device_error(self, stream=None) -> int:
        e = c_int(0)
        _check(lib().oda_get_device_error(self.handle, _stream(stream), ctypes.byref(e)),
               "oda_get_device_error")
        return int(e.value)

    def selftest_wait_timeout(self, timeout_ns: int, stream=None) -> None:
        _check(lib().oda_selftest_wait_timeout(self.handle, int(timeout_ns), _stream(stream)),
               "oda_selftest_wait_timeout")

    # ---------------------------------------------------------- whole step
    @staticmethod
    def step_desc(*, B, q, k_new, v_new, seq_lens, block_table, kv_cache, ring, out, lse=None,
                  h_prev=None, emb=None, h_local=None, H=0, W1=None, b1=None, w2=None, b2=0.0,
                  hidden=0, scores=None, gate_scores=None, theta=0.0, flags=None, idx=None,
                  count=None) -> OdaStepDesc:
        return OdaStepDesc(B, ptr(q), ptr(k_new), ptr(v_new), ptr(seq_lens), ptr(block_table),
                           ptr(kv_cache), ptr(ring), ptr(out), ptr(lse), ptr(h_prev), ptr(emb),
                           ptr(h_local), H, ptr(W1), ptr(b1), ptr(w2), float(b2), hidden,
                           ptr(scores), ptr(gate_scores), float(theta), ptr(flags), ptr(idx),
                           ptr(count))

    def step_run(self, desc: OdaStepDesc, stream=None) -> None:
        _check(lib().oda_step_run(self.handle, ctypes.byref(desc), _stream(stream)),
               "oda_step_run")

    def step_graph(self, desc: OdaStepDesc) -> OdaGraph:
        return OdaGraph(self, desc)


def full_attn_gated_static(cfg: OdaConfig, layer, q, seq_lens, block_table, kv_cache, idx,
                           count, out, lse, B, err=None, stream=None) -> None:
    """oda_full_attn_gated_static: Full attention with no context and no device
    allocation (scratch in liboda's fixed device arrays). For callers whose
    device memory belongs to their own pool allocator."""
    _check(lib().oda_full_attn_gated_static(ctypes.byref(cfg), layer, ptr(q), ptr(seq_lens),
                                            ptr(block_table), ptr(kv_cache), ptr(idx),
                                            ptr(count), ptr(out), ptr(lse), B, ptr(err),
                                            _stream(stream)), "oda_full_attn_gated_static")


def version() -> str:
    return lib().oda_version().decode()
