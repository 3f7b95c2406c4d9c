"""Shared test plumbing: build a context + device workload, call the oracle.

The CUDA side is reached only through gated_local_full_b200 (the C ABI);
expected values come only from oracle/ on inputs from synth/.
"""

from __future__ import annotations

import numpy as np

import oracle as O
from synth.workloads import Workload

BF16_ATOL, BF16_RTOL = 2e-3, 1e-2
F32_ATOL, F32_RTOL = 1e-5, 1e-5


def tol(w: Workload):
    return (BF16_ATOL, BF16_RTOL) if w.dtype == "bf16" else (F32_ATOL, F32_RTOL)


def setup(w: Workload, extra_steps: int = 0, max_batch=None, host_q=None):
    """Returns (ctx, dw): an OdaContext sized for w and its DeviceWorkload,
    with the ring built from the prefilled cache (positions 1..t0-1)."""
    import torch
    from gated_local_full_b200 import oda
    from synth.device import DeviceWorkload

    bt, nb = w.paging(extra_steps)
    cfg = oda.make_config(layers=w.layers, max_batch=max_batch or w.batch, hq=w.hq, hkv=w.hkv,
                          head_dim=w.d, sink=w.sink, window=w.window, dtype=w.dtype,
                          max_blocks_per_seq=bt.shape[1], num_blocks=nb)
    lay = oda.layout(cfg)
    ctx = oda.OdaContext(cfg)
    dw = DeviceWorkload(w, lay, cfg.max_batch, extra_steps=extra_steps, host_q=host_q)
    prefill = torch.from_numpy((w.t0 - 1).astype(np.int32)).cuda()
    ctx.ring_init(0, w.layers, prefill, dw.block_table, dw.cache, dw.ring, w.batch)
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    return ctx, dw


def to_f64(t, w: Workload) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def oracle_kv(w: Workload, layer: int, row: int, t: int):
    """K, V as float64 [hkv][t][d] holding positions 1..t."""
    K = np.stack([w.to_f64(w.kv_history(layer, row, g, 0, t)) for g in range(w.hkv)])
    V = np.stack([w.to_f64(w.kv_history(layer, row, g, 1, t)) for g in range(w.hkv)])
    return K, V


def oracle_row(w: Workload, step: int, layer: int, row: int, q_host=None):
    """Oracle Local and Full outputs for one (step, layer, row)."""
    t = int(w.t0[row]) + step
    q = w.to_f64((q_host if q_host is not None else w.q_step(step))[layer, row])
    K, V = oracle_kv(w, layer, row, t)
    loc, lse_l = O.local_attention(q, K, V, t, w.sink, w.window)
    ful, lse_f = O.full_attention(q, K, V, t)
    return dict(local=loc, lse_local=lse_l, full=ful, lse_full=lse_f, t=t)


def assert_close(got: np.ndarray, ref: np.ndarray, atol: float, rtol: float, what: str):
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {err.size} outside tolerance; "
                             f"worst at {i}: got {got[i]!r} ref {ref[i]!r} "
                             f"(max abs err {err.max():.3e})")
    return float(err.max())


def oracle_kv_head(w: Workload, layer: int, row: int, g: int, t: int, positions=None):
    """K, V of one KV head as float64 [1][t][d] (row p-1 = position p). With
    `positions`, only those rows are generated (the others stay 0); the
    oracle only reads positions of the access set it is given."""
    K = np.zeros((1, t, w.d))
    V = np.zeros((1, t, w.d))
    if positions is None:
        K[0] = w.to_f64(w.kv_history(layer, row, g, 0, t))
        V[0] = w.to_f64(w.kv_history(layer, row, g, 1, t))
        return K, V
    from synth.gen import table_values
    tab = w.kv_table()
    pos = sorted(positions)
    for kv, dst in ((0, K), (1, V)):
        key = w.kv_key(layer, row, g, kv)
        # contiguous runs keep the generator vectorised
        runs, start, prev = [], pos[0], pos[0]
        for p in pos[1:]:
            if p != prev + 1:
                runs.append((start, prev)); start = p
            prev = p
        runs.append((start, prev))
        for a, b in runs:
            vals = table_values(key, (a - 1) * w.d, (b - a + 1) * w.d, tab).reshape(-1, w.d)
            dst[0, a - 1:b] = w.to_f64(vals)
        if kv == 0:
            for n in w.needles:
                if (n.layer, n.row, n.kv_head) == (layer, row, g) and n.position in set(pos):
                    dst[0, n.position - 1] = w.to_f64(n.key)
    return K, V


def oracle_head(w: Workload, q_row: np.ndarray, layer: int, row: int, g: int, t: int,
                full: bool):
    """Oracle output for the G query heads of KV head g: Local, or Full if `full`."""
    G = w.group
    q = w.to_f64(q_row[g * G:(g + 1) * G])
    if full:
        K, V = oracle_kv_head(w, layer, row, g, t)
        return O.full_attention(q, K, V, t)
    K, V = oracle_kv_head(w, layer, row, g, t, O.local_access_set(t, w.sink, w.window))
    return O.local_attention(q, K, V, t, w.sink, w.window)


def _head_task(args):
    """One oracle (layer, row, KV head) evaluation in a worker process."""
    w, q_row, layer, row, g, t, full = args
    return oracle_head(w, q_row, layer, row, g, t, full)


def oracle_heads(w: Workload, tasks, workers=None):
    """Oracle outputs for many (q_row [hq][d], layer, row, kv_head, t, full)
    tasks, in order: [(out [G][d], lse [G]), ...]. Generating a long row's
    K/V dominates, so the tasks run in a pool of processes started with
    spawn (safe beside a CUDA context); small task lists run inline."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import os
    args = [(w, q, l, b, g, t, f) for (q, l, b, g, t, f) in tasks]
    n = workers or min(len(os.sched_getaffinity(0)), 16)
    if len(args) <= 2 or n <= 1:
        return [_head_task(a) for a in args]
    with cf.ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn")) as ex:
        return list(ex.map(_head_task, args, chunksize=1))


def _range_task(args):
    w, q_row, layer, row, g, lo, hi = args
    G = w.group
    q = w.to_f64(q_row[g * G:(g + 1) * G])
    K, V = oracle_kv_head(w, layer, row, g, hi - 1, range(lo, hi))
    return O.range_attention(q, K, V, lo, hi)


def oracle_range_heads(w: Workload, tasks, workers=None):
    """Oracle outputs of range-restricted attention for (q_row, layer, row,
    kv_head, lo, hi) tasks, in order (a spawn process pool, as oracle_heads)."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import os
    args = [(w, *t) for t in tasks]
    n = workers or min(len(os.sched_getaffinity(0)), 16)
    if len(args) <= 2 or n <= 1:
        return [_range_task(a) for a in args]
    with cf.ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn")) as ex:
        return list(ex.map(_range_task, args, chunksize=1))
