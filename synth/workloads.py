"""Workload recipes: shapes, context lengths, flag draws, paging, needles.

Five workloads mirror the pages' operating points (context lengths 16K and
128K, Full-call rates 12.5 % and ~41 %, the Qwen3-1.7B attention shape of 16
query / 8 KV heads, head_dim 128, 28 layers, hidden 2048) plus a tiny fp32
case and a mixed-length serving batch. All values are synthetic and seeded.

Positions are 1-indexed. ``t0[b]`` is the context length t at the first
decode step of row b: the step appends the token at position t0[b] and then
attends over positions drawn from {1..t0[b]}. Step i uses t = t0[b] + i.
History positions 1..t0[b]-1 are "prefill" and are written straight into the
paged cache by the generator.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

from .gen import (
    KIND_HIDDEN, KIND_KV, KIND_NEEDLE, KIND_Q, KIND_VEC, KIND_W1,
    bf16_bits_to_f32, bf16_round_bits, normal_table, stream_key, table_values,
    uniform_table,
)


@dataclass
class Needle:
    """A planted key: K[layer, row, kv_head, position] = u * sqrt(d) (rounded to
    the workload dtype), and every step's query of ``q_head`` is shifted along
    that key so that its raw dot product with it is ``dot`` before rounding."""
    layer: int
    row: int
    kv_head: int
    q_head: int
    position: int
    key: np.ndarray          # [d] in the storage dtype (uint16 bf16 bits or float32)
    dot: float = 8.0


@dataclass
class Workload:
    name: str
    dtype: str               # "bf16" or "f32": storage dtype of q, K, V and outputs
    layers: int
    batch: int
    hq: int
    hkv: int
    d: int
    sink: int                # s
    window: int              # w
    block_size: int
    t0: np.ndarray           # int64 [B]
    steps: int
    seed: int
    sigma_kv: float = 0.5
    sigma_q: float = 1.0
    flag_rate: Optional[float] = None   # Bernoulli rate; None = fixed scores or recall head
    flag_per: str = "row"               # "row": one draw per row; "step": one draw per step (B=1)
    fixed_scores: Optional[np.ndarray] = None
    recall: bool = False
    hidden: int = 2048
    recall_hidden: int = 4096
    needles_on: bool = False
    needles: List[Needle] = field(default_factory=list)

    # ---------------------------------------------------------------- shapes
    @property
    def group(self) -> int:
        return self.hq // self.hkv

    def capacity(self, extra_steps: int = 0) -> np.ndarray:
        """Positions each row must hold after steps + extra_steps appends."""
        return self.t0 + self.steps + extra_steps - 1

    def paging(self, extra_steps: int = 0):
        """(block_table int32 [B][max_blocks], num_blocks).

        Physical block ids are a seeded random permutation handed out to rows in
        order; table entries past a row's capacity are -1."""
        cap = self.capacity(extra_steps)
        nblk = (cap + self.block_size - 1) // self.block_size
        max_blocks = int(nblk.max())
        num_blocks = int(nblk.sum())
        rng = np.random.Generator(np.random.PCG64([self.seed, 7001]))
        perm = rng.permutation(num_blocks).astype(np.int32)
        table = np.full((self.batch, max_blocks), -1, dtype=np.int32)
        o = 0
        for b in range(self.batch):
            n = int(nblk[b])
            table[b, :n] = perm[o:o + n]
            o += n
        return table, num_blocks

    # --------------------------------------------------------------- streams
    def kv_key(self, layer: int, row: int, g: int, kv: int) -> int:
        return stream_key(self.seed, KIND_KV, layer, row, g, kv)

    def kv_keys(self) -> np.ndarray:
        """uint64 [L][B][Hkv][2]."""
        k = np.empty((self.layers, self.batch, self.hkv, 2), dtype=np.uint64)
        for l in range(self.layers):
            for b in range(self.batch):
                for g in range(self.hkv):
                    for kv in range(2):
                        k[l, b, g, kv] = self.kv_key(l, b, g, kv)
        return k

    def q_keys(self) -> np.ndarray:
        """uint64 [L][B][Hq]."""
        k = np.empty((self.layers, self.batch, self.hq), dtype=np.uint64)
        for l in range(self.layers):
            for b in range(self.batch):
                for h in range(self.hq):
                    k[l, b, h] = stream_key(self.seed, KIND_Q, l, b, h)
        return k

    def kv_table(self) -> np.ndarray:
        return normal_table(self.sigma_kv, self.dtype)

    def q_table(self) -> np.ndarray:
        return normal_table(self.sigma_q, self.dtype)

    # ------------------------------------------------------- host-side values
    def kv_history(self, layer: int, row: int, g: int, kv: int, npos: int) -> np.ndarray:
        """Storage-dtype values of K (kv=0) or V (kv=1) at positions 1..npos,
        shape [npos][d], with needles applied."""
        vals = table_values(self.kv_key(layer, row, g, kv), 0, npos * self.d,
                            self.kv_table()).reshape(npos, self.d)
        if kv == 0:
            for n in self.needles:
                if (n.layer, n.row, n.kv_head) == (layer, row, g) and n.position <= npos:
                    vals[n.position - 1] = n.key
        return vals

    def q_step(self, step: int) -> np.ndarray:
        """Storage-dtype queries for one step, [L][B][Hq][d], needles applied."""
        tab = self.q_table()
        q = np.empty((self.layers, self.batch, self.hq, self.d), dtype=tab.dtype)
        for l in range(self.layers):
            for b in range(self.batch):
                for h in range(self.hq):
                    key = stream_key(self.seed, KIND_Q, l, b, h)
                    q[l, b, h] = table_values(key, step * self.d, self.d, tab)
        for n in self.needles:
            q[n.layer, n.row, n.q_head] = self._aim(q[n.layer, n.row, n.q_head], n)
        return q

    def q_step_layer(self, step: int, layer: int) -> np.ndarray:
        """Storage-dtype queries of one layer for one step, [B][Hq][d], needles applied."""
        tab = self.q_table()
        q = np.empty((self.batch, self.hq, self.d), dtype=tab.dtype)
        for b in range(self.batch):
            for h in range(self.hq):
                key = stream_key(self.seed, KIND_Q, layer, b, h)
                q[b, h] = table_values(key, step * self.d, self.d, tab)
        for n in self.needles:
            if n.layer == layer:
                q[n.row, n.q_head] = self._aim(q[n.row, n.q_head], n)
        return q

    def kv_new_step(self, step: int):
        """(k_new, v_new) for one step, each [L][B][Hkv][d] in storage dtype:
        the history streams at position t0[b] + step."""
        tab = self.kv_table()
        out = []
        for kv in range(2):
            a = np.empty((self.layers, self.batch, self.hkv, self.d), dtype=tab.dtype)
            for l in range(self.layers):
                for b in range(self.batch):
                    pos = int(self.t0[b]) + step
                    for g in range(self.hkv):
                        a[l, b, g] = table_values(self.kv_key(l, b, g, kv),
                                                  (pos - 1) * self.d, self.d, tab)
            out.append(a)
        return out[0], out[1]

    def to_f64(self, a: np.ndarray) -> np.ndarray:
        """Exact widening of storage-dtype values to float64."""
        if self.dtype == "bf16":
            return bf16_bits_to_f32(a).astype(np.float64)
        return np.asarray(a, dtype=np.float32).astype(np.float64)

    def _round(self, x: np.ndarray) -> np.ndarray:
        if self.dtype == "bf16":
            return bf16_round_bits(x)
        return np.asarray(x, dtype=np.float64).astype(np.float32)

    def _aim(self, q: np.ndarray, n: Needle) -> np.ndarray:
        """Shift q along the needle key so that q.k = n.dot (then round)."""
        qf = self.to_f64(q)
        kf = self.to_f64(n.key)
        qf = qf + (n.dot - qf @ kf) / (kf @ kf) * kf
        return self._round(qf)

    # ------------------------------------------------------------ gate input
    def flags(self, extra_steps: int = 0) -> Optional[np.ndarray]:
        """uint8 [steps+extra][B] Bernoulli flags, or None if not drawn."""
        if self.flag_rate is None:
            return None
        n = self.steps + extra_steps
        rng = np.random.Generator(np.random.PCG64([self.seed, 7002]))
        if self.flag_per == "step":
            f = (rng.random(n) < self.flag_rate).astype(np.uint8)
            return np.repeat(f[:, None], self.batch, axis=1)
        f = (rng.random(self.batch) < self.flag_rate).astype(np.uint8)
        return np.repeat(f[None, :], n, axis=0)

    def scores(self, extra_steps: int = 0) -> Optional[np.ndarray]:
        """float32 [steps+extra][B] scores fed to the gate: the fixed scores,
        or +1/-1 for drawn flags. None when the recall head decides."""
        if self.fixed_scores is not None:
            n = self.steps + extra_steps
            return np.repeat(np.asarray(self.fixed_scores, np.float32)[None, :], n, axis=0)
        f = self.flags(extra_steps)
        if f is None:
            return None
        return np.where(f > 0, np.float32(1.0), np.float32(-1.0)).astype(np.float32)

    # ----------------------------------------------------------- recall head
    def recall_in_dim(self) -> int:
        return 3 * self.hidden

    def recall_tables(self):
        """(hidden-state table, W1 table, w2 table): N(0,1) states and
        Xavier-uniform weights U(+-sqrt(6/(fan_in+fan_out)))."""
        fin = self.recall_in_dim()
        a1 = np.sqrt(6.0 / (fin + self.recall_hidden))
        a2 = np.sqrt(6.0 / (self.recall_hidden + 1))
        return (normal_table(1.0, "bf16"), uniform_table(a1, "bf16"), uniform_table(a2, "bf16"))

    def hidden_key(self, which: int, row: int) -> int:
        return stream_key(self.seed, KIND_HIDDEN, which, row)

    def w1_key(self) -> int:
        return stream_key(self.seed, KIND_W1, 0)

    def w2_key(self) -> int:
        return stream_key(self.seed, KIND_VEC, 0)

    def hidden_step(self, step: int):
        """(h_prev, emb, h_local) bf16 bits, each [B][H]."""
        tab = self.recall_tables()[0]
        out = []
        for which in range(3):
            a = np.empty((self.batch, self.hidden), dtype=np.uint16)
            for b in range(self.batch):
                a[b] = table_values(self.hidden_key(which, b), step * self.hidden,
                                    self.hidden, tab)
            out.append(a)
        return tuple(out)

    def recall_weights(self):
        """(W1 bf16 bits [hidden_r][3H], b1 f32 zeros, w2 bf16 bits [hidden_r], b2 0.0)."""
        _, t1, t2 = self.recall_tables()
        fin = self.recall_in_dim()
        W1 = table_values(self.w1_key(), 0, self.recall_hidden * fin, t1).reshape(
            self.recall_hidden, fin)
        w2 = table_values(self.w2_key(), 0, self.recall_hidden, t2)
        b1 = np.zeros(self.recall_hidden, dtype=np.float32)
        return W1, b1, w2, np.float32(0.0)


# --------------------------------------------------------------------------
# needles
# --------------------------------------------------------------------------

def _plant_needles(w: Workload, rows) -> None:
    """One needle per listed row: layer 0, KV head 0, query head 0, at a seeded
    position in [s+1, t0-w] (outside the window and not a sink)."""
    rng = np.random.Generator(np.random.PCG64([w.seed, 7003]))
    tab = normal_table(1.0, "f32")
    for b in rows:
        lo, hi = w.sink + 1, int(w.t0[b]) - w.window
        if hi < lo:
            continue
        pos = int(rng.integers(lo, hi, endpoint=True))
        u = table_values(stream_key(w.seed, KIND_NEEDLE, 0, b), 0, w.d, tab).astype(np.float64)
        u = u / np.linalg.norm(u) * np.sqrt(w.d)
        w.needles.append(Needle(layer=0, row=b, kv_head=0, q_head=0, position=pos,
                                key=w._round(u)))


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------

def tiny_fp32() -> Workload:
    """fp32, 1 layer, batch 2, 2 query heads / 1 KV head, head_dim 64,
    contexts 40 and 64, s=4, w=16, 32 decode steps, fixed scores (+1, -1),
    one needle per row with raw dot +8 against query head 0."""
    w = Workload(name="tiny_fp32", dtype="f32", layers=1, batch=2, hq=2, hkv=1, d=64,
                 sink=4, window=16, block_size=16, t0=np.array([40, 64], np.int64),
                 steps=32, seed=0, sigma_kv=1.0, sigma_q=1.0,
                 fixed_scores=np.array([1.0, -1.0], np.float32), needles_on=True)
    _plant_needles(w, range(w.batch))
    return w


def ctx16k(batch: int = 8, steps: int = 1) -> Workload:
    """bf16, 1 layer, batch 8, 16/8 heads, d=128, every context 16384, paged
    block 16, K/V ~ N(0,1)*0.5, flags Bernoulli(0.41) per row, one needle per
    flagged row. `steps` > 1 continues the same requests (t grows by one per
    step)."""
    w = Workload(name="ctx16k_b8", dtype="bf16", layers=1, batch=batch, hq=16, hkv=8, d=128,
                 sink=4, window=2048, block_size=16,
                 t0=np.full(batch, 16384, np.int64), steps=steps, seed=1,
                 flag_rate=0.41, flag_per="row", needles_on=True)
    f = w.flags()[0]
    _plant_needles(w, [b for b in range(batch) if f[b]])
    return w


def ctx128k(steps: int = 1024, layers: int = 28, context: int = 131072,
            rate: float = 0.125) -> Workload:
    """bf16, batch 1, 28 layers, 16/8 heads, d=128, t = 131072 at the first
    step, 1024 decode steps, Full calls Bernoulli(0.125) per step. `context`
    and `rate` give the same request at another length or call rate."""
    name = ("ctx128k_b1_l28" if (context, rate, layers) == (131072, 0.125, 28)
            else f"ctx{context}_rho{rate:g}_b1_l{layers}")
    return Workload(name=name, dtype="bf16", layers=layers, batch=1, hq=16, hkv=8,
                    d=128, sink=4, window=2048, block_size=16,
                    t0=np.array([context], np.int64), steps=steps, seed=2,
                    flag_rate=rate, flag_per="step")


MIXED_RATES = (0.0, 0.125, 0.41, 1.0)


def mixed_batch(rate: float, batch: int = 32, steps: int = 1) -> Workload:
    """bf16, batch 32, contexts uniform in [4096, 65536], 16/8 heads, d=128,
    paged block 16, Full calls Bernoulli(rate) per row, append inside the step."""
    rng = np.random.Generator(np.random.PCG64([3, 7004]))
    t0 = rng.integers(4096, 65536, endpoint=True, size=batch).astype(np.int64)
    sub = MIXED_RATES.index(rate) if rate in MIXED_RATES else 99
    return Workload(name=f"mixed_b{batch}_rho{rate:g}", dtype="bf16", layers=1, batch=batch,
                    hq=16, hkv=8, d=128, sink=4, window=2048, block_size=16, t0=t0,
                    steps=steps, seed=3 * 1000 + sub, flag_rate=rate, flag_per="row")


def recall_step(ctx: int, batch: int = 16, steps: int = 1) -> Workload:
    """bf16, batch 16, hidden 2048, recall MLP 6144 -> 4096 -> 1 (GELU),
    Xavier-uniform weights, N(0,1) hidden states, theta = 0, 16/8 heads, d=128,
    every context ``ctx`` (4096 or 131072)."""
    return Workload(name=f"recall_b{batch}_ctx{ctx}", dtype="bf16", layers=1, batch=batch,
                    hq=16, hkv=8, d=128, sink=4, window=2048, block_size=16,
                    t0=np.full(batch, ctx, np.int64), steps=steps, seed=4, recall=True)


def custom(name: str, *, dtype="bf16", layers=1, batch=None, hq=4, hkv=2, d=128, sink=4,
           window=64, block_size=16, t0=(100, 37), steps=1, seed=11, sigma_kv=0.5,
           flag_rate=None, flag_per="row", fixed_scores=None, recall=False, hidden=2048,
           recall_hidden=4096) -> Workload:
    """Free-form workload for edge cases (ragged tails, t <= s+w, tiny windows)."""
    t0 = np.asarray(t0, np.int64).reshape(-1)
    if batch is None:
        batch = int(t0.size)
    if t0.size == 1 and batch > 1:
        t0 = np.repeat(t0, batch)
    if t0.size != batch:
        raise ValueError("t0 needs one context length per row")
    return Workload(name=name, dtype=dtype, layers=layers, batch=batch, hq=hq, hkv=hkv, d=d,
                    sink=sink, window=window, block_size=block_size,
                    t0=np.asarray(t0, np.int64), steps=steps, seed=seed, sigma_kv=sigma_kv,
                    flag_rate=flag_rate, flag_per=flag_per,
                    fixed_scores=None if fixed_scores is None else np.asarray(fixed_scores, np.float32),
                    recall=recall, hidden=hidden, recall_hidden=recall_hidden)
