"""Plain, slow, obviously-correct float64 restatement of On-Demand Attention's
decode-time hot path.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Every function follows one passage of the pages (abbreviations [SUM], [CARD],
[EXPL] are defined in ``oracle/__init__.py``). Inputs arrive as numpy arrays
already widened exactly to float64 from the stored bf16/fp32 bytes; nothing
here blocks, fuses or reorders beyond the definitions.

Parity status
  full_access_set, local_access_set ... pinned (brute force + closed forms)
  attend ............................... pinned (special cases, closed forms, invariants)
  gate ................................. pinned (bit-exact edge values)
  signed_log, huber1 ................... pinned (closed forms, invariants)
  access_gain, penalized_step_loss ..... pinned (closed forms)
  delta_F and the FLOP counter ......... pinned (exact integer identity; pages' ratios, loose)
  gelu_erf ............................. pinned (erf closed-form values)
  range_access_set, range_attention .... pinned (brute force, Full/window/one-position cases)
  budget_count, select_top,
  net_gain_per_position,
  random_expected_net_gain ............. pinned (brute force over all k-subsets, closed forms)
  recall_score ......................... parity unpinned: the pages give the
      head's inputs and parameter count but not its architecture; the
      6144 -> 4096 -> 1 GELU MLP is this library's stated choice. Pinned only
      through special cases (W1 = 0, a single hidden unit).
"""

from __future__ import annotations

import math
from fractions import Fraction
from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "full_access_set", "local_access_set", "attend", "FlopCounter",
    "local_attention", "full_attention", "gelu_erf", "recall_score", "gate",
    "select_output", "decode_step", "signed_log", "huber1",
    "recall_regression_loss", "access_gain", "penalized_step_loss",
    "best_action", "regression_target", "attention_flops", "recall_flops",
    "delta_F", "model_step_flops", "oda_flop_fraction",
    "range_access_set", "range_attention",
    "budget_count", "select_top", "net_gain_per_position", "random_expected_net_gain",
]


# ---------------------------------------------------------------------------
# Access sets. [SUM] Methodology / Local-First Decoding, access-set equation:
# the Full set is every position 1..t; the Local set is the first min(s, t)
# positions together with the most recent positions max(1, t-w+1)..t.
# ---------------------------------------------------------------------------

def full_access_set(t: int) -> set:
    """S^F_t = {1, ..., t}."""
    return set(range(1, t + 1))


def local_access_set(t: int, s: int, w: int) -> set:
    """S^L_t = {1, ..., min(s, t)} union {max(1, t-w+1), ..., t} (a set union:
    a position in both parts appears once)."""
    sinks = set(range(1, min(s, t) + 1))
    window = set(range(max(1, t - w + 1), t + 1))
    return sinks | window


# ---------------------------------------------------------------------------
# FLOP accounting used by the savings model ([SUM] Computational Savings).
# Attention over a key set S costs 2|S|d multiply-adds-as-FLOPs for q.k and
# 2|S|d for the weighted sum of values, per query head.
# ---------------------------------------------------------------------------

class FlopCounter:
    """Accumulates FLOPs executed by the oracle, by category."""

    def __init__(self) -> None:
        self.by: Dict[str, int] = {}

    def add(self, what: str, n: int) -> None:
        self.by[what] = self.by.get(what, 0) + int(n)

    def total(self) -> int:
        return sum(self.by.values())


# ---------------------------------------------------------------------------
# Softmax attention over an explicit set of positions.
# Local and Full are "two access modes of the same frozen backbone"
# ([SUM] Methodology / Local-First Decoding): the same attention, restricted
# to S^L_t or over S^F_t. Readings used (the pages are silent):
#   scale 1/sqrt(d); query head h reads KV head floor(h / (Hq/Hkv)).
# ---------------------------------------------------------------------------

def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, positions: Iterable[int],
           flops: Optional[FlopCounter] = None, what: str = "attn") -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of every query head over ``positions``.

    q: [Hq][d]; K, V: [Hkv][P][d] with row p-1 holding position p.
    Returns (out [Hq][d], lse [Hq]) where lse = log sum_j exp(q.k_j / sqrt(d)).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    hq, d = q.shape
    hkv = K.shape[0]
    group = hq // hkv
    pos = sorted(positions)
    if len(pos) == 0:
        raise ValueError("attention over an empty set is undefined")
    rows = np.asarray(pos, dtype=np.int64) - 1
    out = np.empty((hq, d), dtype=np.float64)
    lse = np.empty(hq, dtype=np.float64)
    for h in range(hq):
        g = h // group
        z = (K[g, rows] @ q[h]) / math.sqrt(d)
        m = z.max()
        e = np.exp(z - m)
        denom = e.sum()
        out[h] = (e @ V[g, rows]) / denom
        lse[h] = m + math.log(denom)
    if flops is not None:
        flops.add(what, 4 * len(pos) * d * hq)
    return out, lse


def local_attention(q, K, V, t: int, s: int, w: int, flops: Optional[FlopCounter] = None):
    """F^L: attention restricted to S^L_t ([SUM] Methodology / Local-First Decoding)."""
    return attend(q, K, V, local_access_set(t, s, w), flops, "local")


def full_attention(q, K, V, t: int, flops: Optional[FlopCounter] = None):
    """F: attention over S^F_t, run only for requests the gate flags
    ([SUM] Methodology / Local-First Decoding)."""
    return attend(q, K, V, full_access_set(t), flops, "full")


# ---------------------------------------------------------------------------
# Range-restricted ("focus") attention. [DA-1] (zhichai.net post on
# Declarative Attention), "Three Attention Modes", and [DA-2] (kongchang.com
# article), "<focus> Mode: Precise Region Targeting": attention narrowed to one
# region of the context, reading only that region's KV. Reading used (the
# pages give no formula): the region is the half-open position range
# [lo, hi) named by the caller, and the attention is the same softmax
# attention restricted to it.
# ---------------------------------------------------------------------------

def range_access_set(lo: int, hi: int) -> set:
    """{lo, ..., hi-1}."""
    return set(range(lo, hi))


def range_attention(q, K, V, lo: int, hi: int, flops: Optional[FlopCounter] = None):
    """Attention over the positions of [lo, hi) only."""
    return attend(q, K, V, range_access_set(lo, hi), flops, "range")


# ---------------------------------------------------------------------------
# Recall head R_psi(h_{t-1}, E(x_t), h^L_t) ([SUM] Methodology, recall-score
# equation; [EXPL] Jargon / Recall head). The pages fix the three inputs and
# their order, not the architecture. This library's head: concat -> Linear ->
# GELU (erf form) -> Linear to one score.
# ---------------------------------------------------------------------------

def gelu_erf(u: np.ndarray) -> np.ndarray:
    """GELU(u) = u * Phi(u) = u * (1 + erf(u / sqrt 2)) / 2."""
    u = np.asarray(u, dtype=np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return u * 0.5 * (1.0 + erf(u / math.sqrt(2.0)))


def recall_score(h_prev: np.ndarray, emb: np.ndarray, h_local: np.ndarray,
                 W1: np.ndarray, b1: np.ndarray, w2: np.ndarray, b2: float,
                 flops: Optional[FlopCounter] = None) -> np.ndarray:
    """q_t for every row: w2 . GELU(W1 [h_{t-1}; E(x_t); h^L_t] + b1) + b2.

    h_prev, emb, h_local: [B][H]; W1: [hidden][3H]; b1, w2: [hidden]; b2 scalar.
    Returns scores [B] (float64).
    """
    x = np.concatenate([np.asarray(h_prev, np.float64), np.asarray(emb, np.float64),
                        np.asarray(h_local, np.float64)], axis=1)
    W1 = np.asarray(W1, np.float64)
    u = x @ W1.T + np.asarray(b1, np.float64)[None, :]
    a = gelu_erf(u)
    score = a @ np.asarray(w2, np.float64) + float(b2)
    if flops is not None:
        flops.add("recall", x.shape[0] * recall_flops(W1.shape[1], W1.shape[0]))
    return score


# ---------------------------------------------------------------------------
# Threshold gate ([SUM] Methodology / Local-First Decoding: recompute with
# Full when q_t > theta, otherwise accept Local; default theta = 0).
# Readings: the comparison is strict and taken in float32 (the precision the
# scores are stored in), so NaN and scores equal to theta are not flagged.
# Flagged row ids are listed in ascending order, the rest of the list is -1.
# ---------------------------------------------------------------------------

def gate(scores: Sequence[float], theta: float = 0.0):
    """Returns (flags uint8 [B], idx int32 [B], count)."""
    s = np.asarray(scores, dtype=np.float32)
    th = np.float32(theta)
    flags = np.zeros(s.shape[0], dtype=np.uint8)
    chosen = []
    for b in range(s.shape[0]):
        if bool(s[b] > th):
            flags[b] = 1
            chosen.append(b)
    idx = np.full(s.shape[0], -1, dtype=np.int32)
    idx[:len(chosen)] = chosen
    return flags, idx, len(chosen)


def select_output(out_local: np.ndarray, out_full: Dict[int, np.ndarray], flags) -> np.ndarray:
    """Flagged rows take the Full output, the others keep Local."""
    out = np.array(out_local, dtype=np.float64, copy=True)
    for b, f in enumerate(flags):
        if f:
            out[b] = out_full[b]
    return out


def decode_step(q: np.ndarray, K_rows, V_rows, t: Sequence[int], s: int, w: int,
                scores: Sequence[float], theta: float = 0.0,
                q_full: Optional[np.ndarray] = None,
                flops: Optional[FlopCounter] = None):
    """One layer of one decode step for a batch.

    q: [B][Hq][d]; K_rows[b], V_rows[b]: [Hkv][P_b][d] holding positions
    1..P_b (P_b >= t[b], the current token already committed); t[b] the
    current position; scores the recall scores fed to the gate.
    Returns dict(local, lse_local, flags, idx, count, full, lse_full, out).
    """
    B = q.shape[0]
    qf = q if q_full is None else q_full
    local = np.empty(q.shape, np.float64)
    lse_local = np.empty(q.shape[:2], np.float64)
    for b in range(B):
        local[b], lse_local[b] = local_attention(q[b], K_rows[b], V_rows[b], int(t[b]), s, w, flops)
    flags, idx, count = gate(scores, theta)
    full, lse_full = {}, {}
    for i in range(count):
        b = int(idx[i])
        full[b], lse_full[b] = full_attention(qf[b], K_rows[b], V_rows[b], int(t[b]), flops)
    return dict(local=local, lse_local=lse_local, flags=flags, idx=idx, count=count,
                full=full, lse_full=lse_full, out=select_output(local, full, flags))


# ---------------------------------------------------------------------------
# Training-side quantities ([SUM] Learning to Predict Recall Benefit).
# ---------------------------------------------------------------------------

def signed_log(u):
    """T(u) = sign(u) * log(1 + |u|) (natural log)."""
    u = np.asarray(u, dtype=np.float64)
    return np.sign(u) * np.log1p(np.abs(u))


def huber1(r):
    """Huber loss with transition point 1: r^2/2 for |r| <= 1, else |r| - 1/2."""
    r = np.abs(np.asarray(r, dtype=np.float64))
    return np.where(r <= 1.0, 0.5 * r * r, r - 0.5)


def recall_regression_loss(q_scores, targets):
    """L(psi): mean over the training positions of Huber_1(q_t - y_t)."""
    q = np.asarray(q_scores, np.float64)
    y = np.asarray(targets, np.float64)
    return float(np.mean(huber1(q - y)))


def access_gain(logp_full, logp_local):
    """g_t = l^L_t - l^F_t = log p^F_t(x_{t+1}) - log p^L_t(x_{t+1})."""
    return np.asarray(logp_full, np.float64) - np.asarray(logp_local, np.float64)


def penalized_step_loss(loss_local, gain, action, lam: float):
    """l_t(a_t) = l^L_t - a_t (g_t - lambda), a_t in {0 (Local), 1 (Full)}."""
    return (np.asarray(loss_local, np.float64)
            - np.asarray(action, np.float64) * (np.asarray(gain, np.float64) - lam))


def best_action(gain, lam: float):
    """The action minimising the penalized loss: Full (1) iff g_t > lambda
    (a tie keeps Local, whose loss is the same)."""
    return (np.asarray(gain, np.float64) > lam).astype(np.uint8)


def regression_target(gain, lam: float = 0.0):
    """y_t = T(g_t - lambda). Reading: the pages name T and the penalty but not
    how they combine; placing lambda inside T makes q_t > 0 (the default
    theta) the same decision as best_action, since T is odd and increasing."""
    return signed_log(np.asarray(gain, np.float64) - lam)


# ---------------------------------------------------------------------------
# Selection at a call budget ([SUM] State-Dependent Access Effectiveness: at a
# 40 % budget the recall head captures a net gain per reference position,
# compared with the expected gain of random selection; Conclusion: an offline
# Oracle that knows the true gains selects better still). Readings used (the
# pages give no formula): a budget b over n positions allows floor(b n) Full
# calls; a policy spends them on the positions with the largest scores (the
# recall head's q_t, or the true gain g_t for the offline Oracle), equal
# scores going to the earlier position and NaN ranking below every number;
# the net gain per reference position is the sum of g_t over the selected
# positions divided by n; random selection spends the same calls on a
# uniformly random subset.
# ---------------------------------------------------------------------------

def budget_count(n: int, budget) -> int:
    """Full calls a budget allows: floor(budget * n), in exact arithmetic."""
    return int(Fraction(budget) * n // 1)


def select_top(scores, k: int) -> np.ndarray:
    """uint8 flags [n]: 1 for the k positions with the largest scores, compared
    as float32 (equal values, +0 and -0 included, go to the lower position;
    NaN ranks below every number)."""
    s = np.asarray(scores, dtype=np.float32)
    n = s.shape[0]
    if not 0 <= k <= n:
        raise ValueError("k outside 0..n")

    def rank_key(i):
        v = float(s[i])
        return (1, 0.0, i) if math.isnan(v) else (0, -v, i)

    order = sorted(range(n), key=rank_key)
    flags = np.zeros(n, dtype=np.uint8)
    for i in order[:k]:
        flags[i] = 1
    return flags


def net_gain_per_position(gain, selected) -> float:
    """(1/n) * sum of g_t over the selected positions."""
    g = np.asarray(gain, np.float64)
    sel = np.asarray(selected).astype(bool)
    return float(g[sel].sum() / g.shape[0])


def random_expected_net_gain(gain, k: int) -> float:
    """Expected net gain per position of k positions drawn uniformly without
    replacement: each position is drawn with probability k/n."""
    g = np.asarray(gain, np.float64)
    n = g.shape[0]
    return float(k / n * g.sum() / n)


# ---------------------------------------------------------------------------
# Savings model ([SUM] Computational Savings):
#   Delta F(n, rho) = (1 - rho) F_Full(n) - F_Local - F_Recall.
# ---------------------------------------------------------------------------

def attention_flops(n_keys: int, d: int, hq: int) -> int:
    """FLOPs of one layer's attention for one request over n_keys keys."""
    return 4 * int(n_keys) * int(d) * int(hq)


def recall_flops(in_dim: int, hidden: int) -> int:
    """FLOPs of the recall MLP for one request (2 per multiply-add)."""
    return 2 * in_dim * hidden + 2 * hidden


def delta_F(F_full_n, F_local, F_recall, rho) -> Fraction:
    """Average per-step savings of ODA relative to always running Full."""
    rho = Fraction(rho)
    return (1 - rho) * Fraction(F_full_n) - Fraction(F_local) - Fraction(F_recall)


def model_step_flops(n: int, *, layers: int, hidden: int, hq: int, hkv: int, d: int,
                     intermediate: int, vocab: int, attn_keys: Optional[int] = None) -> int:
    """Whole-model FLOPs of one decode step of a dense GQA transformer:
    2 per weight multiply-add of the q/k/v/o projections, the gated MLP and
    the vocabulary projection, plus attention over ``attn_keys`` keys
    (n for Full) in every layer."""
    keys = n if attn_keys is None else attn_keys
    proj = hidden * hq * d + 2 * hidden * hkv * d + hq * d * hidden
    mlp = 3 * hidden * intermediate
    dense = 2 * (layers * (proj + mlp) + hidden * vocab)
    return dense + layers * attention_flops(keys, d, hq)


def oda_flop_fraction(n: int, rho, *, s: int, w: int, recall_params: int, **shape) -> float:
    """ODA decoding FLOPs as a fraction of Full's at context n and Full-call
    rate rho: every step pays Local and the recall head; a fraction rho of
    steps also pays Full ([EXPL] How much faster is it in practice?)."""
    f_full = model_step_flops(n, **shape)
    f_local = model_step_flops(n, attn_keys=min(n, s + w), **shape)
    f_recall = 2 * recall_params
    oda = f_local + f_recall + float(rho) * f_full
    return oda / f_full
