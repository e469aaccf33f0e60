"""HARD-KV decode step: plain, slow, fp64 CPU oracle.  TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's ``cpu_baseline`` /
reference leg may import this module. It shares no code with the CUDA library
(``attention_kv_head_b200``) and imports nothing from it; inputs are plain numpy
arrays holding the exact values the GPU receives (storage-rounded, widened to
float64).

Source: "HARD-KV: Head-Adaptive Regularization for Decoding-time KV Compression"
(gist.science summaries, Italian / Portuguese / Korean technical summaries, sec. 2
"Metodologia"): A. cascade cache (Dense / Sparse / Condensed tiers, four-stage
pipeline), B. Logits Calibration + calibrated top-p, C. Index Regularization
(Rewrite Cache, Flatten Index to the maximum length). The pages state no formulas;
every formula below is a stated reading, listed in the repository's design notes:

  score      s_j = max_{g in G(h)} (q_g . k_j) / sqrt(d)        (sec. 2.B "max-pooled logits")
  calibrate  p_j = exp((s_j - max s)/tau) / sum_i exp((s_i - max s)/tau)
             over the head's Sparse candidates                    (sec. 2.B temperature)
  top-p      order by (s desc, position asc); keep the shortest prefix whose
             mass >= p (p >= 1 keeps all); clamp to the capacity  (sec. 2.A Tier 2)
  regularize kept rows in ascending position order, idx = position,
             index padded with -1 to the capacity                 (sec. 2.C Rewrite / Flatten)
  flatten    the heads' index lists end to end, offsets = exclusive running sum of
  (sum form) the kept counts                                       (sec. 2.C Flatten to the sum)
  condense   oldest Sparse block -> EVICT (drop) or MERGE: each token, in position
             order, into the non-sink slot of highest cosine similarity (ties -> lowest
             slot); k,v <- (w k + x)/(w+1) computed in float64, rounded to the
             storage dtype; w += 1                                 (sec. 2.A Tier 3)
  attention one softmax over Dense U kept U Condensed, Condensed logits + ln w
  boundaries append at pos = len; len += 1; when len - d_lo >= W + block the block
             [d_lo, d_lo+block) moves Dense->Sparse and [s_lo, s_lo+block)
             moves Sparse->Condensed                               (sec. 2.A stages 1, 4)
  entropy    tau_h solves H(softmax(s / tau)) = mean_g H(softmax_j(q_g . k_j / sqrt(d)))
  -matched   over the candidates (bisection on ln tau): the calibrated distribution
  tau        carries the raw attention's entropy     (sec. 2.A Tier 2 "budget based on
             attention entropy"; sec. 2.B; sec. 3 "mapping onto the raw attention")
  top-k      the k best scores, ties to the lower position: the fixed-budget
             selection the pages compare against               (sec. 2.B, sec. 4)
  MTI        per head, rewrite the kept rows or load them in place: rewrite when the
             rewrite's one-off bytes cost less than the scattered-read surcharge over
             the steps the layout lives, with budget thresholds L_lower / L_upper
                                                                   (sec. 2.C trade-off)

Parity pins: every function here is pinned by tests/test_oracle_pins.py against
closed forms, library routines, brute force on tiny inputs and invariants.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

F32, BF16 = "f32", "bf16"
EVICT, MERGE = 0, 1


# ----------------------------------------------------------------------------
# storage rounding (the cache stores K/V in the configured dtype)
# ----------------------------------------------------------------------------

def round_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype (round to nearest, ties to even),
    returned as float64. bf16 keeps 8 significant bits; fp32 keeps 24."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == F32:
        return x.astype(np.float32).astype(np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    m, e = np.frexp(x[nz])              # x = m * 2^e, 0.5 <= |m| < 1
    scale = np.ldexp(1.0, e - 8)         # unit in the last of 8 significant bits
    out[nz] = np.rint(x[nz] / scale) * scale
    return out


# ----------------------------------------------------------------------------
# stage 2a: importance score (max-pooled logits over the GQA group)
# ----------------------------------------------------------------------------

def score(q_group: np.ndarray, k_rows: np.ndarray) -> np.ndarray:
    """s_j = max_g (q_g . k_j) / sqrt(d) for every candidate row j.

    q_group [G, d], k_rows [L, d] (float64) -> [L] float64.
    HARD-KV sec. 2.B: the importance metric is the max-pooled attention logit; the
    pooling runs over the query heads that share KV head h."""
    d = q_group.shape[1]
    if k_rows.shape[0] == 0:
        return np.zeros(0, np.float64)
    logits = k_rows @ q_group.T / math.sqrt(d)          # [L, G]
    return logits.max(axis=1)


# ----------------------------------------------------------------------------
# stage 2b: Logits Calibration
# ----------------------------------------------------------------------------

def calibrate(scores: np.ndarray, tau: float) -> np.ndarray:
    """p_j = softmax(s / tau)_j over the head's candidates (sec. 2.B: temperature
    applied to the attention-score distribution; order of s is preserved)."""
    if scores.size == 0:
        return np.zeros(0, np.float64)
    z = (scores - scores.max()) / float(tau)
    e = np.exp(z)
    return e / e.sum()


# ----------------------------------------------------------------------------
# stage 2c: calibrated top-p with capacity clamp
# ----------------------------------------------------------------------------

@dataclass
class Selection:
    kept: np.ndarray          # local indices (0..L-1) kept, ascending
    order: np.ndarray         # local indices by (s desc, position asc)
    k_mass: int               # prefix length from the mass rule (before the clamp)
    k: int                    # kept count after the clamp
    clamped: bool
    probs: np.ndarray         # calibrated p_j
    cum: np.ndarray           # cumulative mass along `order`

    @property
    def p_theta(self) -> float:
        """Calibrated probability of the last kept token (the threshold token)."""
        return float(self.probs[self.order[self.k - 1]]) if self.k > 0 else 0.0

    def s_k(self, k: int | None = None) -> float:
        k = self.k if k is None else k
        return float(self.cum[k - 1]) if k > 0 else 0.0


def top_p(scores: np.ndarray, tau: float, p: float, cap: int) -> Selection:
    """Shortest (s desc, position asc) prefix whose calibrated mass reaches p; p >= 1
    keeps every candidate; then at most `cap` are kept (the best `cap`).

    HARD-KV sec. 2.A (Tier 2: calibrated top-p keeps the high-information pairs) and
    sec. 2.B (one top-p budget over calibrated distributions)."""
    L = scores.size
    probs = calibrate(scores, tau)
    order = np.lexsort((np.arange(L), -scores))          # s desc, then position asc
    cum = np.cumsum(probs[order])
    p = float(np.float32(p))
    if L == 0:
        k_mass = 0
    elif p >= 1.0:
        k_mass = L
    else:
        k_mass = int(np.argmax(cum >= p)) + 1 if (cum >= p).any() else L
    k = min(k_mass, cap)
    kept = np.sort(order[:k])
    return Selection(kept, order, k_mass, k, k_mass > cap, probs, cum)


def allowed_flips(sel: Selection, p: float, gpu_kept: np.ndarray, eps: float = 1e-6):
    """Whether a kept set computed in lower precision may differ from the oracle's.

    Differences are allowed only where rounding can decide them:
      * same count k: swapped tokens all have |p_j - p_theta| <= eps (near-equal
        probabilities at the threshold ordered differently);
      * count k+1: the oracle's prefix mass S_k is within eps of p, and the extra token
        is the rank-(k+1) token or a near-threshold swap;
      * count k-1: S_{k-1} is within eps of p, and the missing token is the rank-k token
        or a near-threshold swap.
    Returns (ok, number of differing tokens)."""
    L = sel.probs.size
    mine = np.zeros(L, bool)
    mine[sel.kept] = True
    theirs = np.zeros(L, bool)
    theirs[np.asarray(gpu_kept, dtype=np.int64)] = True
    diff = np.nonzero(mine ^ theirs)[0]
    if diff.size == 0:
        return True, 0
    rank = np.empty(L, np.int64)
    rank[sel.order] = np.arange(L)
    p32 = float(np.float32(p))
    k, n_g, pth = sel.k, int(theirs.sum()), sel.p_theta
    if n_g == k:
        edge = None
    elif n_g == k + 1 and not sel.clamped and sel.s_k() - p32 <= eps:
        edge = k                      # 0-based rank of the extra token
    elif n_g == k - 1 and p32 - sel.s_k(k - 1) <= eps:
        edge = k - 1                  # 0-based rank of the missing token
    else:
        return False, int(diff.size)
    for j in diff:
        if not (abs(sel.probs[j] - pth) <= eps or rank[j] == edge):
            return False, int(diff.size)
    return True, int(diff.size)


# ----------------------------------------------------------------------------
# stage 2c': the fixed-budget alternative (top-k)
# ----------------------------------------------------------------------------

def top_k(scores: np.ndarray, k: int) -> Selection:
    """Keep the min(k, L) candidates first in the (s desc, position asc) order: the
    fixed-budget selection (the same k for every head) that the pages contrast with
    calibrated top-p (sec. 2.B "Top-k vs. Top-p"; sec. 4 fixed-budget baselines).
    Nothing is clamped: k is the budget itself."""
    L = scores.size
    order = np.lexsort((np.arange(L), -scores))
    kk = min(int(k), L)
    probs = calibrate(scores, 1.0)
    return Selection(np.sort(order[:kk]), order, kk, kk, False, probs, np.cumsum(probs[order]))


def allowed_flips_topk(scores: np.ndarray, sel: Selection, gpu_kept: np.ndarray,
                       eps: float):
    """Whether a top-k set chosen on lower-precision scores may differ from the oracle's:
    the count must be the same, and every differing token's score must lie within `eps`
    of the score of the oracle's last kept token (rank k), where rounding of the scores
    can reorder it. Returns (ok, number of differing tokens)."""
    L = scores.size
    mine = np.zeros(L, bool)
    mine[sel.kept] = True
    theirs = np.zeros(L, bool)
    theirs[np.asarray(gpu_kept, dtype=np.int64)] = True
    diff = np.nonzero(mine ^ theirs)[0]
    if diff.size == 0:
        return True, 0
    if theirs.sum() != sel.k or sel.k == 0:
        return False, int(diff.size)
    s_theta = scores[sel.order[sel.k - 1]]
    return bool(np.all(np.abs(scores[diff] - s_theta) <= eps)), int(diff.size)


# ----------------------------------------------------------------------------
# stage 2b': entropy-matched Logits Calibration
# ----------------------------------------------------------------------------

def entropy(probs: np.ndarray) -> float:
    """Shannon entropy -sum p ln p (nats) of a probability vector (0 ln 0 = 0)."""
    p = probs[probs > 0]
    return float(-(p * np.log(p)).sum())


def attention_entropy(q_group: np.ndarray, k_rows: np.ndarray) -> float:
    """Mean over the group's queries g of the entropy of the raw attention of q_g over
    the candidate rows: H(softmax_j(q_g . k_j / sqrt(d))). The target of the
    entropy-matched calibration (sec. 2.A Tier 2: a head-adaptive budget based on
    the attention entropy)."""
    if k_rows.shape[0] == 0:
        return 0.0
    d = q_group.shape[1]
    logits = k_rows @ q_group.T / math.sqrt(d)          # [L, G]
    return float(np.mean([entropy(calibrate(logits[:, g], 1.0))
                          for g in range(q_group.shape[0])]))


TAU_MIN, TAU_MAX = 2.0 ** -6, 2.0 ** 6


def entropy_matched_tau(scores: np.ndarray, target: float, iters: int = 200) -> float:
    """The temperature tau in [TAU_MIN, TAU_MAX] with H(softmax(s / tau)) = target.

    Reading of sec. 2.B ("maps the distribution of a selection strategy onto a
    normalised softmax by adjusting the temperature ... preserving order") and sec. 3
    ("mapping the distribution alteration onto the raw attention distribution"): the
    temperature is chosen so that the calibrated distribution of the importance scores
    has the entropy of the raw attention. H(softmax(s/tau)) grows with tau, so the root
    is found by bisection on ln tau; the ends of the range are returned when the target
    lies outside what the range can reach. No candidates or one candidate: tau = 1."""
    if scores.size <= 1:
        return 1.0
    lo, hi = math.log(TAU_MIN), math.log(TAU_MAX)
    if entropy(calibrate(scores, TAU_MAX)) <= target:
        return TAU_MAX
    if entropy(calibrate(scores, TAU_MIN)) >= target:
        return TAU_MIN
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if entropy(calibrate(scores, math.exp(mid))) < target:
            lo = mid
        else:
            hi = mid
    return math.exp(0.5 * (lo + hi))


# ----------------------------------------------------------------------------
# stage 3 policy: Rewrite Cache or Sparse Loading (Memory-Time Integral)
# ----------------------------------------------------------------------------

def mti_rewrite(n: int, reuse_steps: int, l_lower: int, l_upper: int,
                gather_surcharge: float, write_cost: float = 1.0) -> bool:
    """True: rewrite the head's n kept rows into the compact layout; False: load them in
    place from the raw rows through the flattened index (sec. 2.C: Rewrite Cache vs.
    Sparse Loading, chosen per head by a Memory-Time Integral that weighs the one-off
    rewrite against the per-step decode gain, with budget thresholds L_lower, L_upper).

    Reading: a kept row costs 1 per byte to read from a contiguous layout and
    1 + gather_surcharge per byte to read scattered; a rewrite costs write_cost per byte
    once. Over the `reuse_steps` later steps that read the same selection, rewriting
    pays when write_cost < reuse_steps * gather_surcharge (the row count n cancels).
    Budgets below L_lower are always loaded in place, budgets above L_upper always
    rewritten."""
    if n < l_lower:
        return False
    if n > l_upper:
        return True
    return write_cost < reuse_steps * gather_surcharge


# ----------------------------------------------------------------------------
# stage 3: Index Regularization (Rewrite Cache, index flattened to the capacity)
# ----------------------------------------------------------------------------

def regularize(mask: np.ndarray, positions: np.ndarray, k_rows: np.ndarray,
               v_rows: np.ndarray, cap: int):
    """Kept rows moved to slots 0..n-1 in ascending position order; idx = position;
    slots n..cap-1 carry idx -1 (sec. 2.C Rewrite Cache + Flatten Index to max length).
    A mask with more than `cap` bits keeps its first `cap` in position order."""
    sel = np.nonzero(mask)[0][:cap]
    n = sel.size
    idx = np.full(cap, -1, np.int64)
    idx[:n] = positions[sel]
    return n, idx, k_rows[sel], v_rows[sel]


def flatten_sum(index_lists):
    """Flatten Index to the sum of the lengths (sec. 2.C: indices are regularized either
    to the maximum length -- `regularize`'s padded [Cap] rows -- or to their sum). The
    heads' kept-position lists are laid end to end in head order (b major, then h);
    offsets[u] counts the entries before head u, offsets[U] all of them."""
    offsets = [0]
    flat = []
    for lst in index_lists:
        for pos in lst:
            flat.append(int(pos))
        offsets.append(offsets[-1] + len(lst))
    return np.array(offsets, np.int64), np.array(flat, np.int64)


# ----------------------------------------------------------------------------
# stage 4: Condensed tier (eviction / weighted merge)
# ----------------------------------------------------------------------------

@dataclass
class MergeLog:
    slots: list = field(default_factory=list)     # chosen slot per merged token
    gaps: list = field(default_factory=list)      # top-1 minus top-2 cosine


def cosine(a: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """cos(a, rows_i) = a.rows_i / (|a| |rows_i|), 0 where a norm is zero."""
    num = rows @ a
    den = np.sqrt((rows * rows).sum(axis=1) * float(a @ a))
    out = np.zeros(rows.shape[0])
    ok = den > 0
    out[ok] = num[ok] / den[ok]
    return out


def merge_block(blk_k, blk_v, cd_k, cd_v, cd_w, n_sink: int, dtype: str, log=None):
    """Weighted merge of one outgoing block into the Condensed slots (sec. 2.A Tier 3).

    For each token x of the block in position order: s* = argmax cosine(k_x, k_s) over
    slots s >= n_sink with w_s > 0 (ties -> lowest s); then
    k_s* <- (w k_s* + k_x) / (w + 1), v_s* likewise (float64, rounded to the storage
    dtype), w_s* <- w + 1. Arrays are updated in place."""
    C = cd_w.size
    cand = (np.arange(C) >= n_sink) & (cd_w > 0)
    if not cand.any():
        return
    for t in range(blk_k.shape[0]):
        kx, vx = blk_k[t], blk_v[t]
        cos = np.full(C, -np.inf)
        cos[cand] = cosine(kx, cd_k[cand])
        s = int(np.argmax(cos))                     # first maximum -> lowest slot
        if log is not None:
            srt = np.sort(cos[cand])[::-1]
            log.slots.append(s)
            log.gaps.append(float(srt[0] - srt[1]) if srt.size > 1 else math.inf)
        w = float(cd_w[s])
        cd_k[s] = round_storage((w * cd_k[s] + kx) / (w + 1.0), dtype)
        cd_v[s] = round_storage((w * cd_v[s] + vx) / (w + 1.0), dtype)
        cd_w[s] = np.float32(w + 1.0)


# ----------------------------------------------------------------------------
# decode attention over the three tiers
# ----------------------------------------------------------------------------

def attention(q_group: np.ndarray, k_rows: np.ndarray, v_rows: np.ndarray,
              bias: np.ndarray) -> np.ndarray:
    """o_g = sum_t softmax_t(q_g . k_t / sqrt(d) + bias_t) v_t, one joint softmax.
    q_group [G,d], k/v [T,d], bias [T] -> [G,d]."""
    d = q_group.shape[1]
    logits = q_group @ k_rows.T / math.sqrt(d) + bias[None, :]       # [G, T]
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    return (e @ v_rows) / e.sum(axis=1, keepdims=True)


# ----------------------------------------------------------------------------
# one (sequence, KV head) unit through decode steps
# ----------------------------------------------------------------------------

@dataclass
class Params:
    head_dim: int
    group: int
    dense_window: int
    condensed_slots: int
    block: int
    sparse_cap: int
    n_sink: int
    dtype: str
    condense_mode: int


@dataclass
class StepOut:
    moved: bool
    reselected: bool
    sel: Selection | None
    n: int
    idx: np.ndarray
    out: np.ndarray               # [G, d]
    merge: MergeLog | None


class Unit:
    """One (sequence b, KV head h) of the cascade cache, positions stored by index
    (the oracle needs no ring: raw rows are addressed by absolute position)."""

    def __init__(self, prm: Params, k_pos: np.ndarray, v_pos: np.ndarray,
                 cd_k: np.ndarray, cd_v: np.ndarray, cd_w: np.ndarray,
                 len0: int, d_lo: int, s_lo: int, capacity: int):
        self.prm = prm
        d = prm.head_dim
        self.K = np.zeros((capacity, d))
        self.V = np.zeros((capacity, d))
        self.K[:k_pos.shape[0]] = k_pos
        self.V[:v_pos.shape[0]] = v_pos
        self.cd_k, self.cd_v = cd_k.copy(), cd_v.copy()
        self.cd_w = cd_w.astype(np.float64).copy()
        self.len, self.d_lo, self.s_lo = int(len0), int(d_lo), int(s_lo)
        self.n = 0
        self.idx = np.full(prm.sparse_cap, -1, np.int64)
        self.sp_k = np.zeros((0, d))
        self.sp_v = np.zeros((0, d))

    # stage 1 -----------------------------------------------------------------
    def append(self, k_new: np.ndarray, v_new: np.ndarray) -> bool:
        """Linear append at pos = len (sec. 2.A stage 1); block move when the Dense
        window holds W + block tokens: Dense->Sparse and Sparse->Condensed shift by one
        block."""
        P = self.prm
        self.K[self.len] = k_new
        self.V[self.len] = v_new
        self.len += 1
        if self.len - self.d_lo >= P.dense_window + P.block:
            self.d_lo += P.block
            self.s_lo += P.block
            return True
        return False

    # stage 4 -----------------------------------------------------------------
    def condense(self, log: MergeLog | None):
        """The block [s_lo - block, s_lo) that just left the Sparse tier is evicted or
        merged (sec. 2.A stage 4)."""
        P = self.prm
        if P.condense_mode == MERGE:
            a = self.s_lo - P.block
            merge_block(self.K[a:self.s_lo], self.V[a:self.s_lo], self.cd_k, self.cd_v,
                        self.cd_w, P.n_sink, P.dtype, log)

    # stages 2-3 --------------------------------------------------------------
    def select(self, q_group: np.ndarray, tau: float, p: float, rule: str = "topp",
               k: int | None = None, calibration: str = "tau") -> Selection:
        """Score the Sparse candidates and keep a subset: rule "topp" = calibrated top-p
        (calibration "tau": the given temperature; "entropy": the entropy-matched one),
        rule "topk" = the k best scores. The temperature used is kept in self.tau."""
        P = self.prm
        pos = np.arange(self.s_lo, self.d_lo)
        s = score(q_group, self.K[self.s_lo:self.d_lo])
        if rule == "topk":
            sel = top_k(s, min(int(k), P.sparse_cap))
        else:
            if calibration == "entropy":
                tau = entropy_matched_tau(
                    s, attention_entropy(q_group, self.K[self.s_lo:self.d_lo]))
            sel = top_p(s, tau, p, P.sparse_cap)
        self.tau = tau
        self.scores = s
        mask = np.zeros(pos.size, bool)
        mask[sel.kept] = True
        self.n, self.idx, self.sp_k, self.sp_v = regularize(
            mask, pos, self.K[self.s_lo:self.d_lo], self.V[self.s_lo:self.d_lo],
            P.sparse_cap)
        return sel

    def union(self, kept_positions: np.ndarray | None = None):
        """K, V and logit bias of Dense U kept-Sparse U Condensed (w > 0)."""
        P = self.prm
        if kept_positions is None:
            live = self.idx[:self.n] >= self.s_lo
            ks, vs = self.sp_k[live], self.sp_v[live]
        else:
            ks, vs = self.K[kept_positions], self.V[kept_positions]
        kd, vd = self.K[self.d_lo:self.len], self.V[self.d_lo:self.len]
        live_c = self.cd_w > 0
        kc, vc = self.cd_k[live_c], self.cd_v[live_c]
        bias = np.concatenate([np.zeros(ks.shape[0] + kd.shape[0]),
                               np.log(self.cd_w[live_c])])
        return (np.concatenate([ks, kd, kc]), np.concatenate([vs, vd, vc]), bias)

    def attend(self, q_group: np.ndarray) -> np.ndarray:
        K, V, bias = self.union()
        return attention(q_group, K, V, bias)

    def step(self, q_group, k_new, v_new, tau: float, p: float, reselect: str = "all",
             rule: str = "topp", k: int | None = None, calibration: str = "tau"):
        """One decode step: append, condense (block steps), select (if this unit
        reselects: "all" = every step, "moved" = on its block move; rule / k /
        calibration as in select), attend."""
        moved = self.append(k_new, v_new)
        log = None
        if moved:
            log = MergeLog()
            self.condense(log)
        sel = None
        if reselect == "all" or (reselect == "moved" and moved):
            sel = self.select(q_group, tau, p, rule, k, calibration)
        out = self.attend(q_group)
        return StepOut(moved, sel is not None, sel, self.n, self.idx.copy(), out, log)


def full_attention(q_group: np.ndarray, k_all: np.ndarray, v_all: np.ndarray) -> np.ndarray:
    """Exact attention over every position (no compression)."""
    return attention(q_group, k_all, v_all, np.zeros(k_all.shape[0]))
