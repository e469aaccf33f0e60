"""Seeded synthetic workloads for the HARD-KV decode step.

This module is the one piece shared by the CUDA path's tests/benchmark and the CPU
oracle's tests. It holds the workload recipes (shapes, tier sizes, value
distributions) and a counter-based random generator; it contains none of the
method's arithmetic (no scoring, calibration, selection, compaction, merging or
attention).

Generator (published definitions, written out here):
  * splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): state += 0x9E3779B97F4A7C15, then the xor-shift /
    multiply finaliser with constants 0xBF58476D1CE4E5B9, 0x94D049BB133111EB.
  * Box-Muller (1958): two uniforms (0,1) -> two independent N(0,1) draws
    r*cos(2*pi*u2), r*sin(2*pi*u2) with r = sqrt(-2 ln u1).
Every value is a pure function of (seed, tensor tag, ids, element counter), so any
(sequence, head, position) slice can be regenerated alone: the oracle tests
regenerate only the units they sample.

Workloads (HARD-KV pages: "Riepilogo Tecnico" sec. 2.A cascade cache and sec. 4
long-context >10k-token decoding on Qwen3 models; the AIME/U-Math traces and model
weights are not available, seeded Gaussian tensors of the same head shapes stand in).
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1

# tensor tags (arbitrary distinct constants)
TAG_K, TAG_V, TAG_Q, TAG_TEMP, TAG_LEN, TAG_SPIKE, TAG_SPIKE_NOISE, TAG_MASK, TAG_TAU = (
    0x4B, 0x56, 0x51, 0x54, 0x4C, 0x53, 0x4E, 0x4D, 0x43)

F32, BF16 = "f32", "bf16"
EVICT, MERGE = 0, 1
SELECT_ALL, SELECT_MOVED = 0, 1


def _mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 output finaliser on uint64 arrays (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _mix_int(x: int) -> int:
    z = x & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tag: int, *ids: int) -> int:
    """64-bit key of one independent stream, folded from (seed, tag, ids...)."""
    k = _mix_int(seed * 0x9E3779B97F4A7C15 + tag)
    for i in ids:
        k = _mix_int((k ^ (int(i) & _MASK64)) + 0x9E3779B97F4A7C15)
    return k


def uniform(key: int, counters: np.ndarray) -> np.ndarray:
    """U(0,1) in float64 for the given element counters of stream `key`."""
    with np.errstate(over="ignore"):
        x = np.uint64(key) + (counters.astype(np.uint64) + np.uint64(1)) * GOLDEN
        z = _mix(x)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def normal(key: int, start: int, count: int) -> np.ndarray:
    """`count` N(0,1) float64 draws, elements [start, start+count) of stream `key`.

    Element i uses Box-Muller pair i//2 (cos for even i, sin for odd i); the pair's
    two uniforms are splitmix64 outputs 2m and 2m+1 of the stream. Each pair is
    evaluated once and both of its draws are kept.
    """
    if count <= 0:
        return np.zeros(0, np.float64)
    m0, m1 = start >> 1, (start + count - 1) >> 1
    m = np.arange(m0, m1 + 1, dtype=np.uint64)
    u1 = uniform(key, m * np.uint64(2))
    u2 = uniform(key, m * np.uint64(2) + np.uint64(1))
    r = np.sqrt(-2.0 * np.log(u1))
    th = 2.0 * math.pi * u2
    pairs = np.empty((m.size, 2), np.float64)
    pairs[:, 0] = r * np.cos(th)
    pairs[:, 1] = r * np.sin(th)
    off = start - 2 * m0
    return pairs.reshape(-1)[off:off + count]


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> exact float64 values."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float values to the storage dtype. Returns (raw array, exact float64)."""
    if dtype == F32:
        raw = np.ascontiguousarray(x, dtype=np.float32)
        return raw, raw.astype(np.float64)
    bits = to_bf16_bits(np.asarray(x, dtype=np.float32))
    return bits, bf16_bits_to_f64(bits)


# ----------------------------------------------------------------------------
# Workload recipes
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    """One synthetic decode workload (one attention layer)."""
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: str
    context: int | None          # fixed context; None -> per-sequence lengths
    len_range: tuple[int, int] | None
    dense_window: int
    condensed_slots: int
    block: int
    sparse_cap: int
    p: float | tuple[float, ...]
    steps: int
    select_every: int            # 1 = every step; >1 = reselect a sequence on its block move
    condense_mode: int
    temp_mode: str               # "linear" (0.5*(h+1)) or "loguniform"
    temp_range: tuple[float, float] = (0.5, 4.0)
    spike_frac: float = 0.0
    n_sink: int = 4
    sink_scale: float = 8.0
    seed: int = 0
    ring_rows: int = 0           # 0 -> derived (smallest multiple of 64 that holds the span)
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def units(self) -> int:
        return self.batch * self.n_kv_heads

    def max_len(self) -> int:
        hi = self.context if self.context is not None else self.len_range[1]
        return hi + self.steps - 1

    def derived_ring_rows(self) -> int:
        if self.ring_rows:
            return self.ring_rows
        hi = self.context if self.context is not None else self.len_range[1]
        span = hi - self.condensed_slots + self.block  # [s_lo, len) never exceeds this
        return ((span + 63) // 64) * 64

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS: dict[str, Workload] = {
    # 1 sequence, 4 KV heads x 1 query head, d=64, fp32, 1024 tokens:
    # Dense 64 + Sparse 928 + Condensed 32; head h keys scaled 0.5*(h+1).
    "pr1": Workload("pr1", 1, 4, 4, 64, F32, 1024, None, 64, 32, 16, 928, 0.9, 1, 1,
                    EVICT, "linear"),
    # Llama-3-8B-shaped layer, batch 8, context 8192, one step.
    "llama8b_8k": Workload("llama8b_8k", 8, 32, 8, 128, BF16, 8192, None, 256, 256, 16,
                           7680, 0.9, 1, 1, EVICT, "loguniform", (0.5, 4.0)),
    # Long context: batch 32, context 16384, Cap 25% of context, 64 steps, p swept.
    "long16k": Workload("long16k", 32, 32, 8, 128, BF16, 16384, None, 256, 256, 16,
                        4096, (0.8, 0.9, 0.95), 64, 1, EVICT, "loguniform", (0.5, 4.0)),
    # Continuous batching: batch 64, lengths U[1024, 32768], 256 steps, reselect on
    # each sequence's block move (every 16 steps), weighted merge into 512 slots.
    "contbatch": Workload("contbatch", 64, 32, 8, 128, BF16, None, (1024, 32768), 256, 512,
                          16, 8192, 0.9, 256, 16, MERGE, "loguniform", (0.5, 4.0)),
    # Stress: 40/8 heads, batch 16, context 65536, Dense 512, Condensed 1024, Cap 15%,
    # 10% planted spikes aligned with the first query, temperatures in [0.25, 8].
    "stress64k": Workload("stress64k", 16, 40, 8, 128, BF16, 65536, None, 512, 1024, 16,
                          9840, 0.95, 128, 1, MERGE, "loguniform", (0.25, 8.0),
                          spike_frac=0.1),
    # A profiling case for the weighted merge: llama8b_8k's heads with contbatch's 512
    # Condensed slots, context 2048, MERGE; step 16 moves a block in every sequence.
    "merge_c512": Workload("merge_c512", 8, 32, 8, 128, BF16, 2048, None, 256, 512, 16,
                           1280, 0.9, 17, 1, MERGE, "loguniform", (0.5, 4.0)),
}


def small(name: str = "tiny", **kw) -> Workload:
    """A small workload (several tiles + ragged tails) for oracle-speed parity."""
    base = Workload(name, 2, 8, 2, 128, BF16, 700, None, 48, 24, 16, 600, 0.9, 1, 1, EVICT,
                    "loguniform", (0.5, 4.0))
    return base.with_(**kw)


# ----------------------------------------------------------------------------
# Value generators (pure functions of ids -> slices can be regenerated per unit)
# ----------------------------------------------------------------------------

def seq_lengths(w: Workload) -> np.ndarray:
    """Context length of every sequence at the first step (after its append)."""
    if w.context is not None:
        return np.full(w.batch, w.context, np.int64)
    lo, hi = w.len_range
    u = uniform(stream_key(w.seed, TAG_LEN), np.arange(w.batch, dtype=np.uint64))
    return lo + np.minimum((u * (hi - lo + 1)).astype(np.int64), hi - lo)


def temperature(w: Workload, b: int, h: int) -> float:
    """Key temperature T_{b,h} (float32 value)."""
    if w.temp_mode == "linear":
        return float(np.float32(0.5 * (h + 1)))
    lo, hi = w.temp_range
    u = float(uniform(stream_key(w.seed, TAG_TEMP, b, h), np.zeros(1, np.uint64))[0])
    return float(np.float32(math.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))))


def calibration_taus(w: Workload, lo: float = 0.25, hi: float = 8.0) -> np.ndarray:
    """Caller-supplied calibration temperatures tau[b, h] (float32) for tests of the
    temperature path: log-uniform in [lo, hi] per (sequence, KV head), so values fall on
    both sides of 1, with unit (0, 0) exactly 1."""
    B, H = w.batch, w.n_kv_heads
    u = uniform(stream_key(w.seed, TAG_TAU), np.arange(B * H, dtype=np.uint64)).reshape(B, H)
    t = np.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))).astype(np.float32)
    t[0, 0] = 1.0
    return t


def query_f32(w: Workload, step: int, b: int, qh: int) -> np.ndarray:
    """Query row q[b, qh] of decode step `step` (float32 before storage rounding)."""
    return normal(stream_key(w.seed, TAG_Q, step, b, qh), 0, w.head_dim).astype(np.float32)


def queries(w: Workload, step: int) -> tuple[np.ndarray, np.ndarray]:
    """All queries of one step: (raw storage array [B,Hq,d], exact float64 values)."""
    q = np.stack([np.stack([query_f32(w, step, b, qh) for qh in range(w.n_q_heads)])
                  for b in range(w.batch)])
    return storage(q, w.dtype)


def _spike_dir(w: Workload, b: int, h: int) -> np.ndarray:
    g = w.group
    s = np.zeros(w.head_dim, np.float64)
    for j in range(g):
        raw, exact = storage(query_f32(w, 0, b, h * g + j), w.dtype)
        s += exact
    n = np.linalg.norm(s)
    return s / n if n > 0 else s


def key_rows(w: Workload, b: int, h: int, p0: int, p1: int) -> np.ndarray:
    """Keys of positions [p0, p1) of unit (b,h) as float32 (before storage rounding)."""
    d = w.head_dim
    n = max(p1 - p0, 0)
    z = normal(stream_key(w.seed, TAG_K, b, h), p0 * d, n * d).reshape(n, d)
    pos = np.arange(p0, p0 + n)
    if w.spike_frac > 0:
        u = uniform(stream_key(w.seed, TAG_SPIKE, b, h), pos.astype(np.uint64))
        spike = u < w.spike_frac
        if spike.any():
            noise = normal(stream_key(w.seed, TAG_SPIKE_NOISE, b, h), p0 * d, n * d)
            noise = noise.reshape(n, d)
            z = np.where(spike[:, None],
                         4.0 * math.sqrt(d) * _spike_dir(w, b, h)[None, :] + 0.5 * noise, z)
    z = z * temperature(w, b, h)
    z = np.where((pos < w.n_sink)[:, None], z * w.sink_scale, z)
    return z.astype(np.float32)


def value_rows(w: Workload, b: int, h: int, p0: int, p1: int) -> np.ndarray:
    d = w.head_dim
    n = max(p1 - p0, 0)
    return normal(stream_key(w.seed, TAG_V, b, h), p0 * d, n * d).reshape(n, d).astype(np.float32)


def unit_kv(w: Workload, b: int, h: int, p0: int, p1: int):
    """Keys and values of positions [p0,p1): (k_raw, k_exact, v_raw, v_exact)."""
    kr, ke = storage(key_rows(w, b, h, p0, p1), w.dtype)
    vr, ve = storage(value_rows(w, b, h, p0, p1), w.dtype)
    return kr, ke, vr, ve


def random_mask(w: Workload, b: int, h: int, n: int, frac: float, step: int = 0) -> np.ndarray:
    """Seeded Bernoulli(frac) selection over n Sparse candidates (for component tests)."""
    u = uniform(stream_key(w.seed, TAG_MASK, step, b, h), np.arange(n, dtype=np.uint64))
    return u < frac


# ----------------------------------------------------------------------------
# Initial cache state in the device layout (host arrays), built in parallel
# ----------------------------------------------------------------------------

@dataclass
class InitialState:
    w: Workload
    R: int
    lens: np.ndarray          # [B] context at the first step (after its append)
    k_ring: np.ndarray        # [B,H,R,d] storage dtype (uint16 bits for bf16)
    v_ring: np.ndarray
    k_cd: np.ndarray          # [B,H,C,d]
    v_cd: np.ndarray
    w_cd: np.ndarray          # [B,H,C] float32
    len0: np.ndarray          # [B] int32: tokens before the first step's append
    d_lo0: np.ndarray
    s_lo0: np.ndarray
    tau: np.ndarray           # [B,H] float32 calibration temperatures (1.0)


def storage_np_dtype(dtype: str):
    return np.float32 if dtype == F32 else np.uint16


def initial_state(w: Workload, threads: int = 8) -> InitialState:
    """Cascade cache before the first step (HARD-KV sec. 2.A tiers, stated reading):
    Condensed slots hold positions [0, C) verbatim with weight 1; the ring holds
    positions [C, len-1) at row pos mod R; Dense is [len-W, len), Sparse [C, len-W)."""
    B, H, d, C = w.batch, w.n_kv_heads, w.head_dim, w.condensed_slots
    R = w.derived_ring_rows()
    lens = seq_lengths(w)
    nd = storage_np_dtype(w.dtype)
    k_ring = np.zeros((B, H, R, d), nd)
    v_ring = np.zeros((B, H, R, d), nd)
    k_cd = np.zeros((B, H, C, d), nd)
    v_cd = np.zeros((B, H, C, d), nd)

    def fill(bh):
        b, h = divmod(bh, H)
        L = int(lens[b])
        kr, _, vr, _ = unit_kv(w, b, h, 0, L - 1)
        k_cd[b, h] = kr[:C]
        v_cd[b, h] = vr[:C]
        pos = np.arange(C, L - 1)
        k_ring[b, h, pos % R] = kr[C:]
        v_ring[b, h, pos % R] = vr[C:]

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fill, range(B * H)))
    len0 = (lens - 1).astype(np.int32)
    d_lo0 = (lens - w.dense_window).astype(np.int32)
    s_lo0 = np.full(B, C, np.int32)
    return InitialState(w, R, lens, k_ring, v_ring, k_cd, v_cd,
                        np.ones((B, H, C), np.float32), len0, d_lo0, s_lo0,
                        np.ones((B, H), np.float32))


def step_kv(w: Workload, lens: np.ndarray, step: int):
    """k_new, v_new [B,H,d] for decode step `step`: the stream values at the appended
    position lens[b]-1+step. Returns (k_raw, k_exact, v_raw, v_exact)."""
    B, H, d = w.batch, w.n_kv_heads, w.head_dim
    kf = np.zeros((B, H, d), np.float32)
    vf = np.zeros((B, H, d), np.float32)
    for b in range(B):
        pos = int(lens[b]) - 1 + step
        for h in range(H):
            kf[b, h] = key_rows(w, b, h, pos, pos + 1)[0]
            vf[b, h] = value_rows(w, b, h, pos, pos + 1)[0]
    kr, ke = storage(kf, w.dtype)
    vr, ve = storage(vf, w.dtype)
    return kr, ke, vr, ve


def p_values(w: Workload) -> tuple[float, ...]:
    return w.p if isinstance(w.p, tuple) else (w.p,)
