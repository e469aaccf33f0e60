"""The benchmark's algorithmic-byte model (bench.step_bytes / sum_bytes) on CPU.

The roofline fractions the benchmark reports divide these bytes by measured time, so
the model is checked here against a second, loop-per-unit statement of what each
kernel must move (one (sequence, KV head) unit at a time, from the definitions: e the
element size, a row = one K row + one V row):

  append    per unit: k_new and v_new read, their ring rows written      4 d e
  condense  per unit of a moved sequence (MERGE): block + C slots read,
            C slots written                                              (Blk + 2C) 2 d e
  score     per reselecting unit: L candidate keys, G queries, L scores  L d e + G d e + 4 L
  topp      per reselecting unit: L scores read, ceil(L/32) mask words,
            the Cap-long index written (-1 pads included)                4 L + 4 ceil(L/32) + 4 Cap
  attend    per unit: kept rows (gathered + written under Rewrite Cache in a reselecting
            step, gathered only under Sparse Loading, read once when carried over), the
            index, Dense and Condensed rows, Condensed weights, q and the fp32 output

on random states of several shapes, and on one hand-worked unit; and the same for the
step as its standalone calls (bench --path unfused).
"""
import math

import numpy as np
import pytest

import bench
from attention_kv_head_b200 import synth


def _state(w, r):
    B, H = w.batch, w.n_kv_heads
    s_lo = r.randint(0, 400, B)
    d_lo = s_lo + r.randint(0, 3000, B)
    ln = d_lo + r.randint(w.dense_window, w.dense_window + w.block, B)
    n = np.minimum(r.randint(0, w.sparse_cap + 1, (B, H)), (d_lo - s_lo)[:, None])
    live = np.minimum(n, r.randint(0, w.sparse_cap + 1, (B, H)))
    return {"len": ln, "d_lo": d_lo, "s_lo": s_lo, "moved": r.randint(0, 2, B),
            "n_kept": n, "sp_mode": r.randint(0, 2, (B, H)), "live": live,
            "reselect": r.randint(0, 2, B).astype(bool)}


def _by_units(w, st):
    """The same bytes, unit by unit."""
    e = 2 if w.dtype == synth.BF16 else 4
    d, G, C, cap = w.head_dim, w.group, w.condensed_slots, w.sparse_cap
    row = 2 * d * e
    tot = dict(append=0, condense=0, score=0, topp=0, attend=0)
    for b in range(w.batch):
        L = int(st["d_lo"][b] - st["s_lo"][b])
        dense = int(st["len"][b] - st["d_lo"][b])
        sel = bool(st["reselect"][b])
        for h in range(w.n_kv_heads):
            n, live = int(st["n_kept"][b, h]), int(st["live"][b, h])
            rewrite = bool(st["sp_mode"][b, h])
            tot["append"] += 2 * d * e * 2
            if w.condense_mode == synth.MERGE and st["moved"][b]:
                tot["condense"] += (w.block + 2 * C) * row
            if sel:
                tot["score"] += L * d * e + G * d * e + 4 * L
                tot["topp"] += 4 * L + 4 * math.ceil(L / 32) + 4 * cap
                kept = n * row * (2 if rewrite else 1)      # gathered (and written)
            else:
                kept = live * row                            # carried over: read once
            tot["attend"] += (kept + 4 * n + (dense + C) * row + 4 * C
                              + G * d * e + G * d * 4)
    tot["total"] = sum(tot.values())
    return tot


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("shape", ["bf16_merge", "f32_evict", "bf16_g8"])
def test_step_bytes_matches_the_per_unit_statement(shape, seed):
    kw = {"bf16_merge": dict(condense_mode=synth.MERGE),
          "f32_evict": dict(dtype=synth.F32, head_dim=64, n_q_heads=4, n_kv_heads=2),
          "bf16_g8": dict(n_q_heads=16, n_kv_heads=2, batch=5)}[shape]
    w = synth.small(sparse_cap=700, **kw)
    st = _state(w, np.random.RandomState(seed))
    got = bench.step_bytes(w, st)
    want = _by_units(w, st)
    for k, v in want.items():
        assert got[k] == v, (k, got[k], v)
    kept_sel = int((st["n_kept"] * st["reselect"][:, None]).sum())
    L_sel = int(((st["d_lo"] - st["s_lo"]) * st["reselect"]).sum()) * w.n_kv_heads
    assert got["sum_kept"] == kept_sel
    assert got["kept_fraction"] == pytest.approx(kept_sel / max(L_sel, 1))


def test_one_hand_worked_unit():
    """One bf16 unit, d = 128, G = 4, C = 256, Cap = 7680: L = 7936 candidates, 3637
    kept and rewritten, 257 Dense rows, reselecting. Row = 512 bytes."""
    w = synth.small(batch=1, n_q_heads=4, n_kv_heads=1, head_dim=128, condensed_slots=256,
                    sparse_cap=7680, dense_window=256)
    st = {"len": np.array([8449]), "d_lo": np.array([8192]), "s_lo": np.array([256]),
          "moved": np.array([0]), "n_kept": np.array([[3637]]), "sp_mode": np.array([[1]]),
          "live": np.array([[3637]]), "reselect": np.array([True])}
    got = bench.step_bytes(w, st)
    assert got["append"] == 1024                                  # 4 x 128 x 2
    assert got["condense"] == 0                                   # eviction
    assert got["score"] == 7936 * 256 + 4 * 256 + 7936 * 4        # 2 064 384
    assert got["topp"] == 7936 * 4 + 248 * 4 + 7680 * 4           # 63 456
    assert got["attend"] == (2 * 3637 * 512 + 3637 * 4 + (257 + 256) * 512 + 256 * 4
                             + 4 * 256 + 4 * 512)                 # 4 005 588
    assert got["total"] == 1024 + 2064384 + 63456 + 4005588      # 6 134 452


def _by_units_unfused(w, st):
    """The standalone calls, unit by unit: the selection writes only the mask; the
    compaction reads the mask, writes the Cap-long index and, under Rewrite Cache, reads
    the kept rows from the ring and writes them compact; the attention reads every kept
    row once."""
    e = 2 if w.dtype == synth.BF16 else 4
    d, G, C, cap = w.head_dim, w.group, w.condensed_slots, w.sparse_cap
    row = 2 * d * e
    tot = dict(append=0, condense=0, select=0, regularize=0, attend=0)
    for b in range(w.batch):
        L = int(st["d_lo"][b] - st["s_lo"][b])
        dense = int(st["len"][b] - st["d_lo"][b])
        sel = bool(st["reselect"][b])
        for h in range(w.n_kv_heads):
            n, live = int(st["n_kept"][b, h]), int(st["live"][b, h])
            rewrite = bool(st["sp_mode"][b, h])
            tot["append"] += 4 * d * e
            if w.condense_mode == synth.MERGE and st["moved"][b]:
                tot["condense"] += (w.block + 2 * C) * row
            words = 4 * math.ceil(L / 32)
            if sel:
                tot["select"] += L * d * e + G * d * e + 4 * L + 4 * L + words
                tot["regularize"] += words + 4 * cap + (2 * n * row if rewrite else 0)
                kept = n * row
            else:
                kept = live * row
            tot["attend"] += (kept + 4 * n + (dense + C) * row + 4 * C
                              + G * d * e + G * d * 4)
    tot["total"] = sum(tot.values())
    return tot


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("shape", ["bf16_merge", "f32_evict"])
def test_unfused_bytes_match_the_per_unit_statement(shape, seed):
    kw = {"bf16_merge": dict(condense_mode=synth.MERGE),
          "f32_evict": dict(dtype=synth.F32, head_dim=64, n_q_heads=4, n_kv_heads=2)}[shape]
    w = synth.small(sparse_cap=700, **kw)
    st = _state(w, np.random.RandomState(100 + seed))
    got = bench.step_bytes(w, st, fused=False)
    for k, v in _by_units_unfused(w, st).items():
        assert got[k] == v, (k, got[k], v)
    # the fused step moves less: the kept rows are gathered once for both the rewrite and
    # the attention, and the index is written once
    assert bench.step_bytes(w, st)["total"] <= got["total"]


def test_sum_bytes_pools_the_kept_fraction_over_steps():
    w = synth.small(sparse_cap=700)
    r = np.random.RandomState(7)
    steps = [bench.step_bytes(w, _state(w, r)) for _ in range(5)]
    tot = bench.sum_bytes(steps)
    for k in ("append", "condense", "score", "topp", "attend", "total", "sum_kept"):
        assert tot[k] == sum(s[k] for s in steps)
    L = sum(s["sum_kept"] / s["kept_fraction"] for s in steps if s["kept_fraction"] > 0)
    assert tot["kept_fraction"] == pytest.approx(tot["sum_kept"] / L)
