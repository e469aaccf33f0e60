"""Planted mistakes in the oracle (on the CPU) must each fail at least one pin.

Each mutant replaces one oracle function with a plausibly wrong version (a dropped
term, a wrong sign or index, a reversed order) and runs the pins that should catch it.
"""
import math

import numpy as np
import pytest

from oracle import hardkv_oracle as O
from tests import test_oracle_pins as P


def _score_no_scale(q, k):
    return (k @ q.T).max(axis=1) if k.shape[0] else np.zeros(0)


def _score_min(q, k):
    return (k @ q.T / math.sqrt(q.shape[1])).min(axis=1) if k.shape[0] else np.zeros(0)


def _score_first_query_only(q, k):
    return (k @ q[0] / math.sqrt(q.shape[1])) if k.shape[0] else np.zeros(0)


def _calibrate_times_tau(s, tau):
    e = np.exp((s - s.max()) * tau)
    return e / e.sum()


_orig_top_p = O.top_p


def _top_p_position_desc(scores, tau, p, cap):
    L = scores.size
    probs = O.calibrate(scores, tau)
    order = np.lexsort((-np.arange(L), -scores))
    cum = np.cumsum(probs[order])
    k_mass = L if p >= 1 else int(np.argmax(cum >= np.float32(p))) + 1
    k = min(k_mass, cap)
    return O.Selection(np.sort(order[:k]), order, k_mass, k, k_mass > cap, probs, cum)


def _top_p_off_by_one(scores, tau, p, cap):
    sel = _orig_top_p(scores, tau, p, cap)
    k = min(sel.k + 1, scores.size, cap)
    return O.Selection(np.sort(sel.order[:k]), sel.order, sel.k_mass, k, sel.clamped,
                       sel.probs, sel.cum)


def _top_p_no_clamp(scores, tau, p, cap):
    return _orig_top_p(scores, tau, p, 10 ** 9)


def _regularize_desc(mask, positions, k, v, cap):
    n, idx, kc, vc = O.__dict__["_orig_regularize"](mask, positions, k, v, cap)
    idx[:n] = idx[:n][::-1].copy()
    return n, idx, kc[::-1].copy(), vc[::-1].copy()


O._orig_regularize = O.regularize


def _attention_no_bias(q, k, v, bias):
    return O.__dict__["_orig_attention"](q, k, v, np.zeros_like(bias))


O._orig_attention = O.attention


def _attention_no_scale(q, k, v, bias):
    return O.__dict__["_orig_attention"](q * math.sqrt(q.shape[1]), k, v, bias)


def _cosine_unnormalised(a, rows):
    return rows @ a


def _attention_entropy_max(q_group, k_rows):
    if k_rows.shape[0] == 0:
        return 0.0
    logits = k_rows @ q_group.T / math.sqrt(q_group.shape[1])
    return float(max(O.entropy(O.calibrate(logits[:, g], 1.0)) for g in range(q_group.shape[0])))


def _entropy_log2(probs):
    p = probs[probs > 0]
    return float(-(p * np.log2(p)).sum())


def _entropy_matched_tau_inverted(scores, target, iters=200):
    if scores.size <= 1:
        return 1.0
    lo, hi = math.log(O.TAU_MIN), math.log(O.TAU_MAX)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if O.entropy(O.calibrate(scores, math.exp(mid))) > target:   # wrong direction
            lo = mid
        else:
            hi = mid
    return math.exp(0.5 * (lo + hi))


def _top_k_position_desc(scores, k):
    L = scores.size
    order = np.lexsort((-np.arange(L), -scores))
    kk = min(int(k), L)
    probs = O.calibrate(scores, 1.0)
    return O.Selection(np.sort(order[:kk]), order, kk, kk, False, probs, np.cumsum(probs[order]))


def _top_k_one_more(scores, k):
    return _orig_top_k(scores, k + 1)


def _mti_le(n, reuse_steps, l_lower, l_upper, gather_surcharge, write_cost=1.0):
    if n < l_lower:
        return False
    if n > l_upper:
        return True
    return write_cost <= reuse_steps * gather_surcharge


def _flatten_sum_inclusive(index_lists):
    # offsets[u] counts head u's own entries too (an inclusive running sum)
    offsets, flat, run = [], [], 0
    for lst in index_lists:
        run += len(lst)
        offsets.append(run)
        flat.extend(int(x) for x in lst)
    offsets.append(run)
    return np.array(offsets, np.int64), np.array(flat, np.int64)


def _flatten_sum_reversed_heads(index_lists):
    lists = list(index_lists)[::-1]
    offsets, flat = [0], []
    for lst in lists:
        flat.extend(int(x) for x in lst)
        offsets.append(offsets[-1] + len(lst))
    return np.array(offsets, np.int64), np.array(flat, np.int64)


_orig_top_k = O.top_k

MUTANTS = [
    ("score", _score_no_scale, [lambda: P.test_score_brute_force(4, 16, 7)]),
    ("score", _score_min, [lambda: P.test_score_brute_force(4, 16, 7)]),
    ("score", _score_first_query_only, [lambda: P.test_score_brute_force(4, 16, 7)]),
    ("calibrate", _calibrate_times_tau,
     [lambda: P.test_calibrate_temperature_and_order_invariance(0.5)]),
    ("top_p", _top_p_position_desc,
     [lambda: [P.test_top_p_hand_cases(c) for c in P.GOLD["top_p"]]]),
    ("top_p", _top_p_off_by_one,
     [lambda: [P.test_top_p_hand_cases(c) for c in P.GOLD["top_p"]]]),
    ("top_p", _top_p_no_clamp, [P.test_top_p_cap_is_top_cap_by_score]),
    ("regularize", _regularize_desc, [P.test_regularize_order_count_and_rows]),
    ("attention", _attention_no_bias,
     [lambda: [P.test_attention_hand_cases(c) for c in P.GOLD["attention"]]]),
    ("attention", _attention_no_scale, [P.test_attention_equals_torch_sdpa]),
    ("cosine", _cosine_unnormalised,
     [lambda: [P.test_merge_slot_choice_brute_force(s) for s in range(10)]]),
    ("attention_entropy", _attention_entropy_max,
     [P.test_attention_entropy_is_the_mean_of_the_queries_raw_entropies]),
    ("entropy", _entropy_log2, [P.test_entropy_matches_scipy]),
    ("entropy_matched_tau", _entropy_matched_tau_inverted,
     [P.test_entropy_matched_tau_residual_scale_and_range]),
    ("top_k", _top_k_position_desc, [lambda: [P.test_top_k_brute_force_small(s) for s in range(20)]]),
    ("top_k", _top_k_one_more, [lambda: [P.test_top_k_brute_force_small(s) for s in range(20)]]),
    ("mti_rewrite", _mti_le, [P.test_mti_policy_thresholds_and_break_even]),
    ("flatten_sum", _flatten_sum_inclusive, [P.test_flatten_sum_hand_cases]),
    ("flatten_sum", _flatten_sum_reversed_heads,
     [P.test_flatten_sum_hand_cases, P.test_flatten_sum_round_trips_the_max_length_form]),
]


@pytest.mark.parametrize("i", range(len(MUTANTS)))
def test_mutant_is_caught(i, monkeypatch):
    name, fn, pins = MUTANTS[i]
    monkeypatch.setattr(O, name, fn)
    caught = False
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught = True
    assert caught, f"mutant {fn.__name__} of {name} passed every pin"


def test_block_move_off_by_one_is_caught(monkeypatch):
    def append(self, k_new, v_new):
        P_ = self.prm
        self.K[self.len] = k_new
        self.V[self.len] = v_new
        self.len += 1
        if self.len - self.d_lo > P_.dense_window + P_.block:   # '>' instead of '>='
            self.d_lo += P_.block
            self.s_lo += P_.block
            return True
        return False
    monkeypatch.setattr(O.Unit, "append", append)
    with pytest.raises(AssertionError):
        P.test_block_move_schedule()
