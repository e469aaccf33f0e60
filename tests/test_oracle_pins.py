"""Pins of the fp64 oracle against things other than itself: hand-derived cases,
closed forms, library routines, brute force on tiny inputs, invariants.

HARD-KV technical summary sec. 2.A-2.C (cascade tiers, Logits Calibration,
calibrated top-p, Rewrite Cache / Flatten Index, eviction / weighted merge)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

from oracle import hardkv_oracle as O

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")))


def rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- storage rounding

def test_round_storage_bf16_hand_halfway_cases():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0)
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 1 + 2.0 ** -8 + 2.0 ** -30,
                  0.0, 3.0, 2.0 ** -20 * 1.00390625])
    want = np.array([1.0, 1 + 2.0 ** -6, -1.0, 1 + 2.0 ** -7, 0.0, 3.0, 2.0 ** -20])  # last: halfway -> even
    assert np.array_equal(O.round_storage(x, O.BF16), want)


def test_round_storage_bf16_matches_torch_on_float32_inputs():
    x = (rng(1).standard_normal(200000) * 10.0 ** rng(2).uniform(-3, 3, 200000)).astype(np.float32)
    ours = O.round_storage(x.astype(np.float64), O.BF16)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_round_storage_f32_is_float32_cast():
    x = rng(3).standard_normal(1000) / 3.0
    assert np.array_equal(O.round_storage(x, O.F32), x.astype(np.float32).astype(np.float64))


# ---------------------------------------------------------------- score

def brute_score(q, k):
    G, d = q.shape
    out = []
    for j in range(k.shape[0]):
        best = -math.inf
        for g in range(G):
            acc = 0.0
            for c in range(d):
                acc += q[g][c] * k[j][c]
            best = max(best, acc / math.sqrt(d))
        out.append(best)
    return np.array(out)


@pytest.mark.parametrize("G,d,L", [(1, 8, 5), (4, 16, 7), (5, 4, 3), (8, 2, 9)])
def test_score_brute_force(G, d, L):
    r = rng(G * 100 + d)
    q, k = r.standard_normal((G, d)), r.standard_normal((L, d))
    assert np.allclose(O.score(q, k), brute_score(q, k), rtol=1e-13, atol=1e-13)


def test_score_single_query_equals_sdpa_logits():
    # G = 1: the importance score is exactly the raw attention logit q.k/sqrt(d)
    r = rng(5)
    q, k = r.standard_normal((1, 64)), r.standard_normal((50, 64))
    logits = (torch.from_numpy(q) @ torch.from_numpy(k).T).numpy()[0] / 8.0
    assert np.allclose(O.score(q, k), logits, rtol=1e-14, atol=1e-14)


def test_score_is_max_over_group_and_permutation_equivariant():
    r = rng(6)
    q, k = r.standard_normal((4, 32)), r.standard_normal((40, 32))
    s = O.score(q, k)
    per = np.stack([O.score(q[g:g + 1], k) for g in range(4)])
    assert np.allclose(s, per.max(axis=0), rtol=0, atol=1e-14)
    perm = r.permutation(40)
    assert np.allclose(O.score(q, k[perm]), s[perm], rtol=0, atol=1e-14)
    assert np.allclose(O.score(q[::-1].copy(), k), s, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- calibration

def test_calibrate_tau1_equals_scipy_softmax():
    s = rng(7).standard_normal(300) * 3
    assert np.allclose(O.calibrate(s, 1.0), scipy.special.softmax(s), rtol=1e-13, atol=1e-16)


@pytest.mark.parametrize("tau", [0.25, 0.5, 1.0, 2.0, 7.0])
def test_calibrate_temperature_and_order_invariance(tau):
    s = rng(8).standard_normal(500) * 2
    p = O.calibrate(s, tau)
    assert abs(p.sum() - 1) < 1e-12
    assert np.allclose(p, scipy.special.softmax(s / tau), rtol=1e-12, atol=1e-18)
    # order of the calibrated distribution equals the order of the raw scores
    assert np.array_equal(np.argsort(-p, kind="stable"), np.argsort(-s, kind="stable"))


def test_calibrate_limits():
    s = np.array([3.0, 1.0, -2.0, 0.5])
    assert np.allclose(O.calibrate(s, 1e9), 0.25, atol=1e-8)         # tau -> inf: uniform
    assert np.allclose(O.calibrate(s, 1e-3), [1, 0, 0, 0], atol=1e-12)  # tau -> 0: one-hot


# ---------------------------------------------------------------- top-p

@pytest.mark.parametrize("case", GOLD["top_p"], ids=lambda c: c["why"][:30])
def test_top_p_hand_cases(case):
    s = np.log(np.array(case["scores_ln"], np.float64))
    sel = O.top_p(s, case["tau"], case["p"], case["cap"])
    assert sel.kept.tolist() == case["kept"], case["why"]


def test_top_p_keep_all_at_p1():
    for seed in range(5):
        s = rng(seed).standard_normal(333) * 4
        sel = O.top_p(s, 1.0, 1.0, 10 ** 6)
        assert sel.k == 333 and sel.kept.tolist() == list(range(333))


@pytest.mark.parametrize("n,p", [(10, 0.55), (7, 0.9), (928, 0.9), (100, 0.333), (64, 0.95)])
def test_top_p_uniform_keeps_ceil_pn(n, p):
    p32 = float(np.float32(p))
    assert abs(p32 * n - round(p32 * n)) > 1e-9
    sel = O.top_p(np.full(n, 0.37), 1.0, p, 10 ** 6)
    assert sel.k == math.ceil(p32 * n)
    assert sel.kept.tolist() == list(range(sel.k))       # ties broken by position


def test_top_p_one_hot_keeps_one():
    s = np.full(200, -1e3)
    s[77] = 50.0
    for p in (0.5, 0.9, 0.99):
        sel = O.top_p(s, 1.0, p, 100)
        assert sel.kept.tolist() == [77]


def brute_top_p(s, tau, p, cap):
    """Smallest subset with calibrated mass >= p; among equal sizes the largest mass,
    then lexicographically smallest (desc score, asc position) ranking; then clamp."""
    n = len(s)
    pr = scipy.special.softmax(np.asarray(s) / tau)
    p = float(np.float32(p))
    if p >= 1:
        best = tuple(range(n))
    else:
        best = None
        for size in range(1, n + 1):
            cands = []
            for sub in itertools.combinations(range(n), size):
                m = sum(pr[i] for i in sub)
                if m >= p - 1e-15 * n:
                    cands.append((-round(m, 12), sorted((-s[i], i) for i in sub), sub))
            if cands:
                best = min(cands)[2]
                break
    # clamp: the best `cap` of the chosen set by (score desc, position asc)
    ranked = sorted(best, key=lambda i: (-s[i], i))[:cap]
    return sorted(ranked)


@pytest.mark.parametrize("seed", range(40))
def test_top_p_brute_force_small(seed):
    r = rng(100 + seed)
    n = int(r.integers(1, 11))
    s = r.standard_normal(n) * r.uniform(0.2, 3)
    if seed % 5 == 0 and n > 2:
        s[1] = s[0]                                         # a tie
    tau = float(r.choice([0.5, 1.0, 2.0]))
    p = float(r.choice([0.3, 0.5, 0.8, 0.9, 0.95, 1.0]))
    cap = int(r.integers(1, n + 1))
    sel = O.top_p(s, tau, p, cap)
    # skip draws whose cumulative mass sits on p within rounding (ambiguous by design)
    if p < 1 and np.min(np.abs(sel.cum - float(np.float32(p)))) < 1e-9:
        pytest.skip("mass lands on p within rounding")
    assert sel.kept.tolist() == brute_top_p(s, tau, p, cap)


def test_top_p_monotone_in_p_and_tau():
    s = rng(9).standard_normal(2000) * 2
    ks = [O.top_p(s, 1.0, p, 10 ** 6).k for p in np.linspace(0.05, 0.99, 30)]
    assert all(a <= b for a, b in zip(ks, ks[1:]))
    kt = [O.top_p(s, t, 0.9, 10 ** 6).k for t in (0.25, 0.5, 1, 2, 4, 8)]
    assert all(a <= b for a, b in zip(kt, kt[1:]))
    # and the kept sets are nested
    a = set(O.top_p(s, 1.0, 0.5, 10 ** 6).kept)
    b = set(O.top_p(s, 1.0, 0.8, 10 ** 6).kept)
    assert a <= b


def test_top_p_cap_is_top_cap_by_score():
    s = rng(10).standard_normal(1000)
    sel = O.top_p(s, 0.2, 0.99, 50)
    assert sel.clamped and sel.k == 50
    assert sel.kept.tolist() == sorted(np.argsort(-s, kind="stable")[:50].tolist())


@pytest.mark.parametrize("sigma", [0.5, 1.0, 2.0])
def test_top_p_gaussian_kept_fraction_closed_form(sigma):
    """For i.i.d. N(0, sigma^2) logits, the exponentially tilted law is N(sigma^2,
    sigma^2), so the kept fraction tends to 1 - Phi(sigma - Phi^-1(p))."""
    n, p = 200000, 0.9
    s = rng(11).standard_normal(n) * sigma
    frac = O.top_p(s, 1.0, p, n).k / n
    want = 1 - scipy.stats.norm.cdf(sigma - scipy.stats.norm.ppf(p))
    assert abs(frac - want) < 0.01, (frac, want)


# ---------------------------------------------------------------- regularize

def test_regularize_order_count_and_rows():
    r = rng(12)
    L, d, cap = 300, 16, 200
    pos = np.arange(1000, 1000 + L)
    k, v = r.standard_normal((L, d)), r.standard_normal((L, d))
    mask = r.random(L) < 0.3
    n, idx, kc, vc = O.regularize(mask, pos, k, v, cap)
    assert n == mask.sum()
    assert np.all(np.diff(idx[:n]) > 0) and np.all(idx[n:] == -1)
    assert set(idx[:n].tolist()) == set(pos[mask].tolist())
    for slot in range(n):
        j = idx[slot] - 1000
        assert kc[slot].tobytes() == k[j].tobytes() and vc[slot].tobytes() == v[j].tobytes()


def test_regularize_truncates_to_capacity_in_position_order():
    mask = np.ones(50, bool)
    n, idx, kc, _ = O.regularize(mask, np.arange(50), np.eye(50), np.eye(50), 20)
    assert n == 20 and idx[:20].tolist() == list(range(20)) and kc.shape == (20, 50)


def test_flatten_sum_hand_cases():
    for c in GOLD["flatten_sum"]:
        offsets, flat = O.flatten_sum([np.array(x, np.int64) for x in c["lists"]])
        assert offsets.tolist() == c["offsets"], c["why"]
        assert flat.tolist() == c["flat"], c["why"]


def test_flatten_sum_round_trips_the_max_length_form():
    """The sum form holds exactly the max-length form's non-pad entries: slicing the flat
    list by the offsets gives back each head's regularized index, and the total is the
    sum of the kept counts."""
    r = rng(31)
    cap, rows, ns = 40, [], []
    for u in range(9):
        mask = r.random(60) < r.random()
        n, idx, _, _ = O.regularize(mask, np.arange(100 * u, 100 * u + 60), np.zeros((60, 1)),
                                    np.zeros((60, 1)), cap)
        rows.append(idx)
        ns.append(n)
    offsets, flat = O.flatten_sum([row[:n] for row, n in zip(rows, ns)])
    assert offsets[0] == 0 and offsets[-1] == sum(ns) == flat.size
    assert np.all(np.diff(offsets) == np.array(ns))
    for u, (row, n) in enumerate(zip(rows, ns)):
        seg = flat[offsets[u]:offsets[u + 1]]
        assert np.array_equal(seg, row[:n]) and np.all(row[n:] == -1)


# ---------------------------------------------------------------- merge / condense

def test_merge_hand_case():
    c = GOLD["merge"][0]
    ck = np.array(c["slots_k"], float)
    cv = ck.copy()
    w = np.array(c["w"], float)
    log = O.MergeLog()
    O.merge_block(np.array(c["x_k"], float), np.array(c["x_k"], float), ck, cv, w,
                  c["n_sink"], O.F32, log)
    assert log.slots == [c["slot"]]
    assert np.allclose(ck, c["slots_k_after"], rtol=1e-7) and w.tolist() == c["w_after"]


def brute_argmax_cos(x, slots, w, n_sink):
    best, arg = -math.inf, -1
    for s in range(len(slots)):
        if s < n_sink or w[s] <= 0:
            continue
        num = sum(a * b for a, b in zip(x, slots[s]))
        den = math.sqrt(sum(a * a for a in x) * sum(b * b for b in slots[s]))
        c = num / den if den > 0 else 0.0
        if c > best:
            best, arg = c, s
    return arg


@pytest.mark.parametrize("seed", range(10))
def test_merge_slot_choice_brute_force(seed):
    r = rng(200 + seed)
    C, d = 12, 6
    ck = r.standard_normal((C, d))
    cv = r.standard_normal((C, d))
    w = r.integers(0, 4, C).astype(float)
    w[5] = 1.0
    blk = r.standard_normal((4, d))
    ck0, w0 = ck.copy(), w.copy()
    log = O.MergeLog()
    O.merge_block(blk, blk, ck, cv.copy(), w, 2, O.F32, log)
    # replay by hand: each token picks by brute force on the evolving slots
    sk, sw = ck0.copy(), w0.copy()
    for t in range(4):
        s = brute_argmax_cos(blk[t], sk, sw, 2)
        assert log.slots[t] == s
        sk[s] = np.float32((sw[s] * sk[s] + blk[t]) / (sw[s] + 1))
        sw[s] += 1
    assert np.array_equal(w, sw)


def test_merge_ties_go_to_lowest_slot_and_sinks_are_pinned():
    ck = np.array([[1.0, 0], [1.0, 0], [2.0, 0], [1.0, 0]])
    w = np.array([1.0, 1.0, 1.0, 1.0])
    log = O.MergeLog()
    O.merge_block(np.array([[3.0, 0]]), np.array([[3.0, 0]]), ck, ck.copy(), w, 1, O.F32, log)
    assert log.slots == [1]          # slots 1,2,3 tie at cos 1; slot 0 is a sink
    assert w.tolist() == [1, 2, 1, 1]


@pytest.mark.parametrize("m", [2, 3, 7])
def test_merging_identical_tokens_equals_separate_tokens(m):
    """A slot holding k with w=1 absorbs m-1 copies of k: the slot stays k exactly and
    attention with bias ln m equals attention over the m copies."""
    r = rng(300 + m)
    d = 8
    kx = O.round_storage(r.standard_normal(d), O.BF16)
    vx = O.round_storage(r.standard_normal(d), O.BF16)
    other_k = O.round_storage(r.standard_normal((3, d)), O.BF16)
    other_v = O.round_storage(r.standard_normal((3, d)), O.BF16)
    ck = np.vstack([other_k[:1] * 0 - 5, kx[None]])     # slot 0 sink, slot 1 = kx
    cv = np.vstack([other_v[:1], vx[None]])
    w = np.array([1.0, 1.0])
    O.merge_block(np.tile(kx, (m - 1, 1)), np.tile(vx, (m - 1, 1)), ck, cv, w, 1, O.BF16)
    assert np.array_equal(ck[1], kx) and np.array_equal(cv[1], vx) and w[1] == m
    q = r.standard_normal((4, d))
    merged = O.attention(q, np.vstack([other_k, ck[1:]]), np.vstack([other_v, cv[1:]]),
                         np.r_[np.zeros(3), math.log(m)])
    separate = O.attention(q, np.vstack([other_k] + [kx[None]] * m),
                           np.vstack([other_v] + [vx[None]] * m), np.zeros(3 + m))
    assert np.allclose(merged, separate, rtol=1e-13, atol=1e-13)


def test_merge_running_mean_fp32():
    r = rng(13)
    d = 5
    k0 = r.standard_normal(d)
    xs = r.standard_normal((6, d))
    ck = np.vstack([np.zeros(d), k0[None].astype(np.float32)]).astype(float)
    w = np.array([1.0, 1.0])
    O.merge_block(xs, xs, ck, ck.copy(), w, 1, O.F32)
    assert w[1] == 7
    assert np.allclose(ck[1], (np.float32(k0).astype(float) + xs.sum(0)) / 7, rtol=1e-6, atol=1e-6)


# ---------------------------------------------------------------- attention

@pytest.mark.parametrize("case", GOLD["attention"], ids=lambda c: c["why"][:25])
def test_attention_hand_cases(case):
    q = np.array(case["q"])
    k = np.log(np.array(case["k_ln_times_sqrt_d"], float)) * math.sqrt(q.shape[1])
    out = O.attention(q, k, np.array(case["v"]),
                      np.log(np.array(case["bias_ln"], float)))
    assert np.allclose(out, case["out"], rtol=1e-12, atol=1e-12)


def test_attention_equals_torch_sdpa():
    r = rng(14)
    G, T, d = 5, 123, 64
    q, k, v = r.standard_normal((G, d)), r.standard_normal((T, d)), r.standard_normal((T, d))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None])[0, 0].numpy()
    assert np.allclose(O.attention(q, k, v, np.zeros(T)), ref, rtol=1e-12, atol=1e-12)


def test_attention_bias_is_additive_logit():
    r = rng(15)
    q, k, v = r.standard_normal((2, 16)), r.standard_normal((9, 16)), r.standard_normal((9, 16))
    bias = r.uniform(0, 2, 9)
    # bias b_t == scaling the unnormalised weight by e^{b_t} == repeating token t e^{b_t} times
    lg = q @ k.T / 4.0
    wts = np.exp(lg) * np.exp(bias)
    want = wts @ v / wts.sum(1, keepdims=True)
    assert np.allclose(O.attention(q, k, v, bias), want, rtol=1e-12)


# ---------------------------------------------------------------- cascade unit

def make_unit(seed, L, d=16, G=2, W=8, C=6, blk=4, cap=None, mode=O.EVICT, dtype=O.F32,
              steps=0):
    r = rng(seed)
    K = O.round_storage(r.standard_normal((L + steps, d)), dtype)
    V = O.round_storage(r.standard_normal((L + steps, d)), dtype)
    prm = O.Params(d, G, W, C, blk, cap if cap else L, 2, dtype, mode)
    u = O.Unit(prm, K[:L - 1], V[:L - 1], K[:C], V[:C], np.ones(C), L - 1, L - W, C,
               L + steps + 1)
    return u, K, V, r


def test_dense_only_keep_all_equals_full_attention():
    """p = 1 with capacity >= Sparse length and unmerged Condensed slots (w = 1):
    Dense U kept U Condensed covers every position once -> exact full attention."""
    for seed in range(4):
        u, K, V, r = make_unit(seed, L=120)
        q = r.standard_normal((2, 16))
        out = u.step(q, K[119], V[119], 1.0, 1.0).out
        assert np.allclose(out, O.full_attention(q, K[:120], V[:120]), rtol=1e-12, atol=1e-12)


def test_union_partitions_positions():
    u, K, V, r = make_unit(20, L=200)
    q = r.standard_normal((2, 16))
    u.step(q, K[199], V[199], 1.0, 0.5)
    kept = u.idx[:u.n]
    dense = np.arange(u.d_lo, u.len)
    assert np.all(kept >= u.s_lo) and np.all(kept < u.d_lo)
    assert u.s_lo == 6 and u.d_lo == 192 and u.len == 200
    assert np.intersect1d(kept, dense).size == 0


def test_block_move_schedule():
    """len - d_lo reaches W + block every block-th step; d_lo and s_lo move together so
    the Sparse length stays constant (stated reading of the per-step block move)."""
    W, blk, C = 8, 4, 6
    u, K, V, r = make_unit(21, L=40, W=W, C=C, blk=blk, steps=20)
    q = r.standard_normal((2, 16))
    moves = []
    for t in range(20):
        res = u.step(q, K[39 + t], V[39 + t], 1.0, 0.9)
        moves.append(res.moved)
        assert u.d_lo - u.s_lo == 40 - W - C
        assert W <= u.len - u.d_lo < W + blk
    # first move when len = 40 + 4 = d_lo0 + W + blk = 32 + 12 = 44 -> step index 4
    assert [i for i, m in enumerate(moves) if m] == [4, 8, 12, 16]


def test_evict_leaves_condensed_unchanged_and_merge_conserves_weight():
    u, K, V, r = make_unit(22, L=40, steps=12, mode=O.EVICT)
    ck0 = u.cd_k.copy()
    q = r.standard_normal((2, 16))
    for t in range(12):
        u.step(q, K[39 + t], V[39 + t], 1.0, 0.9)
    assert np.array_equal(u.cd_k, ck0) and u.cd_w.sum() == 6
    u, K, V, r = make_unit(22, L=40, steps=12, mode=O.MERGE)
    for t in range(12):
        u.step(q, K[39 + t], V[39 + t], 1.0, 0.9)
    # 12 steps -> block moves at steps 4 and 8 -> 2 x 4 tokens merged; sinks untouched
    assert u.cd_w.sum() == 6 + 8 and u.cd_w[0] == 1 and u.cd_w[1] == 1


def test_merged_stale_rows_are_not_attended_twice():
    """Between reselections a compact row whose position left the Sparse tier is
    skipped (its content now lives in the Condensed tier)."""
    u, K, V, r = make_unit(23, L=40, steps=8, mode=O.MERGE)
    q = r.standard_normal((2, 16))
    u.step(q, K[39], V[39], 1.0, 1.0)                    # select everything once
    for t in range(1, 8):
        u.step(q, K[39 + t], V[39 + t], 1.0, 1.0, reselect="none")
    Ku, Vu, bias = u.union()
    assert Ku.shape[0] == (u.idx[:u.n] >= u.s_lo).sum() + (u.len - u.d_lo) + 6


def test_allowed_flips_rule():
    s = np.log(np.array([8, 4, 2, 1, 1.0]))
    sel = O.top_p(s, 1.0, 0.9, 10)
    assert O.allowed_flips(sel, 0.9, [0, 1, 2, 3]) == (True, 0)
    assert O.allowed_flips(sel, 0.9, [0, 1, 2, 4])[0]       # equal p: tie may go either way
    assert not O.allowed_flips(sel, 0.9, [0, 1, 2])[0]      # rank-4 token is not marginal
    assert not O.allowed_flips(sel, 0.9, [1, 2, 3, 4])[0]
    assert not O.allowed_flips(sel, 0.9, [0, 1, 2, 3, 4])[0]   # S_4 = .9375, not near .9
    # a prefix mass that sits on p: p = 0.875 exactly representable; S_3 = .875
    sel = O.top_p(s, 1.0, 0.875, 10)
    assert sel.k in (3, 4)
    assert O.allowed_flips(sel, 0.875, [0, 1, 2])[0] and O.allowed_flips(sel, 0.875, [0, 1, 2, 3])[0]


# ---------------------------------------------------------------- top-k (fixed budget)

@pytest.mark.parametrize("seed", range(20))
def test_top_k_brute_force_small(seed):
    """n <= 9: among all k-subsets exactly one holds every score at least as high as
    every score left out, and takes the lowest positions among the scores tied at the
    boundary; it is the oracle's."""
    r = rng(300 + seed)
    n = int(r.integers(1, 10))
    s = np.round(r.normal(size=n), 1)          # coarse values: ties happen
    for k in range(0, n + 2):
        good = []
        for sub in itertools.combinations(range(n), min(k, n)):
            inn = np.zeros(n, bool)
            inn[list(sub)] = True
            if inn.all() or not inn.any():
                good.append(sub)
                continue
            lo_in, hi_out = s[inn].min(), s[~inn].max()
            if lo_in < hi_out:
                continue
            if lo_in == hi_out:   # boundary ties: kept ones must have the lower positions
                tied_in = np.nonzero(inn & (s == lo_in))[0]
                tied_out = np.nonzero(~inn & (s == lo_in))[0]
                if tied_in.max() > tied_out.min():
                    continue
            good.append(sub)
        assert len(good) == 1
        sel = O.top_k(s, k)
        assert sel.kept.tolist() == sorted(good[0]) and sel.k == min(k, n) and not sel.clamped


def test_top_k_is_the_capacity_clamp_of_keep_all_and_ignores_monotone_maps():
    s = rng(7).normal(size=300) * 2
    for k in (1, 17, 150, 299, 300, 400):
        ref = O.top_k(s, k).kept
        assert np.array_equal(O.top_p(s, 1.0, 1.0, k).kept, ref)      # p = 1 clamped to k
        assert np.array_equal(O.top_k(np.exp(s), k).kept, ref)        # order-only
        assert np.array_equal(O.top_k(3 * s - 5, k).kept, ref)
    assert O.top_k(s, 1).kept.tolist() == [int(np.argmax(s))]


def test_allowed_flips_topk_rule():
    s = np.array([5.0, 4.0, 3.0, 3.0 + 1e-9, 1.0])
    sel = O.top_k(s, 3)
    assert sel.kept.tolist() == [0, 1, 3]
    assert O.allowed_flips_topk(s, sel, [0, 1, 3], 1e-6) == (True, 0)
    assert O.allowed_flips_topk(s, sel, [0, 1, 2], 1e-6)[0]          # within eps of s_theta
    assert not O.allowed_flips_topk(s, sel, [0, 1, 2], 1e-12)[0]
    assert not O.allowed_flips_topk(s, sel, [0, 1, 4], 1e-6)[0]      # far from the boundary
    assert not O.allowed_flips_topk(s, sel, [0, 1, 2, 3], 1e-6)[0]   # count must match


# ---------------------------------------------------------------- entropy-matched calibration

def test_entropy_matches_scipy():
    for seed in range(5):
        p = scipy.special.softmax(rng(400 + seed).normal(size=50) * 3)
        assert abs(O.entropy(p) - scipy.stats.entropy(p)) < 1e-12
    assert O.entropy(np.array([1.0, 0.0, 0.0])) == 0.0
    assert abs(O.entropy(np.full(8, 1 / 8)) - math.log(8)) < 1e-12


def test_attention_entropy_is_the_mean_of_the_queries_raw_entropies():
    r = rng(11)
    q = r.normal(size=(3, 16))
    k = r.normal(size=(40, 16)) * 2
    want = np.mean([scipy.stats.entropy(scipy.special.softmax(k @ q[g] / 4.0)) for g in range(3)])
    assert abs(O.attention_entropy(q, k) - want) < 1e-12
    assert abs(O.attention_entropy(q, np.zeros((40, 16))) - math.log(40)) < 1e-12
    assert O.attention_entropy(q, np.zeros((0, 16))) == 0.0


def test_entropy_matched_tau_single_query_is_one():
    """G = 1: the max-pooled score is the raw logit, so the raw attention's entropy is
    reached at tau = 1."""
    r = rng(12)
    for T in (0.5, 1.0, 3.0):
        q = r.normal(size=(1, 64))
        k = r.normal(size=(500, 64)) * T
        s = O.score(q, k)
        tau = O.entropy_matched_tau(s, O.attention_entropy(q, k))
        assert abs(tau - 1.0) < 1e-9


@pytest.mark.parametrize("sigma,target_drop", [(1.0, 0.2), (2.0, 0.5), (0.7, 0.05)])
def test_entropy_matched_tau_gaussian_closed_form(sigma, target_drop):
    """i.i.d. N(0, sigma^2) scores, large L: H(softmax(s/tau)) -> ln L - sigma^2/(2 tau^2)
    (the softmax of N(0, v) logits tilts them to N(v, v): H = ln E[e^x] + ln L - E_p[x]),
    so the target ln L - D is met at tau = sigma / sqrt(2 D)."""
    L = 400000
    s = rng(13).normal(size=L) * sigma
    tau = O.entropy_matched_tau(s, math.log(L) - target_drop)
    assert abs(tau / (sigma / math.sqrt(2 * target_drop)) - 1) < 0.02


def test_entropy_matched_tau_residual_scale_and_range():
    r = rng(14)
    s = r.normal(size=2000) * 1.7
    for target in (1.0, 3.0, 6.0, 7.5):
        tau = O.entropy_matched_tau(s, target)
        assert abs(O.entropy(O.calibrate(s, tau)) - target) < 1e-9
        assert abs(O.entropy_matched_tau(4 * s, target) / tau - 4) < 1e-9     # scale equivariant
    taus = [O.entropy_matched_tau(s, t) for t in (2.0, 4.0, 6.0)]
    assert taus[0] < taus[1] < taus[2]                                          # monotone
    assert O.entropy_matched_tau(s, math.log(s.size) + 1) == O.TAU_MAX         # unreachable
    assert O.entropy_matched_tau(s, -1.0) == O.TAU_MIN
    assert O.entropy_matched_tau(np.array([2.0]), 0.3) == 1.0


# ---------------------------------------------------------------- MTI policy

def test_mti_policy_thresholds_and_break_even():
    # one-off write (1 per byte) against a 0.5 per byte scattered-read surcharge:
    # rewriting pays once the selection is read in more than 2 later steps
    assert not O.mti_rewrite(1000, 0, 64, 10 ** 6, 0.5)      # reselected every step
    assert not O.mti_rewrite(1000, 2, 64, 10 ** 6, 0.5)      # 2 * 0.5 = 1: break-even, no gain
    assert O.mti_rewrite(1000, 3, 64, 10 ** 6, 0.5)
    assert O.mti_rewrite(1000, 15, 64, 10 ** 6, 0.5)
    assert not O.mti_rewrite(10, 15, 64, 10 ** 6, 0.5)       # below L_lower: load in place
    assert O.mti_rewrite(5000, 0, 64, 4096, 0.5)             # above L_upper: rewrite
    assert O.mti_rewrite(64, 15, 64, 64, 0.5) and not O.mti_rewrite(63, 15, 64, 64, 0.5)
