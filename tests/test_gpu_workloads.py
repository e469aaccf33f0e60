"""Multi-step workloads at full size: the GPU runs every sequence through every decode
step (fused step, the launch configuration the benchmark uses); the fp64 oracle follows
sampled (sequence, KV-head) units from the same initial state with the same per-step
inputs. Per step and sampled unit: boundaries and block moves bit-exact, masks within
the flip rule, compaction bit-exact when the masks agree, Condensed slots and weights
bit-exact (until a merge near-tie, after which the unit may legitimately diverge),
attention within the bf16 bounds."""
import numpy as np
import pytest
import torch

from attention_kv_head_b200 import binding as B
from attention_kv_head_b200 import synth
from attention_kv_head_b200.cache import DecodeCache
from oracle import hardkv_oracle as O
from tests import gpu_util as U
from tests.test_gpu_parity import oracle_unit_from_state

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def sample_units(w, st, k=16):
    """At least k units: first, last, middle; the units with the lowest and highest key
    temperature (flattest and most peaked scores: the most and the fewest kept, so the
    clamp and the threshold extremes); for ragged batches the shortest and longest
    sequences; the rest seeded-random."""
    B_, H = w.batch, w.n_kv_heads
    picks = [(0, 0), (B_ - 1, H - 1), (B_ // 2, H // 2)]
    temps = np.array([[synth.temperature(w, b, h) for h in range(H)] for b in range(B_)])
    order = np.argsort(temps, axis=None)
    for flat in order[:3].tolist() + order[-3:].tolist():
        picks.append(divmod(int(flat), H))
    if w.context is None:
        picks += [(int(np.argmin(st.lens)), 1 % H), (int(np.argmax(st.lens)), 2 % H)]
    rng = np.random.default_rng(1234)
    picks = list(dict.fromkeys(picks))
    while len(picks) < k:
        bh = (int(rng.integers(B_)), int(rng.integers(H)))
        if bh not in picks:
            picks.append(bh)
    return picks


MERGE_TIE = U.MERGE_TIE


_STATES: dict = {}


def state_of(w):
    """Initial host state, generated once per workload (the p sweep reuses it)."""
    if w.name not in _STATES:
        _STATES.clear()
        _STATES[w.name] = synth.initial_state(w, threads=16)
    return _STATES[w.name]


def run_and_compare(w, p, select_on_move):
    st = state_of(w)
    dc = DecodeCache.from_state(st)
    picks = sample_units(w, st)
    units = {bh: oracle_unit_from_state(st, *bh, steps=w.steps) for bh in picks}
    cmp = U.StepCompare(w.dtype)
    G, H = w.group, w.n_kv_heads
    diverged = set()
    flips_per_unit = {}
    moves = merged = ties = 0
    rows = torch.tensor([b * H + h for (b, h) in picks], device=dc.device)
    flat = lambda x: x.reshape(w.batch * H, *x.shape[2:]).index_select(0, rows).cpu()
    for t in range(w.steps):
        (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, t)
        reselect = "moved" if (select_on_move and t > 0) else "all"
        mode = B.SELECT_MOVED if reselect == "moved" else B.SELECT_ALL
        mask, out = U.run_fused_step(dc, q, k, v, p, select_mode=mode)
        torch.cuda.synchronize()
        m = flat(mask).numpy().view(np.uint32)
        n_kept = flat(dc.n_kept).numpy()
        sp_idx = flat(dc.sp_idx).numpy()
        w_cd = flat(dc.w_cd).numpy()
        k_cd = U.device_rows(flat(dc.k_cd))
        v_cd = U.device_rows(flat(dc.v_cd))
        o = out.cpu().numpy()
        bounds = [x.cpu().numpy() for x in (dc.len, dc.d_lo, dc.s_lo, dc.moved)]
        for i, (b, h) in enumerate(picks):
            if (b, h) in diverged:
                continue
            un = units[b, h]
            res = un.step(q_ex[b, h * G:(h + 1) * G], k_ex[b, h], v_ex[b, h], 1.0, p,
                          reselect=reselect)
            assert (bounds[0][b], bounds[1][b], bounds[2][b], bool(bounds[3][b])) == \
                (un.len, un.d_lo, un.s_lo, res.moved), (t, b, h)
            moves += int(res.moved)
            if res.merge is not None and res.merge.gaps:
                merged += len(res.merge.gaps)
                ties += sum(g_ <= MERGE_TIE for g_ in res.merge.gaps)
                if min(res.merge.gaps) <= MERGE_TIE:
                    diverged.add((b, h))
                    continue
            assert np.array_equal(w_cd[i], un.cd_w.astype(np.float32)), (t, b, h)
            assert np.array_equal(k_cd[i], un.cd_k), (t, b, h)
            assert np.array_equal(v_cd[i], un.cd_v), (t, b, h)
            same, ref = True, res.out
            if res.sel is not None:
                L = un.d_lo - un.s_lo
                kept = U.mask_bits(m[i], L)
                same = cmp.selection(res.sel, p, kept)
                if not same:
                    # the accepted GPU set becomes the unit's set: attention this step
                    # is evaluated on it and a unit that keeps its set carries it on
                    U.adopt_selection(un, kept)
                    ref = un.attend(q_ex[b, h * G:(h + 1) * G])
                    flips_per_unit[b, h] = flips_per_unit.get((b, h), 0) + 1
            assert n_kept[i] == un.n and np.array_equal(sp_idx[i], un.idx), (t, b, h)
            cmp.attention(o[b, h * G:(h + 1) * G], ref, flipped=not same)
    status = dc.read_status()
    assert status[B.ST_FLAGS] == 0, status
    # device counters against the final bookkeeping: every block move shifts d_lo by
    # one block; a reselecting step selects every KV head of the sequences it covers
    n_moves = (dc.d_lo.cpu().numpy() - st.d_lo0) // w.block
    assert status[B.ST_MOVES] == n_moves.sum()
    if select_on_move:
        assert status[B.ST_SELECTIONS] == H * (w.batch + n_moves.sum())
    else:
        assert status[B.ST_SELECTIONS] == H * w.batch * w.steps
    if w.condense_mode == synth.MERGE:
        assert status[B.ST_MERGED] == H * w.block * n_moves.sum()
    assert len(diverged) <= len(picks) // 2
    U.record("workload", workload=w.name, p=p, steps=w.steps, units_followed=len(picks),
             oracle_moves=moves, oracle_merged_tokens=merged, oracle_merge_near_ties=ties,
             diverged_after_near_tie=len(diverged),
             device_clamps=int(status[B.ST_CLAMPS]), device_near_ties=int(status[B.ST_NEAR_TIES]),
             device_selections=int(status[B.ST_SELECTIONS]),
             flips_per_unit={f"{b},{h}": c for (b, h), c in flips_per_unit.items()},
             **cmp.summary())
    print(w.name, p, "units", len(picks), "oracle moves", moves, "oracle merges", merged,
          "diverged", len(diverged), "flipped", cmp.flipped_units, cmp.flipped_tokens,
          "compared", cmp.units, "worst abs", cmp.worst_abs, "rel", cmp.worst_rel,
          "clamps", int(status[B.ST_CLAMPS]), "near-ties", int(status[B.ST_NEAR_TIES]))
    return status, n_moves


@pytest.mark.parametrize("p", [0.8, 0.9, 0.95])
def test_long16k_every_step_reselection(p):
    """batch 32, context 16384, Cap 25%: 64 steps with a fresh selection each step,
    block moves at steps 16, 32, 48, eviction."""
    _, n_moves = run_and_compare(synth.WORKLOADS["long16k"], p, select_on_move=False)
    assert np.all(n_moves == 3)


def test_contbatch_ragged_merge_reselect_on_move():
    """batch 64, contexts U[1024, 32768], 256 steps: a sequence reselects only on its
    block move; weighted merge into 512 slots."""
    _, n_moves = run_and_compare(synth.WORKLOADS["contbatch"], 0.9, select_on_move=True)
    assert np.all(n_moves == 15)


def test_stress64k_spikes_merge():
    """batch 16, 40/8 heads, context 65536, planted spikes, Cap 15%: 128 steps with a
    fresh selection each step, weighted merge into 1024 slots."""
    _, n_moves = run_and_compare(synth.WORKLOADS["stress64k"], 0.95, select_on_move=False)
    assert np.all(n_moves == 7)


@pytest.mark.parametrize("name,launches", [("long16k", 24), ("stress64k", 12)])
def test_score_kernel_repeated_launches_full_size(name, launches):
    """Every score of every unit, over repeated launches of the score stage at full size,
    within 1e-5 relative of the oracle's fp64 scores. (A stage of the key pipeline reused
    before all of its readers were done corrupts a few rows of a tile now and then; this
    catches it where single launches and sampled units would not.)"""
    w = synth.WORKLOADS[name]
    st = state_of(w)
    dc = DecodeCache.from_state(st)
    (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, 0)
    dc.append(k, v)
    torch.cuda.synchronize()
    G, H = w.group, w.n_kv_heads
    ref, scale = {}, {}
    for b in range(w.batch):
        # the Sparse candidates are rows of the uploaded initial state (the append only
        # adds a Dense row); the oracle scores them from the host arrays
        pos = np.arange(int(st.s_lo0[b]), int(st.d_lo0[b])) % st.R
        for h in range(H):
            kk = U.storage_exact(st.k_ring[b, h, pos], w.dtype)
            ref[b, h] = O.score(q_ex[b, h * G:(h + 1) * G], kk)
            scale[b, h] = max(1.0, float(np.abs(ref[b, h]).max()))
    for t in range(launches):
        mask = dc.new_mask()
        dc.score_calibrate_topp(q, synth.p_values(w)[0], mask)
        torch.cuda.synchronize()
        sc = U.scores_from_ws(dc)
        for (b, h), r in ref.items():
            got = sc[b * H + h, :r.size].astype(np.float64)
            err = np.abs(got - r).max()
            assert err <= 1e-5 * scale[b, h], (t, b, h, err)
    assert dc.read_status()[B.ST_FLAGS] == 0
