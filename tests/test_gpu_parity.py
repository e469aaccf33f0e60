"""GPU (sm_100a) vs fp64 oracle on the same seeded inputs, through the C ABI.

Bars: compaction indices, kept counts and boundaries bit-exact; masks identical except
near-threshold tokens (oracle.allowed_flips, counted); attention max-abs <= 1e-2 and
rel-L2 <= 2e-3 for bf16 (1e-4 / 1e-5 for fp32 storage); scores within 1e-5 relative.
"""
import numpy as np
import pytest
import torch

from attention_kv_head_b200 import binding as B
from attention_kv_head_b200 import synth
from attention_kv_head_b200.cache import DecodeCache
from oracle import hardkv_oracle as O
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


oracle_unit_from_state = U.oracle_unit_from_state


SMALL = {
    "bf16_d128_g4": synth.small(),
    "bf16_d64_g5": synth.small(n_q_heads=10, n_kv_heads=2, head_dim=64),
    "f32_d64_g1": synth.small(dtype=synth.F32, n_q_heads=2, n_kv_heads=2, head_dim=64),
    "f32_d128_g4": synth.small(dtype=synth.F32),
    "bf16_g16": synth.small(n_q_heads=32, n_kv_heads=2),
    "bf16_g8_d64": synth.small(n_q_heads=16, n_kv_heads=2, head_dim=64, temp_range=(2.0, 6.0)),
    "clamp": synth.small(sparse_cap=100),
    "keep_all": synth.small(p=1.0),
    "keep_all_clamped": synth.small(p=1.0, sparse_cap=50),
    "ring_wrap": synth.small(context=1000, condensed_slots=400),
    "no_sparse": synth.small(context=72, dense_window=48, condensed_slots=24),
    "p_low": synth.small(p=0.3, temp_range=(0.25, 8.0)),
    "batch5": synth.small(batch=5, context=333, sparse_cap=250),
}


def compare_step(w, st, dc, mask, out, units, q_ex, k_ex, v_ex, p, cmp, tau=None):
    """Steps every oracle unit once and checks the GPU's step against it: boundaries,
    mask (flip rule), compaction of the GPU's own mask bit-exact, attention on the GPU's
    mask for every unit (a flipped unit's oracle set is the GPU's accepted one)."""
    G = w.group
    m = mask.cpu().numpy().view(np.uint32)
    n_kept = dc.n_kept.cpu().numpy()
    sp_idx = dc.sp_idx.cpu().numpy()
    k_sp = U.device_rows(dc.k_sp)
    v_sp = U.device_rows(dc.v_sp)
    o = out.cpu().numpy()
    lens, dlo, slo = (t.cpu().numpy() for t in (dc.len, dc.d_lo, dc.s_lo))
    results = {}
    for (b, h), unit in units.items():
        qg = q_ex[b, h * G:(h + 1) * G]
        res = unit.step(qg, k_ex[b, h], v_ex[b, h], U.tau_of(tau, b, h), p)
        assert (lens[b], dlo[b], slo[b]) == (unit.len, unit.d_lo, unit.s_lo)
        L = unit.d_lo - unit.s_lo
        kept = U.mask_bits(m[b, h], L)
        allbits = U.mask_bits(m[b, h], m.shape[-1] * 32)
        assert np.all(allbits < L)                      # no bit past the Sparse length
        n = int(n_kept[b, h])
        assert n == min(kept.size, w.sparse_cap) == kept.size
        assert np.array_equal(sp_idx[b, h, :n], unit.s_lo + kept)
        assert np.all(sp_idx[b, h, n:] == -1)
        # compact rows are byte-identical to the raw rows of those positions
        assert np.array_equal(k_sp[b, h, :n], unit.K[sp_idx[b, h, :n]])
        assert np.array_equal(v_sp[b, h, :n], unit.V[sp_idx[b, h, :n]])
        same = cmp.selection(res.sel, p, kept) if res.sel is not None else True
        if same:
            assert n == res.n and np.array_equal(sp_idx[b, h], res.idx)
            ref = res.out
        else:
            U.adopt_selection(unit, kept)
            ref = unit.attend(qg)
        cmp.attention(o[b, h * G:(h + 1) * G], ref, flipped=not same)
        results[b, h] = (res, same, ref)
    return results


def run_small_step(name, w, tau_np):
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    dc2 = DecodeCache.from_state(st)
    (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, 0)
    tau = None if tau_np is None else torch.from_numpy(tau_np).to(dc.device)
    p = synth.p_values(w)[0]
    mask, out = U.run_unfused_step(dc, q, k, v, p, tau=tau)
    mask2, out2 = U.run_fused_step(dc2, q, k, v, p, tau=tau)
    torch.cuda.synchronize()
    units = {(b, h): oracle_unit_from_state(st, b, h) for b in range(w.batch)
             for h in range(w.n_kv_heads)}
    # scores (white box): fp32 vs fp64 within 1e-5 relative to the unit's scale
    sc = U.scores_from_ws(dc)
    for (b, h), un in units.items():
        L = int(st.d_lo0[b] - st.s_lo0[b])
        if L == 0:
            continue
        ref = O.score(q_ex[b, h * w.group:(h + 1) * w.group], un.K[un.s_lo:un.d_lo])
        got = sc[b * w.n_kv_heads + h, :L]
        assert np.allclose(got, ref, rtol=1e-5, atol=1e-5 * np.abs(ref).max()), name
    cmp = U.StepCompare(w.dtype)
    results = compare_step(w, st, dc, mask, out, units, q_ex, k_ex, v_ex, p, cmp, tau=tau_np)
    # fused step == unfused path (selection, compaction and bookkeeping bit for bit)
    assert torch.equal(mask, mask2)
    assert torch.equal(dc.n_kept, dc2.n_kept) and torch.equal(dc.sp_idx, dc2.sp_idx)
    for t1, t2 in ((dc.len, dc2.len), (dc.d_lo, dc2.d_lo), (dc.s_lo, dc2.s_lo)):
        assert torch.equal(t1, t2)
    n = dc.n_kept.cpu().numpy()
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            assert torch.equal(dc.k_sp[b, h, :n[b, h]], dc2.k_sp[b, h, :n[b, h]])
            assert torch.equal(dc.v_sp[b, h, :n[b, h]], dc2.v_sp[b, h, :n[b, h]])
    # the fused path splits the work by cost (gathered rows weigh more), the standalone
    # attention by rows: same math, different split-K summation order, so the fused
    # output is held to the oracle bound itself (on the same, GPU-chosen mask)
    o2 = out2.cpu().numpy()
    for (b, h), (res, same, ref) in results.items():
        cmp.attention(o2[b, h * w.group:(h + 1) * w.group], ref, flipped=not same)
    st_words = dc.read_status()
    assert st_words[B.ST_FLAGS] == 0
    assert st_words[B.ST_SELECTIONS] == w.units
    # clamps counted on the device = the oracle's (a flip at the boundary may move one)
    assert abs(int(st_words[B.ST_CLAMPS]) - cmp.clamps) <= cmp.flipped_units
    U.record("small_step", name=name, tau=tau_np is not None, **cmp.summary())
    print(name, "tau" if tau_np is not None else "", cmp.summary())


@pytest.mark.parametrize("name", list(SMALL))
def test_small_step_unfused_vs_oracle_and_fused(name):
    run_small_step(name, SMALL[name], None)


TAU_CASES = ["bf16_d128_g4", "f32_d64_g1", "bf16_g16", "clamp", "p_low", "batch5", "keep_all_clamped"]


@pytest.mark.parametrize("name", TAU_CASES)
def test_small_step_with_calibration_temperatures(name):
    """Caller-supplied temperatures tau[b,h] log-uniform in [0.25, 8] (unit (0,0) = 1)
    drive the calibration softmax(s / tau) of both the separate and the fused path."""
    w = SMALL[name]
    run_small_step(name, w, synth.calibration_taus(w))


@pytest.mark.parametrize("frac,cap", [(0.3, 600), (0.9, 200), (0.0, 600), (1.0, 600)])
@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32])
def test_regularize_and_attention_given_mask(frac, cap, dtype):
    """A seeded mask drives both sides: compaction bit-exact, attention within tolerance."""
    w = synth.small(dtype=dtype, sparse_cap=cap)
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, 0)
    dc.append(k, v)
    masks = {}
    mask_np = np.zeros((w.batch, w.n_kv_heads, dc.mask_words), np.uint32)
    for b in range(w.batch):
        L = int(st.d_lo0[b] - st.s_lo0[b])
        for h in range(w.n_kv_heads):
            mk = synth.random_mask(w, b, h, L, frac)
            masks[b, h] = mk
            bits = np.zeros(dc.mask_words * 32, np.uint32)
            bits[:L] = mk
            mask_np[b, h] = (bits.reshape(-1, 32) << np.arange(32, dtype=np.uint32)).sum(1)
            # bits past the Sparse length must be ignored by the kernel
            mask_np[b, h, -1] |= np.uint32(0x80000000)
    mask = torch.from_numpy(mask_np.view(np.int32)).to(dc.device)
    dc.regularize(mask)
    out = torch.empty(w.batch, w.n_q_heads, w.head_dim, device=dc.device)
    dc.decode_attn(q, out)
    torch.cuda.synchronize()
    n_kept = dc.n_kept.cpu().numpy()
    sp_idx = dc.sp_idx.cpu().numpy()
    k_sp, v_sp = U.device_rows(dc.k_sp), U.device_rows(dc.v_sp)
    o = out.cpu().numpy()
    cmp = U.StepCompare(dtype)
    clamps = 0
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            un = oracle_unit_from_state(st, b, h)
            un.append(k_ex[b, h], v_ex[b, h])
            pos = np.arange(un.s_lo, un.d_lo)
            n, idx, kc, vc = O.regularize(masks[b, h], pos, un.K[un.s_lo:un.d_lo],
                                          un.V[un.s_lo:un.d_lo], cap)
            clamps += int(masks[b, h].sum() > cap)
            assert n_kept[b, h] == n
            assert np.array_equal(sp_idx[b, h], idx)
            assert np.array_equal(k_sp[b, h, :n], kc) and np.array_equal(v_sp[b, h, :n], vc)
            un.n, un.idx, un.sp_k, un.sp_v = n, idx, kc, vc
            cmp.attention(o[b, h * w.group:(h + 1) * w.group],
                          un.attend(q_ex[b, h * w.group:(h + 1) * w.group]))
    assert dc.read_status()[B.ST_CLAMPS] == clamps


def test_uniform_and_one_hot_heads():
    """Planted keys: a head whose candidates are all equal keeps ceil(p n) lowest
    positions; a head with one dominant key keeps exactly that key."""
    w = synth.small(batch=1, n_kv_heads=2, n_q_heads=8, p=0.6)
    st = synth.initial_state(w)
    R, C = st.R, w.condensed_slots
    L0 = int(st.len0[0])
    pos = np.arange(C, L0)
    st.k_ring[0, 0, pos % R] = st.k_ring[0, 0, C % R]        # head 0: all keys identical
    hot = int(C + (L0 - C) // 3)
    st.k_ring[0, 1, pos % R] = 0                              # head 1: zero keys ...
    st.k_ring[0, 1, hot % R] = synth.to_bf16_bits(np.full(w.head_dim, 30.0, np.float32))
    dc = DecodeCache.from_state(st)
    (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, 0)
    qh = q_ex.copy()
    # make every query of head 1 positive so the planted key dominates
    q_dev = q.clone()
    q_dev[0, 4:8] = q_dev[0, 4:8].abs()
    qh[0, 4:8] = np.abs(qh[0, 4:8])
    mask, out = U.run_unfused_step(dc, q_dev, k, v, w.p)
    torch.cuda.synchronize()
    m = mask.cpu().numpy().view(np.uint32)
    L = int(dc.d_lo[0] - dc.s_lo[0])
    kept0 = U.mask_bits(m[0, 0], L)
    p32 = float(np.float32(w.p))
    assert kept0.tolist() == list(range(int(np.ceil(p32 * L))))
    kept1 = U.mask_bits(m[0, 1], L)
    assert kept1.tolist() == [hot - C]
    for h in range(2):
        un = oracle_unit_from_state(st, 0, h)
        res = un.step(qh[0, h * 4:(h + 1) * 4], k_ex[0, h], v_ex[0, h], 1.0, w.p)
        assert res.sel.kept.tolist() == (kept0 if h == 0 else kept1).tolist()


@pytest.mark.parametrize("mode", [synth.MERGE, synth.EVICT])
@pytest.mark.parametrize("select", ["all", "moved"])
def test_multistep_small(mode, select):
    """40 steps: block moves every 16 steps, merges into the Condensed tier, per-step
    parity of boundaries, masks, compaction, Condensed state and attention."""
    w = synth.small(condense_mode=mode, steps=40, batch=2, context=300 + 0)
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    units = {(b, h): oracle_unit_from_state(st, b, h, steps=w.steps) for b in range(w.batch)
             for h in range(w.n_kv_heads)}
    sel_mode = B.SELECT_ALL if select == "all" else B.SELECT_MOVED
    cmp = U.StepCompare(w.dtype)
    G = w.group
    diverged = set()
    for t in range(w.steps):
        (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, t)
        if t == 0 and select == "moved":
            mask, out = U.run_fused_step(dc, q, k, v, w.p, select_mode=B.SELECT_ALL)
            rs = "all"
        else:
            mask, out = U.run_fused_step(dc, q, k, v, w.p, select_mode=sel_mode)
            rs = select
        torch.cuda.synchronize()
        m = mask.cpu().numpy().view(np.uint32)
        n_kept, sp_idx = dc.n_kept.cpu().numpy(), dc.sp_idx.cpu().numpy()
        k_cd, v_cd = U.device_rows(dc.k_cd), U.device_rows(dc.v_cd)
        w_cd = dc.w_cd.cpu().numpy()
        o = out.cpu().numpy()
        bounds = [t_.cpu().numpy() for t_ in (dc.len, dc.d_lo, dc.s_lo, dc.moved)]
        for (b, h), un in units.items():
            if (b, h) in diverged:
                continue
            res = un.step(q_ex[b, h * G:(h + 1) * G], k_ex[b, h], v_ex[b, h], 1.0, w.p, reselect=rs)
            assert (bounds[0][b], bounds[1][b], bounds[2][b], bool(bounds[3][b])) == \
                (un.len, un.d_lo, un.s_lo, res.moved)
            if res.merge is not None and res.merge.gaps and min(res.merge.gaps) <= U.MERGE_TIE:
                diverged.add((b, h))      # a near-tie may legitimately pick another slot
                continue
            assert np.array_equal(w_cd[b, h], un.cd_w.astype(np.float32))
            assert np.array_equal(k_cd[b, h], un.cd_k) and np.array_equal(v_cd[b, h], un.cd_v)
            same, ref = True, res.out
            if res.sel is not None:
                L = un.d_lo - un.s_lo
                kept = U.mask_bits(m[b, h], L)
                same = cmp.selection(res.sel, w.p, kept)
                if not same:          # carry the accepted GPU set on (select on move keeps it)
                    U.adopt_selection(un, kept)
                    ref = un.attend(q_ex[b, h * G:(h + 1) * G])
            assert n_kept[b, h] == un.n and np.array_equal(sp_idx[b, h], un.idx)
            cmp.attention(o[b, h * G:(h + 1) * G], ref, flipped=not same)
    assert dc.read_status()[B.ST_FLAGS] == 0
    assert len(diverged) <= 1
    U.record("multistep_small", mode=mode, select=select, diverged=len(diverged), **cmp.summary())


@pytest.mark.parametrize("with_tau", [False, True], ids=["tau1", "tau"])
@pytest.mark.parametrize("name", ["pr1", "llama8b_8k"])
def test_full_size_single_step(name, with_tau):
    """The single-step workloads at full size, every unit against the oracle; with_tau:
    caller-supplied calibration temperatures log-uniform in [0.25, 8]."""
    w = synth.WORKLOADS[name]
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, 0)
    tau_np = synth.calibration_taus(w) if with_tau else None
    tau = None if tau_np is None else torch.from_numpy(tau_np).to(dc.device)
    mask, out = U.run_fused_step(dc, q, k, v, w.p, tau=tau)
    torch.cuda.synchronize()
    units = {(b, h): oracle_unit_from_state(st, b, h) for b in range(w.batch)
             for h in range(w.n_kv_heads)}
    cmp = U.StepCompare(w.dtype)
    compare_step(w, st, dc, mask, out, units, q_ex, k_ex, v_ex, w.p, cmp, tau=tau_np)
    assert cmp.flipped_units <= max(1, w.units // 50)
    status = dc.read_status()
    assert status[B.ST_FLAGS] == 0
    U.record("full_size", workload=name, tau=with_tau, kept=int(dc.n_kept.sum().item()),
             device_clamps=int(status[B.ST_CLAMPS]), **cmp.summary())
    print(name, with_tau, cmp.summary(), "kept", dc.n_kept.sum().item())


def test_graph_capture_replays_the_step():
    w = synth.small(batch=3)
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    (q, k, v), _ = U.upload_step(dc, w, st, 0)
    snap = dc.snapshot_bounds()
    mask_e, out_e = U.run_fused_step(dc, q, k, v, w.p)
    torch.cuda.synchronize()
    mask_e, out_e = mask_e.clone(), out_e.clone()
    dc.restore_bounds(snap)
    mask = dc.new_mask()
    out = torch.empty_like(out_e)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        dc.step(q, k, v, out, w.p, mask=mask, stream=s)   # warm-up (sets kernel attributes)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    dc.restore_bounds(snap)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dc.step(q, k, v, out, w.p, mask=mask)
    for _ in range(3):
        dc.restore_bounds(snap)
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, out_e) and torch.equal(mask, mask_e)


@pytest.mark.parametrize("pinned", [(1, 1, 1, 1), (0, 0, 0, 0), (1, 1, 0, 1), (0, 1, 1, 0)],
                         ids=["pinned", "pageable", "mixed_kv", "mixed_out"])
@pytest.mark.parametrize("with_tau", [False, True], ids=["tau1", "tau"])
def test_host_entry_point_matches_device_step(pinned, with_tau):
    """Host buffers: pinned mapped ones are used in place by the kernels, pageable ones
    are staged by copies (tau always is); every combination gives the device step's
    result."""
    w = synth.small(batch=2)
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    dc2 = DecodeCache.from_state(st)
    (q, k, v), _ = U.upload_step(dc, w, st, 0)
    tau_np = synth.calibration_taus(w) if with_tau else None
    tau = None if tau_np is None else torch.from_numpy(tau_np).to(dc.device)
    mask = dc.new_mask()
    out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
    dc.step(q, k, v, out, w.p, tau=tau, mask=mask)
    host = [t.cpu() for t in (q, k, v)] + [torch.full(out.shape, float("nan"))]
    qh, kh, vh, oh = (t.pin_memory() if pn else t for t, pn in zip(host, pinned))
    tau_h = None if tau_np is None else torch.from_numpy(tau_np.copy())
    mask2 = dc2.new_mask()
    dc2.step_host(qh, kh, vh, oh, w.p, tau=tau_h, mask=mask2)
    torch.cuda.synchronize()
    assert torch.equal(oh, out.cpu())
    assert torch.equal(mask2, mask)
    assert torch.equal(dc2.len, dc.len) and torch.equal(dc2.sp_idx, dc.sp_idx)
    if with_tau:   # the temperatures changed the selection (they are not all 1)
        dc3 = DecodeCache.from_state(st)
        mask3 = dc3.new_mask()
        dc3.step(q, k, v, torch.empty_like(out), w.p, mask=mask3)
        torch.cuda.synchronize()
        assert not torch.equal(mask3, mask)


def topk_eps(s: np.ndarray) -> float:
    """Score rounding the top-k rule may see: the GPU's fp32 scores are within 1e-5 of
    the fp64 ones relative to the unit's largest |s| (checked above), so two candidates
    can swap only if their exact scores are within twice that."""
    return 2e-5 * max(1.0, float(np.abs(s).max()) if s.size else 1.0)


def check_selection_units(w, st, dc, mask, q_ex, k_ex, v_ex, check, units=None):
    """Append-stepped oracle units vs the GPU mask: `check(un, qg, L, kept)` returns the
    oracle set the GPU's kept set was accepted against (positions, local)."""
    G = w.group
    m = mask.cpu().numpy().view(np.uint32)
    units = units or {(b, h): oracle_unit_from_state(st, b, h) for b in range(w.batch)
                      for h in range(w.n_kv_heads)}
    for (b, h), un in units.items():
        un.append(k_ex[b, h], v_ex[b, h])
        L = un.d_lo - un.s_lo
        kept = U.mask_bits(m[b, h], L)
        check(b, h, un, q_ex[b, h * G:(h + 1) * G], L, kept)
    return units


@pytest.mark.parametrize("name", ["bf16_d128_g4", "f32_d64_g1", "bf16_g16", "batch5", "bf16_d64_g5"])
@pytest.mark.parametrize("kfrac", [0.0, 0.1, 0.5, 1.0])
def test_topk_selection_separate_and_fused(name, kfrac):
    """Fixed-budget top-k (hardkv_score_topk and the fused step's RULE_TOPK) against the
    oracle's top_k: the k best scores, ties to the lower position; indices bit-exact
    except candidates whose exact score lies within the fp32 score rounding of the k-th
    score; compaction and attention as for top-p."""
    w = SMALL[name]
    k_sel = max(1, int(round(kfrac * w.sparse_cap)))
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    dc2 = DecodeCache.from_state(st)
    (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, 0)
    dc.append(k, v)
    mask = dc.new_mask()
    dc.score_topk(q, k_sel, mask)
    mask2 = dc2.new_mask()
    out2 = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
    dc2.step(q, k, v, out2, 1.0, mask=mask2, rule=B.RULE_TOPK, top_k=k_sel)
    torch.cuda.synchronize()
    assert torch.equal(mask, mask2)
    cmp = U.StepCompare(w.dtype)
    n_kept = dc2.n_kept.cpu().numpy()
    sp_idx = dc2.sp_idx.cpu().numpy()
    o2 = out2.cpu().numpy()
    flips = [0, 0]

    def check(b, h, un, qg, L, kept):
        s = O.score(qg, un.K[un.s_lo:un.d_lo])
        sel = O.top_k(s, k_sel)
        ok, nd = O.allowed_flips_topk(s, sel, kept, topk_eps(s))
        assert ok, (name, b, h, nd)
        flips[0] += int(nd > 0)
        flips[1] += nd
        assert kept.size == min(k_sel, L) == n_kept[b, h]
        assert np.array_equal(sp_idx[b, h, :kept.size], un.s_lo + kept)
        U.adopt_selection(un, kept)
        cmp.attention(o2[b, h * w.group:(h + 1) * w.group], un.attend(qg), flipped=nd > 0)

    check_selection_units(w, st, dc, mask, q_ex, k_ex, v_ex, check)
    status = dc2.read_status()
    assert status[B.ST_FLAGS] == 0 and status[B.ST_CLAMPS] == 0
    U.record("topk", name=name, k=k_sel, flipped_units=flips[0], flipped_tokens=flips[1],
             attention_units=cmp.units, worst_abs=cmp.worst_abs, worst_rel_l2=cmp.worst_rel)


ENTROPY_CASES = ["bf16_d128_g4", "f32_d64_g1", "f32_d128_g4", "bf16_g16", "bf16_g8_d64", "p_low",
                 "clamp", "batch5", "no_sparse"]


@pytest.mark.parametrize("name", ENTROPY_CASES)
def test_entropy_matched_calibration_separate_and_fused(name):
    """Entropy-matched temperatures: each unit's tau (tau_out) within 1e-4 relative of the
    oracle's bisection root of H(softmax(s/tau)) = mean_g H(raw attention of g); the mask
    within the flip rule of the oracle's top-p at that tau (the oracle's masks at its own
    tau are counted too); the fused step reproduces the separate call bit for bit."""
    w = SMALL[name]
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    dc2 = DecodeCache.from_state(st)
    (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, 0)
    p = synth.p_values(w)[0]
    dc.append(k, v)
    mask = dc.new_mask()
    tau_out = torch.zeros(w.batch, w.n_kv_heads, dtype=torch.float32, device=dc.device)
    dc.score_calibrate_entropy_topp(q, p, mask, tau_out=tau_out)
    mask2 = dc2.new_mask()
    tau2 = torch.zeros_like(tau_out)
    out2 = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
    dc2.step(q, k, v, out2, p, mask=mask2, calibration=B.CAL_ENTROPY, tau_out=tau2)
    torch.cuda.synchronize()
    assert torch.equal(mask, mask2) and torch.equal(tau_out, tau2)
    taus = tau_out.cpu().numpy()
    o2 = out2.cpu().numpy()
    cmp = U.StepCompare(w.dtype)
    stats = {"worst_tau_rel": 0.0, "masks_differing_at_oracle_tau": 0}

    def check(b, h, un, qg, L, kept):
        K = un.K[un.s_lo:un.d_lo]
        s = O.score(qg, K)
        tau_or = O.entropy_matched_tau(s, O.attention_entropy(qg, K))
        tg = float(taus[b, h])
        rel = abs(tg / tau_or - 1.0)
        stats["worst_tau_rel"] = max(stats["worst_tau_rel"], rel)
        assert rel <= 1e-4, (name, b, h, tg, tau_or)
        if w.group == 1 and L > 1:
            assert abs(tg - 1.0) <= 1e-4           # one query: the raw attention itself
        sel = O.top_p(s, tg, p, w.sparse_cap)
        same = cmp.selection(sel, p, kept)
        stats["masks_differing_at_oracle_tau"] += int(
            not np.array_equal(O.top_p(s, tau_or, p, w.sparse_cap).kept, kept))
        U.adopt_selection(un, kept)
        cmp.attention(o2[b, h * w.group:(h + 1) * w.group], un.attend(qg), flipped=not same)

    check_selection_units(w, st, dc, mask, q_ex, k_ex, v_ex, check)
    assert dc.read_status()[B.ST_FLAGS] == 0
    U.record("entropy", name=name, taus=[float(x) for x in taus.reshape(-1)[:8]], **stats,
             **cmp.summary())
    print(name, stats, cmp.summary())


@pytest.mark.parametrize("mode", ["topk", "entropy"])
def test_full_size_topk_and_entropy(mode):
    """llama8b_8k at full size, every unit: the fixed budget at the top-p run's mean kept
    count (the same-box A/B of the pages' fixed-budget comparison), and the
    entropy-matched calibration."""
    w = synth.WORKLOADS["llama8b_8k"]
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, 0)
    out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
    mask = dc.new_mask()
    tau_out = torch.zeros(w.batch, w.n_kv_heads, dtype=torch.float32, device=dc.device)
    k_sel = 3638   # mean kept count of the calibrated top-p step (232804 / 64 units)
    if mode == "topk":
        dc.step(q, k, v, out, 1.0, mask=mask, rule=B.RULE_TOPK, top_k=k_sel)
    else:
        dc.step(q, k, v, out, w.p, mask=mask, calibration=B.CAL_ENTROPY, tau_out=tau_out)
    torch.cuda.synchronize()
    taus = tau_out.cpu().numpy()
    o = out.cpu().numpy()
    cmp = U.StepCompare(w.dtype)
    worst = [0.0, 0]

    def check(b, h, un, qg, L, kept):
        K = un.K[un.s_lo:un.d_lo]
        s = O.score(qg, K)
        if mode == "topk":
            ok, nd = O.allowed_flips_topk(s, O.top_k(s, k_sel), kept, topk_eps(s))
            assert ok, (b, h, nd)
            worst[1] += int(nd > 0)
            flipped = nd > 0
        else:
            tau_or = O.entropy_matched_tau(s, O.attention_entropy(qg, K))
            worst[0] = max(worst[0], abs(float(taus[b, h]) / tau_or - 1))
            assert worst[0] <= 1e-4
            flipped = not cmp.selection(O.top_p(s, float(taus[b, h]), w.p, w.sparse_cap), w.p, kept)
        U.adopt_selection(un, kept)
        cmp.attention(o[b, h * w.group:(h + 1) * w.group], un.attend(qg), flipped=flipped)

    check_selection_units(w, st, dc, mask, q_ex, k_ex, v_ex, check)
    assert dc.read_status()[B.ST_FLAGS] == 0
    U.record("full_size_" + mode, workload=w.name, kept=int(dc.n_kept.sum()), worst_tau_rel=worst[0],
             topk_flipped_units=worst[1], tau_min=float(taus.min()), tau_max=float(taus.max()),
             **cmp.summary())
    print(mode, int(dc.n_kept.sum()), worst, cmp.summary())


def layout(mode, l_lower=0, l_upper=1 << 30, surcharge=0.5, reuse=-1):
    return B.LayoutPolicy(mode, reuse, l_lower, l_upper, surcharge)


@pytest.mark.parametrize("name", ["bf16_d128_g4", "f32_d64_g1", "bf16_g16", "batch5", "ring_wrap",
                                  "clamp"])
def test_sparse_loading_step_and_regularize(name):
    """Sparse Loading (sec. 2.C): the fused step and hardkv_regularize_policy write the
    same flattened index as the Rewrite Cache path but no compact rows, mark the units
    sp_mode = 0, and the attention (which then reads the kept rows from the ring through
    sp_idx) matches the oracle on the GPU's mask."""
    w = SMALL[name]
    st = synth.initial_state(w)
    dcr, dcl, dcu = (DecodeCache.from_state(st) for _ in range(3))
    (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dcr, w, st, 0)
    p = synth.p_values(w)[0]
    mask_r, out_r = U.run_fused_step(dcr, q, k, v, p)
    mask_l = dcl.new_mask()
    out_l = torch.empty_like(out_r)
    dcl.step(q, k, v, out_l, p, mask=mask_l, layout=layout(B.LAYOUT_SPARSE_LOAD))
    # separate calls: regularize with the Sparse Loading policy, then attention
    dcu.append(k, v)
    mask_u = dcu.new_mask()
    dcu.score_calibrate_topp(q, p, mask_u)
    dcu.regularize(mask_u, layout=layout(B.LAYOUT_SPARSE_LOAD))
    out_u = torch.empty_like(out_r)
    dcu.decode_attn(q, out_u)
    torch.cuda.synchronize()
    assert torch.equal(mask_r, mask_l) and torch.equal(mask_r, mask_u)
    for dc in (dcl, dcu):
        assert torch.equal(dc.sp_idx, dcr.sp_idx) and torch.equal(dc.n_kept, dcr.n_kept)
        assert int(dc.sp_mode.abs().sum()) == 0
        assert int(dc.k_sp.abs().sum()) == 0 and int(dc.v_sp.abs().sum()) == 0   # never written
    assert int(dcr.sp_mode.sum()) == w.units
    cmp = U.StepCompare(w.dtype)
    G = w.group
    ol, ou = out_l.cpu().numpy(), out_u.cpu().numpy()

    def check(b, h, un, qg, L, kept):
        U.adopt_selection(un, kept)
        ref = un.attend(qg)
        cmp.attention(ol[b, h * G:(h + 1) * G], ref)
        cmp.attention(ou[b, h * G:(h + 1) * G], ref)

    check_selection_units(w, st, dcl, mask_l, q_ex, k_ex, v_ex, check)
    U.record("sparse_load", name=name, **cmp.summary())


@pytest.mark.parametrize("select", ["all", "moved"])
@pytest.mark.parametrize("mode", [synth.MERGE, synth.EVICT])
def test_multistep_mti_policy(select, mode):
    """40 steps under the MTI policy (L_lower 96, L_upper 400, scattered-read surcharge
    0.5): each reselecting unit's layout is the oracle's mti_rewrite decision (select on
    move: 15 reuse steps, so budgets in [96, 400] and above are rewritten, smaller ones
    loaded in place; select every step: nothing to reuse, everything below L_upper is
    loaded in place); steps that do not reselect read each unit's rows from wherever its
    layout keeps them; attention per step against the oracle."""
    w = synth.small(condense_mode=mode, steps=40, batch=2, context=300, p=0.8,
                    temp_range=(0.3, 6.0))
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    units = {(b, h): oracle_unit_from_state(st, b, h, steps=w.steps) for b in range(w.batch)
             for h in range(w.n_kv_heads)}
    sel_mode = B.SELECT_ALL if select == "all" else B.SELECT_MOVED
    pol = layout(B.LAYOUT_MTI, l_lower=96, l_upper=400, surcharge=0.5)
    cmp = U.StepCompare(w.dtype)
    G = w.group
    diverged, decisions = set(), {True: 0, False: 0}
    for t in range(w.steps):
        (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, t)
        first = t == 0 and select == "moved"
        mask = dc.new_mask()
        out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
        dc.step(q, k, v, out, w.p, mask=mask, layout=pol,
                select_mode=B.SELECT_ALL if first else sel_mode)
        rs = "all" if first else select
        reuse = 0 if rs == "all" else w.block - 1
        torch.cuda.synchronize()
        m = mask.cpu().numpy().view(np.uint32)
        n_kept, sp_idx = dc.n_kept.cpu().numpy(), dc.sp_idx.cpu().numpy()
        sp_mode = dc.sp_mode.cpu().numpy()
        o = out.cpu().numpy()
        for (b, h), un in units.items():
            if (b, h) in diverged:
                continue
            res = un.step(q_ex[b, h * G:(h + 1) * G], k_ex[b, h], v_ex[b, h], 1.0, w.p, reselect=rs)
            if res.merge is not None and res.merge.gaps and min(res.merge.gaps) <= U.MERGE_TIE:
                diverged.add((b, h))
                continue
            same, ref = True, res.out
            if res.sel is not None:
                L = un.d_lo - un.s_lo
                kept = U.mask_bits(m[b, h], L)
                same = cmp.selection(res.sel, w.p, kept)
                if not same:
                    U.adopt_selection(un, kept)
                    ref = un.attend(q_ex[b, h * G:(h + 1) * G])
                want = O.mti_rewrite(int(n_kept[b, h]), reuse, 96, 400, float(np.float32(0.5)))
                assert bool(sp_mode[b, h]) == want, (t, b, h, int(n_kept[b, h]))
                decisions[want] += 1
            assert n_kept[b, h] == un.n and np.array_equal(sp_idx[b, h], un.idx)
            cmp.attention(o[b, h * G:(h + 1) * G], ref, flipped=not same)
    assert dc.read_status()[B.ST_FLAGS] == 0
    if select == "moved":
        assert decisions[True] > 0 and decisions[False] > 0      # both layouts exercised
    U.record("multistep_mti", select=select, mode=mode, rewrite=decisions[True],
             load=decisions[False], **cmp.summary())


def test_bounded_wait_gives_up_and_reports():
    """The bounded mbarrier wait used by every pipeline: on a barrier nothing completes it
    gives up after its poll limit, sets HARDKV_DEV_WAIT_TIMEOUT and the kernel returns
    (the context stays usable: a step runs afterwards)."""
    lib = B.load()
    status = torch.zeros(B.STATUS_WORDS, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.hardkv_selftest_wait_timeout(status.data_ptr(), 4096, stream) == B.OK
    torch.cuda.synchronize()
    st = status.cpu().numpy().view(np.uint32)
    assert st[B.ST_FLAGS] & B.DEV_WAIT_TIMEOUT and st[7] == 4096
    assert lib.hardkv_selftest_wait_timeout(status.data_ptr(), 0, stream) == B.EINVAL
    w = synth.small(batch=1)
    st0 = synth.initial_state(w)
    dc = DecodeCache.from_state(st0)
    (q, k, v), _ = U.upload_step(dc, w, st0, 0)
    mask, out = U.run_fused_step(dc, q, k, v, w.p)
    torch.cuda.synchronize()
    assert dc.read_status()[B.ST_FLAGS] == 0 and torch.isfinite(out).all()


@pytest.mark.parametrize("p", [0.5, 0.95])
def test_long_rows_read_from_global(p):
    """Rows longer than the top-p kernel's shared-memory score cache (R > 40960): every
    pass reads the scores from global memory in batches and the mask words are staged
    for the index pass. One head of 45k candidates and one of 44k (ragged), through
    the mask-only entry and the fused step, against the oracle."""
    w = synth.small(batch=2, n_kv_heads=1, n_q_heads=4, context=None, len_range=(44000, 45500),
                    sparse_cap=48000, dense_window=64, condensed_slots=32, p=p, temp_range=(0.5, 3.0))
    st = synth.initial_state(w)
    assert st.R > 40960
    dc = DecodeCache.from_state(st)
    dc2 = DecodeCache.from_state(st)
    (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, 0)
    dc.append(k, v)
    mask = dc.new_mask()
    dc.score_calibrate_topp(q, p, mask)
    mask2, out2 = U.run_fused_step(dc2, q, k, v, p)
    torch.cuda.synchronize()
    assert torch.equal(mask, mask2)
    units = {(b, h): oracle_unit_from_state(st, b, h) for b in range(w.batch)
             for h in range(w.n_kv_heads)}
    cmp = U.StepCompare(w.dtype)
    compare_step(w, st, dc2, mask2, out2, units, q_ex, k_ex, v_ex, p, cmp)
    assert dc2.read_status()[B.ST_FLAGS] == 0
    U.record("long_rows", p=p, **cmp.summary())
