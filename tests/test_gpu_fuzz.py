"""Seeded random configurations of the decode step against the oracle.

Each case draws the shapes (dtype, head_dim, KV heads, GQA group 1-16, batch, Dense
window, block, Condensed slots, sinks, Sparse capacity, fixed or ragged lengths), the
selection rule (calibrated top-p at p from 0.5 to 1, or fixed top-k), the calibration
of top-p (tau = 1, caller temperatures on both sides of 1, or the entropy-matched
temperature), the layout (Rewrite Cache, Sparse Loading, or the MTI rule with random
thresholds), the compact tier (contiguous or a paged pool), the condense mode, the
reselection cadence and the entry points (the fused step, or in a quarter of the cases
its standalone calls: append, condense, selection, regularization under the layout
policy, attention; some fused cases through the host-buffer entry point, pinned or
pageable), and runs several steps with the oracle following every unit.
Under the entropy-matched calibration the oracle selects at the GPU's temperature, and
that temperature must match the oracle's own solve within 1e-4 (relative). Bars as in
the other parity tests: boundaries, kept counts and indices bit-exact (on the GPU's
accepted mask), masks within the near-threshold rule (top-k: within the score rounding
of the k-th score), the layout decision equal to the oracle's MTI rule, attention
within the dtype's tolerance, Condensed state bit-exact except after merge near-ties,
the pool a partition of its blocks.
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

N_CASES = 256


def draw(seed: int):
    r = np.random.RandomState(1000 + seed)
    # a second stream for the calibration and the wide groups, so the draws from `r`
    # stay what they were before those were added
    r2 = np.random.RandomState(5000 + seed)
    cal_pick = ["tau1", "tau", "entropy"][r2.choice(3, p=[0.4, 0.3, 0.3])]
    wide = r2.rand() < 0.12   # G = 12 or 16: two query tiles of 8 in the kernels
    G_wide = int([12, 16][r2.randint(2)])
    # the fused step, or the same step as its standalone calls (append, condense,
    # selection, regularization with the layout policy, attention)
    path = "unfused" if r2.rand() < 0.25 else "fused"
    # some fused cases through the host-buffer entry point, pinned or pageable
    if r2.rand() < 0.2 and path == "fused":
        path = "host_pinned" if r2.rand() < 0.5 else "host_pageable"
    dtype = [synth.BF16, synth.F32][r.randint(2)]
    d = [64, 128][r.randint(2)]
    H = int(r.randint(1, 4))
    G = int([1, 2, 4, 5, 8][r.randint(5)])
    if wide:
        G = G_wide
    Bn = int(r.randint(1, 5))
    W = int([16, 32, 48, 64][r.randint(4)])
    blk = int([8, 16][r.randint(2)])
    C = int([8, 24, 64][r.randint(3)])
    sinks = int(r.randint(0, min(4, C) + 1))
    base = C + W
    if r.rand() < 0.5:
        ctx = dict(context=int(base + r.randint(0, 700)), len_range=None)
    else:
        lo = int(base + r.randint(0, 200))
        ctx = dict(context=None, len_range=(lo, int(lo + r.randint(1, 600))))
    cap = int(r.randint(16, 900))
    w = synth.small(f"fuzz{seed}", dtype=dtype, head_dim=d, n_kv_heads=H, n_q_heads=H * G,
                    batch=Bn, dense_window=W, block=blk, condensed_slots=C, n_sink=sinks,
                    sparse_cap=cap, p=float([0.5, 0.8, 0.9, 0.99, 1.0][r.randint(5)]),
                    condense_mode=[synth.EVICT, synth.MERGE][r.randint(2)],
                    steps=int(r.randint(4, 2 * blk + 3)), temp_range=(0.3, 6.0), seed=seed, **ctx)
    rule = "topk" if r.rand() < 0.3 else "topp"
    k = int(r.randint(1, cap + 1))
    layout = ["rewrite", "sparse", "mti"][r.randint(3)]
    lo = int(r.randint(0, 200))
    mti = (lo, int(lo + r.randint(0, 400)), float(np.float32(r.choice([0.05, 0.5, 2.0]))))
    select = ["all", "moved"][r.randint(2)]
    paged = bool(r.rand() < 0.5)
    cal = "tau1" if rule == "topk" else cal_pick
    return w, rule, k, layout, mti, select, paged, cal, path


def pool_partition(dc: DecodeCache):
    ctl = dc.pool_ctl.cpu().numpy()
    free, ret = max(int(ctl[B.POOL_FREE]), 0), int(ctl[B.POOL_RETURNED])
    tab, cnt = dc.blk_tab.cpu().numpy(), dc.blk_cnt.cpu().numpy()
    parts = [tab[b, h, :cnt[b, h]] for b in range(tab.shape[0]) for h in range(tab.shape[1])]
    parts += [dc.free_list[:free].cpu().numpy(), dc.ret_list[:ret].cpu().numpy()]
    assert np.array_equal(np.sort(np.concatenate(parts)), np.arange(dc.pool_blocks))


@pytest.mark.parametrize("seed", range(N_CASES))
def test_random_configuration(seed):
    w, rule, k, layout, (l_lo, l_hi, surcharge), select, paged, cal, path = draw(seed)
    st = synth.initial_state(w)
    pool = w.batch * w.n_kv_heads * (-(-w.sparse_cap // B.PAGE_ROWS)) if paged else None
    dc = DecodeCache.from_state(st, pool_blocks=pool)
    units = {(b, h): U.oracle_unit_from_state(st, b, h, steps=w.steps) for b in range(w.batch)
             for h in range(w.n_kv_heads)}
    mode = {"rewrite": B.LAYOUT_REWRITE, "sparse": B.LAYOUT_SPARSE_LOAD, "mti": B.LAYOUT_MTI}[layout]
    pol = B.LayoutPolicy(mode, -1, l_lo, l_hi, surcharge)
    sel_kw = dict(rule=B.RULE_TOPK, top_k=min(k, w.sparse_cap)) if rule == "topk" else {}
    tau_np = synth.calibration_taus(w) if cal == "tau" else None
    tau_dev = None if tau_np is None else torch.from_numpy(tau_np).to(dc.device)
    tau_out = None
    if cal == "entropy":
        tau_out = torch.zeros(w.batch, w.n_kv_heads, dtype=torch.float32, device=dc.device)
        sel_kw = dict(calibration=B.CAL_ENTROPY, tau_out=tau_out)
    worst_tau = 0.0
    cmp = U.StepCompare(w.dtype)
    G = w.group
    diverged = set()
    for t in range(w.steps):
        (q, kn, vn), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, t)
        rs = "all" if (t == 0 or select == "all") else "moved"
        mask = dc.new_mask()
        out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
        smode = B.SELECT_ALL if rs == "all" else B.SELECT_MOVED
        if path == "fused":
            dc.step(q, kn, vn, out, w.p, tau=tau_dev, mask=mask, layout=pol, select_mode=smode,
                    **sel_kw)
        elif path.startswith("host"):
            host = [t_.cpu() for t_ in (q, kn, vn)] + [torch.full(out.shape, float("nan"))]
            if path == "host_pinned":
                host = [t_.pin_memory() for t_ in host]
            qh, kh, vh, out = host
            dc.step_host(qh, kh, vh, out, w.p, tau=None if tau_np is None else torch.from_numpy(tau_np),
                         mask=mask, layout=pol, select_mode=smode, **sel_kw)
        else:
            dc.append(kn, vn)
            dc.condense()
            if rule == "topk":
                dc.score_topk(q, min(k, w.sparse_cap), mask, select_mode=smode)
            elif cal == "entropy":
                dc.score_calibrate_entropy_topp(q, w.p, mask, tau_out=tau_out, select_mode=smode)
            else:
                dc.score_calibrate_topp(q, w.p, mask, tau=tau_dev, select_mode=smode)
            dc.regularize(mask, select_mode=smode, layout=pol)
            dc.decode_attn(q, out)
        torch.cuda.synchronize()
        taus = None if tau_out is None else tau_out.cpu().numpy()
        m = mask.cpu().numpy().view(np.uint32)
        n_kept, sp_idx, sp_mode = (dc.n_kept.cpu().numpy(), dc.sp_idx.cpu().numpy(),
                                   dc.sp_mode.cpu().numpy())
        k_cd, v_cd, w_cd = U.device_rows(dc.k_cd), U.device_rows(dc.v_cd), dc.w_cd.cpu().numpy()
        bounds = [t_.cpu().numpy() for t_ in (dc.len, dc.d_lo, dc.s_lo)]
        o = out.cpu().numpy()
        for (b, h), un in units.items():
            if (b, h) in diverged:
                continue
            qg = q_ex[b, h * G:(h + 1) * G]
            tau_u = float(taus[b, h]) if taus is not None else U.tau_of(tau_np, b, h)
            res = un.step(qg, k_ex[b, h], v_ex[b, h], tau_u, w.p, reselect=rs, rule=rule,
                          k=min(k, w.sparse_cap))
            if cal == "entropy" and res.sel is not None and un.d_lo - un.s_lo > 1:
                Ks = un.K[un.s_lo:un.d_lo]
                tau_or = O.entropy_matched_tau(O.score(qg, Ks), O.attention_entropy(qg, Ks))
                worst_tau = max(worst_tau, abs(tau_u / tau_or - 1.0))
                assert worst_tau <= 1e-4, (seed, t, b, h, tau_u, tau_or)
            assert (bounds[0][b], bounds[1][b], bounds[2][b]) == (un.len, un.d_lo, un.s_lo)
            if res.merge is not None and res.merge.gaps and min(res.merge.gaps) <= U.MERGE_TIE:
                diverged.add((b, h))
                continue
            assert np.array_equal(w_cd[b, h], un.cd_w.astype(np.float32))
            assert np.array_equal(k_cd[b, h], un.cd_k) and np.array_equal(v_cd[b, h], un.cd_v)
            same, ref = True, res.out
            if res.sel is not None:
                L = un.d_lo - un.s_lo
                kept = U.mask_bits(m[b, h], L)
                if rule == "topk":
                    ok, nd = O.allowed_flips_topk(un.scores, res.sel, kept,
                                                  2e-5 * max(1.0, float(np.abs(un.scores).max())
                                                             if un.scores.size else 1.0))
                    assert ok, (seed, t, b, h, nd)
                    same = nd == 0
                else:
                    same = cmp.selection(res.sel, w.p, kept)
                if not same:
                    U.adopt_selection(un, kept)
                    ref = un.attend(qg)
                n = int(n_kept[b, h])
                if layout == "rewrite":
                    assert sp_mode[b, h] == 1
                elif layout == "sparse":
                    assert sp_mode[b, h] == 0
                else:
                    reuse = 0 if rs == "all" else w.block - 1
                    assert bool(sp_mode[b, h]) == O.mti_rewrite(n, reuse, l_lo, l_hi, surcharge), \
                        (seed, t, b, h, n)
            assert n_kept[b, h] == un.n and np.array_equal(sp_idx[b, h], un.idx), (seed, t, b, h)
            cmp.attention(o[b, h * G:(h + 1) * G], ref, flipped=not same)
        if paged:
            pool_partition(dc)
    assert dc.read_status()[B.ST_FLAGS] == 0
    assert len(diverged) <= max(1, len(units) // 4)
    U.record("fuzz", seed=seed, path=path, rule=rule, calibration=cal, layout=layout, select=select,
             paged=paged, dtype=w.dtype, units=len(units), steps=w.steps, diverged=len(diverged),
             worst_tau_rel=worst_tau, **cmp.summary())
