"""Paged compact tier (head-wise block manager, HARD-KV technical summary sec. 2.C,
"Metadati"): one pool of 16-row blocks shared by all heads, per-head block tables.

Bars: with a pool large enough, every observable of the paged cache (step outputs,
masks, kept counts, compact indices, layouts, compact rows read through the block
tables) is bit-identical to the contiguous cache on the same inputs, and the pool is a
partition of its blocks after every launch. With a pool too small, the flag is raised,
each short head keeps the position-order prefix its blocks hold, and its attention
matches the oracle evaluated on that truncated selection.
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

PR = B.PAGE_ROWS


def layout(mode, l_lower=0, l_upper=1 << 30, surcharge=0.5, reuse=-1):
    return B.LayoutPolicy(mode, reuse, l_lower, l_upper, surcharge)


def tab_blocks(w) -> int:
    return -(-w.sparse_cap // PR)


def pool_state(dc: DecodeCache):
    """Host copy of the pool bookkeeping; asserts that held, free and returned blocks
    partition the pool (every block exactly once)."""
    nb = dc.pool_blocks
    ctl = dc.pool_ctl.cpu().numpy()
    free, ret = max(int(ctl[B.POOL_FREE]), 0), int(ctl[B.POOL_RETURNED])
    tab = dc.blk_tab.cpu().numpy()
    cnt = dc.blk_cnt.cpu().numpy()
    assert 0 <= free <= nb and 0 <= ret <= nb
    parts = [tab[b, h, :cnt[b, h]] for b in range(tab.shape[0]) for h in range(tab.shape[1])]
    parts += [dc.free_list[:free].cpu().numpy(), dc.ret_list[:ret].cpu().numpy()]
    every = np.sort(np.concatenate(parts))
    assert np.array_equal(every, np.arange(nb)), "pool blocks lost or held twice"
    return tab, cnt


def paged_rows(dc: DecodeCache, tab_row: np.ndarray, n: int):
    """Compact slots 0..n-1 of one head, read through its block table."""
    j = torch.arange(n, device=dc.device)
    blk = torch.from_numpy(tab_row.astype(np.int64)).to(dc.device)[j // PR]
    return dc.k_pool[blk, j % PR], dc.v_pool[blk, j % PR]


def assert_same_compact(dc0: DecodeCache, dc1: DecodeCache, need_exact_blocks=True):
    """Index, counts, layouts and rewritten rows of the contiguous (dc0) and paged (dc1)
    caches agree bit for bit."""
    n0, n1 = dc0.n_kept.cpu().numpy(), dc1.n_kept.cpu().numpy()
    assert np.array_equal(n0, n1)
    assert torch.equal(dc0.sp_idx, dc1.sp_idx)
    assert torch.equal(dc0.sp_mode, dc1.sp_mode)
    tab, cnt = pool_state(dc1)
    mode = dc1.sp_mode.cpu().numpy()
    for b in range(n0.shape[0]):
        for h in range(n0.shape[1]):
            n = int(n1[b, h])
            if need_exact_blocks:
                assert cnt[b, h] == (-(-n // PR) if mode[b, h] else 0), (b, h, n, cnt[b, h])
            if mode[b, h] and n:
                k1, v1 = paged_rows(dc1, tab[b, h], n)
                assert torch.equal(k1, dc0.k_sp[b, h, :n]) and torch.equal(v1, dc0.v_sp[b, h, :n])


WORKLOADS = {
    "bf16": dict(),
    "f32_d64": dict(dtype=synth.F32, n_q_heads=2, n_kv_heads=2, head_dim=64),
}


@pytest.mark.parametrize("wname", list(WORKLOADS))
@pytest.mark.parametrize("policy", ["rewrite", "mti"])
@pytest.mark.parametrize("select", ["all", "moved"])
def test_paged_steps_match_contiguous(wname, policy, select):
    """40 fused steps on a contiguous and on a paged cache (pool of B*H*ceil(Cap/16)
    blocks, enough for every head): identical outputs, masks, indices, layouts and
    compact rows; each head holds exactly ceil(n/16) blocks when rewritten, none when
    loaded in place; the pool stays a partition."""
    w = synth.small(condense_mode=synth.MERGE, steps=40, batch=2, context=300, p=0.8,
                    temp_range=(0.3, 6.0), **WORKLOADS[wname])
    st = synth.initial_state(w)
    dc0 = DecodeCache.from_state(st)
    nb = w.batch * w.n_kv_heads * tab_blocks(w)
    dc1 = DecodeCache.from_state(st, pool_blocks=nb)
    pol = layout(B.LAYOUT_MTI, l_lower=96, l_upper=400) if policy == "mti" else None
    sel_mode = B.SELECT_ALL if select == "all" else B.SELECT_MOVED
    modes_seen = set()
    for t in range(w.steps):
        (q, k, v), _ = U.upload_step(dc0, w, st, t)
        sm = B.SELECT_ALL if (t == 0 and select == "moved") else sel_mode
        outs, masks = [], []
        for dc in (dc0, dc1):
            mask = dc.new_mask()
            out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32,
                              device=dc.device)
            dc.step(q, k, v, out, w.p, mask=mask, layout=pol, select_mode=sm)
            outs.append(out)
            masks.append(mask)
        torch.cuda.synchronize()
        assert torch.equal(masks[0], masks[1]), t
        assert torch.equal(outs[0], outs[1]), t
        assert_same_compact(dc0, dc1)
        modes_seen.update(np.unique(dc1.sp_mode.cpu().numpy()).tolist())
    assert dc0.read_status()[B.ST_FLAGS] == 0 and dc1.read_status()[B.ST_FLAGS] == 0
    if policy == "mti" and select == "moved":
        assert modes_seen == {0, 1}  # both layouts went through the pool
    U.record("paged_vs_contiguous", workload=wname, policy=policy, select=select, steps=w.steps)


def test_paged_regularize_given_masks():
    """Standalone regularization on the paged tier (merge, allocation and compaction
    launches) from masks of decreasing and increasing size: heads return blocks and take
    them back across calls, with the same index, rows and attention as the contiguous
    cache and the pool a partition after every call."""
    w = synth.small(batch=2, context=600, sparse_cap=600, temp_range=(0.3, 6.0))
    st = synth.initial_state(w)
    dc0 = DecodeCache.from_state(st)
    nb = w.batch * w.n_kv_heads * tab_blocks(w)
    dc1 = DecodeCache.from_state(st, pool_blocks=nb)
    (q, _, _), _ = U.upload_step(dc0, w, st, 0)
    for p in (0.95, 0.3, 1.0, 0.6):
        mask = dc0.new_mask()
        dc0.score_calibrate_topp(q, p, mask)
        outs = []
        for dc in (dc0, dc1):
            dc.regularize(mask)
            out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32,
                              device=dc.device)
            dc.decode_attn(q, out)
            outs.append(out)
        torch.cuda.synchronize()
        assert_same_compact(dc0, dc1)
        assert torch.equal(outs[0], outs[1]), p
    assert dc1.read_status()[B.ST_FLAGS] == 0


def test_paged_pool_shortage_keeps_prefix():
    """A pool of a quarter of what every head would need: the shortage flag is raised,
    each head keeps the first rows (in position order) that its blocks hold, the pool
    stays a partition, heads that were short get blocks back as others return them, and
    every head's attention matches the oracle on the selection it actually kept."""
    w = synth.small(condense_mode=synth.EVICT, steps=8, batch=2, context=500, sparse_cap=500,
                    p=0.95, temp_range=(0.3, 6.0))
    st = synth.initial_state(w)
    nb = w.batch * w.n_kv_heads * tab_blocks(w) // 4
    dc = DecodeCache.from_state(st, pool_blocks=nb)
    units = {(b, h): U.oracle_unit_from_state(st, b, h, steps=w.steps) for b in range(w.batch)
             for h in range(w.n_kv_heads)}
    cmp = U.StepCompare(w.dtype)
    G = w.group
    short_units = 0
    for t in range(w.steps):
        (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, t)
        mask = dc.new_mask()
        out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
        dc.step(q, k, v, out, w.p, mask=mask)
        torch.cuda.synchronize()
        tab, cnt = pool_state(dc)
        m = mask.cpu().numpy().view(np.uint32)
        n_kept, sp_idx = dc.n_kept.cpu().numpy(), dc.sp_idx.cpu().numpy()
        o = out.cpu().numpy()
        for (b, h), un in units.items():
            res = un.step(q_ex[b, h * G:(h + 1) * G], k_ex[b, h], v_ex[b, h], 1.0, w.p,
                          reselect="all")
            L = un.d_lo - un.s_lo
            kept = U.mask_bits(m[b, h], L)
            cmp.selection(res.sel, w.p, kept)
            n_sel = min(len(kept), w.sparse_cap)
            n = int(n_kept[b, h])
            assert cnt[b, h] <= -(-n_sel // PR)
            assert n == min(n_sel, int(cnt[b, h]) * PR), (t, b, h)
            assert np.array_equal(sp_idx[b, h, :n], un.s_lo + kept[:n])
            assert (sp_idx[b, h, n:] == -1).all()
            short_units += n < n_sel
            U.adopt_selection(un, kept[:n])
            ref = un.attend(q_ex[b, h * G:(h + 1) * G])
            cmp.attention(o[b, h * G:(h + 1) * G], ref, flipped=True)
    assert short_units > 0
    assert dc.read_status()[B.ST_FLAGS] & B.DEV_POOL_SHORT
    U.record("paged_shortage", short_units=short_units, **cmp.summary())


@pytest.mark.parametrize("paged", [False, True], ids=["contiguous", "paged"])
@pytest.mark.parametrize("name", ["bf16_ragged", "clamp", "f32_d64"])
def test_flatten_sum_matches_oracle(name, paged):
    """The sum form of the flattened index (offsets + flat list) against the oracle's
    flatten_sum of the oracle units' own indices: before any selection (every count 0),
    then after each of 6 steps under the MTI policy with reselection on block moves
    (heads rewritten and heads loaded in place alike)."""
    kw = {"bf16_ragged": dict(batch=5, context=None, len_range=(200, 700)),
          "clamp": dict(sparse_cap=100),
          "f32_d64": dict(dtype=synth.F32, n_q_heads=2, n_kv_heads=2, head_dim=64)}[name]
    w = synth.small(steps=6, temp_range=(0.3, 6.0), **kw)
    st = synth.initial_state(w)
    pool = w.batch * w.n_kv_heads * tab_blocks(w) if paged else None
    dc = DecodeCache.from_state(st, pool_blocks=pool)
    units = [U.oracle_unit_from_state(st, b, h, steps=w.steps) for b in range(w.batch)
             for h in range(w.n_kv_heads)]
    cmp = U.StepCompare(w.dtype)
    G, H = w.group, w.n_kv_heads
    pol = layout(B.LAYOUT_MTI, l_lower=64, l_upper=300)
    for t in range(-1, w.steps):
        if t >= 0:
            (q, k, v), (q_ex, k_ex, v_ex) = U.upload_step(dc, w, st, t)
            mask = dc.new_mask()
            out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32,
                              device=dc.device)
            sm = B.SELECT_ALL if t == 0 else B.SELECT_MOVED
            dc.step(q, k, v, out, w.p, mask=mask, layout=pol, select_mode=sm)
            torch.cuda.synchronize()
            m = mask.cpu().numpy().view(np.uint32)
            for u, un in enumerate(units):
                b, h = divmod(u, H)
                res = un.step(q_ex[b, h * G:(h + 1) * G], k_ex[b, h], v_ex[b, h], 1.0, w.p,
                              reselect="all" if t == 0 else "moved")
                if res.sel is not None:
                    kept = U.mask_bits(m[b, h], un.d_lo - un.s_lo)
                    if not cmp.selection(res.sel, w.p, kept):
                        U.adopt_selection(un, kept)
        offsets, flat = dc.flatten_sum()
        torch.cuda.synchronize()
        want_off, want_flat = O.flatten_sum([un.idx[:un.n] for un in units])
        got_off = offsets.cpu().numpy()
        assert np.array_equal(got_off, want_off), t
        assert np.array_equal(flat[:int(want_off[-1])].cpu().numpy(), want_flat), t
    assert dc.read_status()[B.ST_FLAGS] == 0
    U.record("flatten_sum", workload=name, paged=paged, **cmp.summary())


def test_full_size_paged_step_and_sum_form():
    """llama8b_8k at full size (64 heads, 7680 candidates each): one fused step on a
    paged and on a contiguous cache gives bit-identical outputs, masks, indices and
    compact rows, the pool is a partition, and the sum form of the flattened index holds
    at any size: offsets are the running kept counts and each head's slice of the flat
    list is its max-length row up to n_kept."""
    w = synth.WORKLOADS["llama8b_8k"]
    st = synth.initial_state(w)
    dc0 = DecodeCache.from_state(st)
    dc1 = DecodeCache.from_state(st, pool_blocks=w.batch * w.n_kv_heads * tab_blocks(w))
    (q, k, v), _ = U.upload_step(dc0, w, st, 0)
    outs, masks = [], []
    for dc in (dc0, dc1):
        mask = dc.new_mask()
        out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
        dc.step(q, k, v, out, w.p, mask=mask)
        outs.append(out)
        masks.append(mask)
    torch.cuda.synchronize()
    assert torch.equal(masks[0], masks[1]) and torch.equal(outs[0], outs[1])
    assert_same_compact(dc0, dc1)
    for dc in (dc0, dc1):
        offsets, flat = dc.flatten_sum()
        torch.cuda.synchronize()
        n = dc.n_kept.cpu().numpy().reshape(-1).astype(np.int64)
        off = offsets.cpu().numpy()
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(n)]))
        idx = dc.sp_idx.cpu().numpy().reshape(n.size, -1)
        fl = flat.cpu().numpy()
        for u in range(n.size):
            assert np.array_equal(fl[off[u]:off[u + 1]], idx[u, :n[u]]), u
        assert dc.read_status()[B.ST_FLAGS] == 0


@pytest.mark.parametrize("sel", ["topk", "entropy"])
def test_paged_steps_other_rules(sel):
    """The block manager is independent of how the selection was made: 12 fused steps
    with the fixed top-k rule, and with the entropy-matched temperature, bit-identical on
    the paged and the contiguous cache."""
    w = synth.small(condense_mode=synth.MERGE, steps=12, batch=2, context=300, p=0.8,
                    temp_range=(0.3, 6.0))
    st = synth.initial_state(w)
    dc0 = DecodeCache.from_state(st)
    dc1 = DecodeCache.from_state(st, pool_blocks=w.batch * w.n_kv_heads * tab_blocks(w))
    kw = dict(rule=B.RULE_TOPK, top_k=90) if sel == "topk" else dict(calibration=B.CAL_ENTROPY)
    for t in range(w.steps):
        (q, k, v), _ = U.upload_step(dc0, w, st, t)
        outs, masks = [], []
        for dc in (dc0, dc1):
            mask = dc.new_mask()
            out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32,
                              device=dc.device)
            dc.step(q, k, v, out, w.p, mask=mask, **kw)
            outs.append(out)
            masks.append(mask)
        torch.cuda.synchronize()
        assert torch.equal(masks[0], masks[1]) and torch.equal(outs[0], outs[1]), t
        assert_same_compact(dc0, dc1)
    assert dc1.read_status()[B.ST_FLAGS] == 0
