"""Selection on importance scores the caller supplies (hardkv_select_from_scores): the
calibrated top-p and the fixed top-k of HARD-KV sec. 2.B / 2.A Tier 2 applied to any
metric. The metric here is the group-MEAN logit (instead of the max-pooled one), made
by the test in fp64 from the exact stored keys and rounded to fp32; the same fp32
values go to the GPU and, widened, to the oracle's top_p / top_k.

Bars: top-p masks within the near-threshold flip rule; top-k bit-exact (both sides
rank the same fp32 values, ties to the lower position); entries past each head's
candidates are NaN and must not matter; the library's own scores through this entry
give the same mask as hardkv_score_calibrate_topp.
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

CASES = {
    "bf16_g4": synth.small(temp_range=(0.3, 6.0)),
    "f32_d64_g2": synth.small(dtype=synth.F32, n_q_heads=4, n_kv_heads=2, head_dim=64),
    "ragged_clamp": synth.small(batch=5, context=None, len_range=(150, 700), sparse_cap=120),
}


def mean_logit_scores(w, st, q_ex):
    """[B,H,R] float32: candidate j of (b,h) = mean_g q_g . k_{s_lo+j} / sqrt(d); NaN
    elsewhere. Also the oracle units (their K rows are the exact stored keys)."""
    G = w.group
    sc = np.full((w.batch, w.n_kv_heads, st.R), np.nan, np.float32)
    units = {}
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            un = U.oracle_unit_from_state(st, b, h)
            kk = un.K[un.s_lo:un.d_lo]
            logits = q_ex[b, h * G:(h + 1) * G] @ kk.T / np.sqrt(w.head_dim)
            sc[b, h, :kk.shape[0]] = logits.mean(axis=0).astype(np.float32)
            units[(b, h)] = un
    return sc, units


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("with_tau", [False, True], ids=["tau1", "tau"])
def test_topp_on_supplied_scores(name, with_tau):
    w = CASES[name]
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    _, q_ex = synth.queries(w, 0)
    sc, units = mean_logit_scores(w, st, q_ex)
    tau_np = synth.calibration_taus(w) if with_tau else None
    tau = torch.from_numpy(tau_np).to(dc.device) if with_tau else None
    mask = dc.new_mask()
    dc.select_from_scores(torch.from_numpy(sc).to(dc.device), w.p, mask, tau=tau)
    torch.cuda.synchronize()
    m = mask.cpu().numpy().view(np.uint32)
    cmp = U.StepCompare(w.dtype)
    for (b, h), un in units.items():
        L = un.d_lo - un.s_lo
        sel = O.top_p(sc[b, h, :L].astype(np.float64), U.tau_of(tau_np, b, h), w.p, w.sparse_cap)
        cmp.selection(sel, w.p, U.mask_bits(m[b, h], L))
    assert dc.read_status()[B.ST_FLAGS] == 0
    U.record("supplied_scores_topp", name=name, tau=with_tau, **cmp.summary())


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("kfrac", [0.0, 0.3, 1.0])
def test_topk_on_supplied_scores(name, kfrac):
    w = CASES[name]
    k_sel = max(1, int(round(kfrac * w.sparse_cap)))
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    _, q_ex = synth.queries(w, 0)
    sc, units = mean_logit_scores(w, st, q_ex)
    mask = dc.new_mask()
    dc.select_from_scores(torch.from_numpy(sc).to(dc.device), 0.0, mask, rule=B.RULE_TOPK,
                          top_k=k_sel)
    torch.cuda.synchronize()
    m = mask.cpu().numpy().view(np.uint32)
    for (b, h), un in units.items():
        L = un.d_lo - un.s_lo
        sel = O.top_k(sc[b, h, :L].astype(np.float64), k_sel)
        assert np.array_equal(U.mask_bits(m[b, h], L), np.sort(sel.kept)), (name, b, h)


def test_own_scores_through_the_hook_match_the_fused_selection():
    """The library's max-pooled scores, read back from the workspace and passed in again,
    select exactly what hardkv_score_calibrate_topp selected (same kernel, same masses;
    the maximum now comes from the scores instead of the tile maxima, the same value)."""
    w = CASES["bf16_g4"]
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    (q, _, _), _ = U.upload_step(dc, w, st, 0)
    mask = dc.new_mask()
    dc.score_calibrate_topp(q, w.p, mask)
    torch.cuda.synchronize()
    own = U.scores_from_ws(dc)
    mask2 = dc.new_mask()
    dc.select_from_scores(torch.from_numpy(np.ascontiguousarray(own)).to(dc.device), w.p, mask2)
    torch.cuda.synchronize()
    assert torch.equal(mask, mask2)
