"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and the fp64
oracle on the same seeded inputs, and compare them."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from attention_kv_head_b200 import binding as B
from attention_kv_head_b200 import synth
from attention_kv_head_b200.cache import DecodeCache
from oracle import hardkv_oracle as O

# bf16 attention tolerance: max-abs 1e-2 and rel-L2 2e-3 (fixed by the target bounds);
# fp32 inputs: the same arithmetic with fp32 storage -> 1e-4 / 1e-5.
TOL = {"bf16": (1e-2, 2e-3), "f32": (1e-4, 1e-5)}

# Merge slot choices: the kernel ranks cosines in fp32; for d = 128 the error of an
# fp32 cosine is below d * 2^-24 ~ 7.6e-6, so a slot decision may legitimately differ
# from the fp64 oracle only where the oracle's top-1/top-2 gap is under 1e-5. Such a
# unit is followed no further (its Condensed state may then differ by design).
MERGE_TIE = 1e-5


def record(kind: str, **fields) -> None:
    """Append one JSON record of parity counts (flips, clamps, near-ties) to the file
    named by HARDKV_PARITY_RECORD, if that variable is set."""
    path = os.environ.get("HARDKV_PARITY_RECORD")
    if not path:
        return
    fields["kind"] = kind
    with open(path, "a") as f:
        f.write(json.dumps(fields, default=lambda x: x.item() if hasattr(x, "item") else str(x)) + "\n")


def oracle_params(w: synth.Workload) -> O.Params:
    return O.Params(w.head_dim, w.group, w.dense_window, w.condensed_slots, w.block,
                    w.sparse_cap, w.n_sink, w.dtype, w.condense_mode)


def oracle_unit(w: synth.Workload, st: synth.InitialState, b: int, h: int, steps: int = 1):
    L0 = int(st.len0[b])
    _, ke, _, ve = synth.unit_kv(w, b, h, 0, L0)
    C = w.condensed_slots
    return O.Unit(oracle_params(w), ke, ve, ke[:C], ve[:C], np.ones(C), L0, int(st.d_lo0[b]),
                  int(st.s_lo0[b]), L0 + steps + 1)


def oracle_unit_from_state(st: synth.InitialState, b: int, h: int, steps: int = 1):
    """Oracle unit built from the very host arrays uploaded to the GPU."""
    w = st.w
    C, R = w.condensed_slots, st.R
    L0 = int(st.len0[b])
    K = np.zeros((L0, w.head_dim))
    V = np.zeros((L0, w.head_dim))
    K[:C] = storage_exact(st.k_cd[b, h], w.dtype)
    V[:C] = storage_exact(st.v_cd[b, h], w.dtype)
    pos = np.arange(C, L0)
    K[C:] = storage_exact(st.k_ring[b, h, pos % R], w.dtype)
    V[C:] = storage_exact(st.v_ring[b, h, pos % R], w.dtype)
    return O.Unit(oracle_params(w), K, V, K[:C], V[:C], st.w_cd[b, h].astype(np.float64), L0,
                  int(st.d_lo0[b]), int(st.s_lo0[b]), L0 + steps + 1)


def mask_bits(mask_words_row: np.ndarray, L: int) -> np.ndarray:
    """Local indices j < L whose bit is set in one unit's mask words."""
    words = mask_words_row.astype(np.uint32)
    bits = ((words[:, None] >> np.arange(32, dtype=np.uint32)[None, :]) & 1).reshape(-1)
    return np.nonzero(bits[:L])[0]


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def upload_step(dc: DecodeCache, w: synth.Workload, st: synth.InitialState, t: int):
    qraw, qex = synth.queries(w, t)
    kr, ke, vr, ve = synth.step_kv(w, st.lens, t)
    return (dc.to_dev(qraw), dc.to_dev(kr), dc.to_dev(vr)), (qex, ke, ve)


def storage_exact(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return synth.bf16_bits_to_f64(a)
    return a.astype(np.float64)


def device_rows(t: torch.Tensor) -> np.ndarray:
    """Device tensor of the cache dtype -> exact float64 numpy."""
    return t.float().cpu().numpy().astype(np.float64)


class StepCompare:
    """Accumulates the comparison of one step (or run) over units."""

    def __init__(self, dtype):
        self.atol, self.rtol = TOL[dtype]
        self.flipped_units = 0
        self.flipped_tokens = 0
        self.selections = 0
        self.clamps = 0
        self.units = 0
        self.flipped_attended = 0
        self.worst_abs = 0.0
        self.worst_rel = 0.0

    def selection(self, sel: O.Selection, p: float, gpu_kept: np.ndarray):
        """The GPU's kept set must equal the oracle's up to the near-threshold flip rule;
        returns True when they are identical."""
        ok, nd = O.allowed_flips(sel, p, gpu_kept)
        assert ok, f"mask differs beyond the flip rule ({nd} tokens)"
        self.selections += 1
        self.clamps += int(sel.clamped)
        if nd:
            self.flipped_units += 1
            self.flipped_tokens += nd
        return nd == 0

    def attention(self, gpu: np.ndarray, ref: np.ndarray, flipped: bool = False):
        self.units += 1
        self.flipped_attended += int(flipped)
        a = float(np.abs(gpu - ref).max())
        r = rel_l2(gpu, ref)
        self.worst_abs = max(self.worst_abs, a)
        self.worst_rel = max(self.worst_rel, r)
        assert a <= self.atol and r <= self.rtol, (a, r)

    def summary(self) -> dict:
        return dict(selections=self.selections, flipped_units=self.flipped_units,
                    flipped_tokens=self.flipped_tokens, clamps=self.clamps,
                    attention_units=self.units, attention_units_flipped=self.flipped_attended,
                    worst_abs=self.worst_abs, worst_rel_l2=self.worst_rel)


def adopt_selection(un: O.Unit, kept_local: np.ndarray) -> None:
    """Make the oracle unit's Sparse set the given kept candidates (local indices, as
    read from a GPU mask that O.allowed_flips accepted): the attention of a step whose
    selection flipped a near-threshold token is evaluated on the GPU's mask, and a unit
    that keeps its set across steps (select on move) carries that set on. Rows, order
    and index come from the oracle's own arrays and O.regularize."""
    L = un.d_lo - un.s_lo
    mask = np.zeros(L, bool)
    mask[np.asarray(kept_local, np.int64)] = True
    pos = np.arange(un.s_lo, un.d_lo)
    un.n, un.idx, un.sp_k, un.sp_v = O.regularize(
        mask, pos, un.K[un.s_lo:un.d_lo], un.V[un.s_lo:un.d_lo], un.prm.sparse_cap)


def tau_of(tau, b: int, h: int) -> float:
    """Calibration temperature of unit (b, h): 1 when no array is given."""
    return 1.0 if tau is None else float(tau[b, h])


def run_unfused_step(dc: DecodeCache, q, k, v, p, select_mode=B.SELECT_ALL, tau=None):
    dc.append(k, v)
    dc.condense()
    mask = dc.new_mask()
    dc.score_calibrate_topp(q, p, mask, tau=tau, select_mode=select_mode)
    dc.regularize(mask, select_mode=select_mode)
    d = dc.desc
    out = torch.empty(d.batch, d.n_q_heads, d.head_dim, dtype=torch.float32, device=dc.device)
    dc.decode_attn(q, out)
    return mask, out


def run_fused_step(dc: DecodeCache, q, k, v, p, select_mode=B.SELECT_ALL, tau=None):
    mask = dc.new_mask()
    d = dc.desc
    out = torch.empty(d.batch, d.n_q_heads, d.head_dim, dtype=torch.float32, device=dc.device)
    dc.step(q, k, v, out, p, tau=tau, mask=mask, select_mode=select_mode)
    return mask, out


def scores_from_ws(dc: DecodeCache) -> np.ndarray:
    """The workspace starts with the fp32 score array [B*H, R] (white-box check)."""
    d = dc.desc
    n = d.batch * d.n_kv_heads * d.ring_rows
    return dc.ws[: n * 4].view(torch.float32).cpu().numpy().reshape(d.batch * d.n_kv_heads,
                                                                     d.ring_rows)
