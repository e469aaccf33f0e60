"""Device-resident cascade cache for one attention layer (torch owns the memory).

`DecodeCache` allocates the tensors the C ABI expects, uploads an initial state and
forwards each stage to libhardkv.so through `binding`. It only marshals arguments:
every stage of the decode step runs in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import binding as B


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class DecodeCache:
    """Cascade cache (Dense / Sparse / Condensed tiers) of B sequences x H KV heads."""

    def __init__(self, *, batch, n_q_heads, n_kv_heads, head_dim, block, dense_window,
                 condensed_slots, n_sink, sparse_cap, ring_rows, dtype, condense_mode,
                 device="cuda", pool_blocks=None):
        """pool_blocks: None keeps Cap compact rows per head (contiguous tier); an integer
        gives the paged tier, one pool of that many PAGE_ROWS-row blocks shared by all heads."""
        self.lib = B.load()
        self.desc = B.Desc(batch, n_q_heads, n_kv_heads, head_dim, block, dense_window,
                           condensed_slots, n_sink, sparse_cap, ring_rows,
                           B.BF16 if dtype == "bf16" else B.F32, condense_mode)
        B.check("hardkv_validate", self.lib.hardkv_validate(ctypes.byref(self.desc)))
        self.dtype = dtype
        self.tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.device = torch.device(device)
        Bn, H, d, R, C, cap = batch, n_kv_heads, head_dim, ring_rows, condensed_slots, sparse_cap
        dev, td = self.device, self.tdtype
        self.k_ring = torch.zeros(Bn, H, R, d, dtype=td, device=dev)
        self.v_ring = torch.zeros(Bn, H, R, d, dtype=td, device=dev)
        self.len = torch.zeros(Bn, dtype=torch.int32, device=dev)
        self.d_lo = torch.zeros(Bn, dtype=torch.int32, device=dev)
        self.s_lo = torch.zeros(Bn, dtype=torch.int32, device=dev)
        self.moved = torch.zeros(Bn, dtype=torch.int32, device=dev)
        self.pool_blocks = pool_blocks
        if pool_blocks is None:
            self.k_sp = torch.zeros(Bn, H, cap, d, dtype=td, device=dev)
            self.v_sp = torch.zeros(Bn, H, cap, d, dtype=td, device=dev)
            self.k_pool = self.v_pool = self.blk_tab = self.blk_cnt = None
            self.free_list = self.ret_list = self.pool_ctl = None
        else:
            nb = int(pool_blocks)
            tab = -(-cap // B.PAGE_ROWS)
            self.k_sp = self.v_sp = None
            self.k_pool = torch.zeros(nb, B.PAGE_ROWS, d, dtype=td, device=dev)
            self.v_pool = torch.zeros(nb, B.PAGE_ROWS, d, dtype=td, device=dev)
            self.blk_tab = torch.full((Bn, H, tab), -1, dtype=torch.int32, device=dev)
            self.blk_cnt = torch.zeros(Bn, H, dtype=torch.int32, device=dev)
            self.free_list = torch.arange(nb, dtype=torch.int32, device=dev)
            self.ret_list = torch.zeros(nb, dtype=torch.int32, device=dev)
            self.pool_ctl = torch.tensor([nb, 0, 0, 0], dtype=torch.int32, device=dev)
        self.sp_idx = torch.full((Bn, H, cap), -1, dtype=torch.int32, device=dev)
        self.n_kept = torch.zeros(Bn, H, dtype=torch.int32, device=dev)
        self.sp_mode = torch.zeros(Bn, H, dtype=torch.int32, device=dev)
        self.k_cd = torch.zeros(Bn, H, C, d, dtype=td, device=dev)
        self.v_cd = torch.zeros(Bn, H, C, d, dtype=td, device=dev)
        self.w_cd = torch.zeros(Bn, H, C, dtype=torch.float32, device=dev)
        self.status = torch.zeros(B.STATUS_WORDS, dtype=torch.int32, device=dev)
        ws_bytes = self.lib.hardkv_workspace_bytes(ctypes.byref(self.desc))
        self.ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
        self.mask_words = self.lib.hardkv_mask_words(ctypes.byref(self.desc))
        self.cstruct = B.Cache(*[_ptr(t) for t in (
            self.k_ring, self.v_ring, self.len, self.d_lo, self.s_lo, self.moved, self.k_sp,
            self.v_sp, self.sp_idx, self.n_kept, self.sp_mode, self.k_cd, self.v_cd, self.w_cd,
            self.status, self.k_pool, self.v_pool, self.blk_tab, self.blk_cnt, self.free_list,
            self.ret_list, self.pool_ctl)], 0 if pool_blocks is None else int(pool_blocks))

    # ------------------------------------------------------------------ state
    @classmethod
    def from_state(cls, st, device="cuda", pool_blocks=None) -> "DecodeCache":
        """Upload a synth.InitialState."""
        w = st.w
        self = cls(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block=w.block, dense_window=w.dense_window,
                   condensed_slots=w.condensed_slots, n_sink=w.n_sink, sparse_cap=w.sparse_cap,
                   ring_rows=st.R, dtype=w.dtype, condense_mode=w.condense_mode, device=device,
                   pool_blocks=pool_blocks)
        self.load_arrays(st.k_ring, st.v_ring, st.k_cd, st.v_cd, st.w_cd, st.len0, st.d_lo0,
                         st.s_lo0)
        return self

    def to_dev(self, a: np.ndarray) -> torch.Tensor:
        """Host storage array (uint16 bf16 bits or float32) -> device tensor of the cache dtype."""
        t = torch.from_numpy(np.ascontiguousarray(a))
        if self.dtype == "bf16":
            t = t.view(torch.bfloat16)
        return t.to(self.device, non_blocking=False)

    def load_arrays(self, k_ring, v_ring, k_cd, v_cd, w_cd, len0, d_lo0, s_lo0):
        self.k_ring.copy_(self.to_dev(k_ring))
        self.v_ring.copy_(self.to_dev(v_ring))
        self.k_cd.copy_(self.to_dev(k_cd))
        self.v_cd.copy_(self.to_dev(v_cd))
        self.w_cd.copy_(torch.from_numpy(np.ascontiguousarray(w_cd, np.float32)))
        self.set_bounds(len0, d_lo0, s_lo0)

    def set_bounds(self, len0, d_lo0, s_lo0):
        self.len.copy_(torch.from_numpy(np.asarray(len0, np.int32)))
        self.d_lo.copy_(torch.from_numpy(np.asarray(d_lo0, np.int32)))
        self.s_lo.copy_(torch.from_numpy(np.asarray(s_lo0, np.int32)))
        self.moved.zero_()

    def snapshot_bounds(self):
        return tuple(t.clone() for t in (self.len, self.d_lo, self.s_lo, self.moved))

    def restore_bounds(self, snap):
        for t, s in zip((self.len, self.d_lo, self.s_lo, self.moved), snap):
            t.copy_(s)

    def new_mask(self) -> torch.Tensor:
        d = self.desc
        return torch.zeros(d.batch, d.n_kv_heads, self.mask_words, dtype=torch.int32,
                           device=self.device)

    # ------------------------------------------------------------------ stages
    def _c(self, name, *args):
        return B.call(name, ctypes.byref(self.desc), ctypes.byref(self.cstruct), *args)

    def append(self, k_new, v_new, stream=None):
        self._c("hardkv_append", _ptr(k_new), _ptr(v_new), _ptr(self.ws), _stream(stream))

    def condense(self, stream=None):
        self._c("hardkv_condense", _ptr(self.ws), _stream(stream))

    def score_calibrate_topp(self, q, p, mask, tau=None, select_mode=B.SELECT_ALL, stream=None):
        self._c("hardkv_score_calibrate_topp", _ptr(q), _ptr(tau), ctypes.c_float(p),
                select_mode, _ptr(mask), _ptr(self.ws), _stream(stream))

    def score_calibrate_entropy_topp(self, q, p, mask, tau_out=None, select_mode=B.SELECT_ALL,
                                     stream=None):
        self._c("hardkv_score_calibrate_entropy_topp", _ptr(q), ctypes.c_float(p), select_mode,
                _ptr(mask), _ptr(tau_out), _ptr(self.ws), _stream(stream))

    def score_topk(self, q, k, mask, select_mode=B.SELECT_ALL, stream=None):
        self._c("hardkv_score_topk", _ptr(q), int(k), select_mode, _ptr(mask), _ptr(self.ws),
                _stream(stream))

    def regularize(self, mask, select_mode=B.SELECT_ALL, stream=None, layout=None):
        if layout is None:
            self._c("hardkv_regularize", _ptr(mask), select_mode, _ptr(self.ws), _stream(stream))
        else:
            self._c("hardkv_regularize_policy", _ptr(mask), select_mode, ctypes.byref(layout),
                    _ptr(self.ws), _stream(stream))

    def select_from_scores(self, scores, p, mask, tau=None, rule=B.RULE_TOPP, top_k=0,
                           select_mode=B.SELECT_ALL, stream=None):
        """Calibrated top-p (or top-k) on caller importance scores [B,H,R] (float32)."""
        self._c("hardkv_select_from_scores", _ptr(scores), _ptr(tau), ctypes.c_float(p), rule, top_k,
                select_mode, _ptr(mask), _ptr(self.ws), _stream(stream))

    def flatten_sum(self, offsets=None, flat=None, stream=None):
        """Sum form of the flattened index: (offsets [B*H+1], flat [B*H*Cap]) int32;
        flat[offsets[u]:offsets[u+1]] is unit u's kept positions."""
        d = self.desc
        U = d.batch * d.n_kv_heads
        if offsets is None:
            offsets = torch.empty(U + 1, dtype=torch.int32, device=self.device)
        if flat is None:
            flat = torch.empty(U * d.sparse_cap, dtype=torch.int32, device=self.device)
        self._c("hardkv_flatten_sum", _ptr(offsets), _ptr(flat), _stream(stream))
        return offsets, flat

    def decode_attn(self, q, out, stream=None):
        self._c("hardkv_decode_attn", _ptr(q), _ptr(out), _ptr(self.ws), _stream(stream))

    def step_args(self, q, k_new, v_new, out, p, tau=None, mask=None,
                  select_mode=B.SELECT_ALL, events=None, rule=B.RULE_TOPP, top_k=0,
                  calibration=B.CAL_TAU, tau_out=None, layout=None) -> B.StepArgs:
        ev = None
        if events is not None:
            self._ev_arr = (ctypes.c_void_p * B.STEP_EVENTS)(
                *[e.cuda_event if e is not None else None for e in events])
            ev = ctypes.cast(self._ev_arr, ctypes.c_void_p)
        self._layout = layout          # kept alive while the call reads it
        return B.StepArgs(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(tau), ctypes.c_float(p),
                          select_mode, _ptr(mask), _ptr(out), ev, rule, int(top_k), calibration,
                          _ptr(tau_out), ctypes.pointer(layout) if layout is not None else None)

    def step(self, q, k_new, v_new, out, p, tau=None, mask=None, select_mode=B.SELECT_ALL,
             events=None, stream=None, **sel):
        """One fused decode step through hardkv_decode_step (device tensors); `sel` may
        set rule / top_k / calibration / tau_out (hardkv_step_args)."""
        args = self.step_args(q, k_new, v_new, out, p, tau, mask, select_mode, events, **sel)
        self._c("hardkv_decode_step", ctypes.byref(args), _ptr(self.ws), _stream(stream))

    def step_host(self, q, k_new, v_new, out, p, tau=None, mask=None, select_mode=B.SELECT_ALL,
                  stream=None, **sel):
        """hardkv_decode_step_host: q/k_new/v_new/tau/out are (pinned) host tensors."""
        args = self.step_args(q, k_new, v_new, out, p, tau, mask, select_mode, **sel)
        self._c("hardkv_decode_step_host", ctypes.byref(args), _ptr(self.ws), _stream(stream))

    def read_status(self) -> np.ndarray:
        return self.status.cpu().numpy().view(np.uint32)
