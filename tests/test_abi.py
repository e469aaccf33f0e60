"""The C-ABI library loads and exports every symbol include/hardkv.h declares, and its
host-side validation returns the documented codes without touching a GPU."""
import ctypes
import subprocess

import pytest

from attention_kv_head_b200 import binding as B
from attention_kv_head_b200 import build as Bd


@pytest.fixture(scope="module")
def lib():
    Bd.build()
    return B.load()


def desc(**kw):
    base = dict(batch=8, n_q_heads=32, n_kv_heads=8, head_dim=128, block=16, dense_window=200,
                condensed_slots=256, n_sink=4, sparse_cap=7680, ring_rows=8000, dtype=B.BF16,
                condense_mode=B.EVICT)
    base.update(kw)
    return B.Desc(**base)


def test_every_declared_function_is_exported(lib):
    names = B.header_functions()
    assert len(names) >= 11
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)


def test_hot_path_entry_points_declared():
    for n in ("hardkv_append", "hardkv_score_calibrate_topp", "hardkv_regularize",
              "hardkv_condense", "hardkv_decode_attn"):
        assert n in B.header_functions()


@pytest.mark.parametrize("field,value,code", [
    ("dtype", 7, B.EDTYPE), ("batch", 0, B.EINVAL), ("n_q_heads", 12, B.EINVAL),
    ("n_q_heads", 8 * 17, B.EINVAL), ("head_dim", 96, B.EINVAL), ("block", 0, B.EINVAL),
    ("condensed_slots", 0, B.EINVAL), ("n_sink", 300, B.EINVAL), ("sparse_cap", 0, B.ECAP),
    ("ring_rows", 8001, B.ECAP), ("ring_rows", 192, B.ECAP), ("dense_window", 7990, B.ECAP), ("condense_mode", 3, B.EINVAL),
    ("ring_rows", (1 << 18) + 64, B.EINVAL),   # per-bin partial mass sums are 32-bit
])
def test_validate_rejects(lib, field, value, code):
    d = desc(**{field: value})
    assert lib.hardkv_validate(ctypes.byref(d)) == code
    assert lib.hardkv_workspace_bytes(ctypes.byref(d)) == 0


def test_ring_rows_limit_inclusive(lib):
    assert lib.hardkv_validate(ctypes.byref(desc(ring_rows=1 << 18))) == B.OK


def test_validate_accepts_all_workloads(lib):
    from attention_kv_head_b200 import synth
    for w in synth.WORKLOADS.values():
        d = B.Desc(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.dense_window,
                   w.condensed_slots, w.n_sink, w.sparse_cap, w.derived_ring_rows(),
                   B.BF16 if w.dtype == "bf16" else B.F32, w.condense_mode)
        assert lib.hardkv_validate(ctypes.byref(d)) == B.OK, w.name
        ws = lib.hardkv_workspace_bytes(ctypes.byref(d))
        assert 0 < ws < 2 ** 31
        assert lib.hardkv_mask_words(ctypes.byref(d)) * 32 >= d.ring_rows


def test_merge_slot_limit(lib):
    assert lib.hardkv_validate(ctypes.byref(desc(condense_mode=B.MERGE, condensed_slots=2048))) == B.OK
    assert lib.hardkv_validate(ctypes.byref(desc(condense_mode=B.MERGE, condensed_slots=4096))) == B.EINVAL


POOL_FIELDS = ("k_pool", "v_pool", "blk_tab", "blk_cnt", "free_list", "ret_list", "pool_ctl")


def _fake_cache(misalign=None, null=None, paged=False):
    vals = {}
    for i, (name, _) in enumerate(B.Cache._fields_):
        vals[name] = 0x10000 * (i + 1)
    if not paged:  # contiguous compact tier: the pool fields stay NULL
        for name in POOL_FIELDS:
            vals[name] = None
        vals["pool_blocks"] = 0
    else:
        vals["pool_blocks"] = 4096
    if misalign:
        vals[misalign] += 4
    if null:
        vals[null] = None
    return B.Cache(**vals)


def test_entry_points_validate_before_any_launch(lib):
    """Bad arguments return their code with nothing enqueued (fake pointers are never
    dereferenced because validation fails first)."""
    d = desc()
    c = _fake_cache()
    ws = ctypes.c_void_p(0x7000000)
    assert lib.hardkv_append(ctypes.byref(d), None, 0x100, 0x200, ws, None) == B.EINVAL
    assert lib.hardkv_append(ctypes.byref(d), ctypes.byref(_fake_cache(null="len")), 0x100, 0x200,
                             ws, None) == B.EINVAL
    assert lib.hardkv_append(ctypes.byref(d), ctypes.byref(_fake_cache(misalign="k_sp")), 0x100,
                             0x200, ws, None) == B.EALIGN
    assert lib.hardkv_append(ctypes.byref(d), ctypes.byref(c), 0x104, 0x200, ws, None) == B.EALIGN
    for p in (0.0, -0.5, 1.5, float("nan")):
        assert lib.hardkv_score_calibrate_topp(ctypes.byref(d), ctypes.byref(c), 0x100, None,
                                               ctypes.c_float(p), 0, 0x300, ws, None) == B.EINVAL
    assert lib.hardkv_score_calibrate_topp(ctypes.byref(d), ctypes.byref(c), 0x100, None,
                                           ctypes.c_float(0.9), 5, 0x300, ws, None) == B.EINVAL
    assert lib.hardkv_regularize(ctypes.byref(d), ctypes.byref(c), None, 0, ws, None) == B.EINVAL
    assert lib.hardkv_decode_attn(ctypes.byref(d), ctypes.byref(c), 0x100, None, ws, None) == B.EINVAL
    sel = lib.hardkv_select_from_scores
    assert sel(ctypes.byref(d), ctypes.byref(c), None, None, ctypes.c_float(0.9), B.RULE_TOPP, 0, 0,
               0x300, ws, None) == B.EINVAL                      # no scores
    assert sel(ctypes.byref(d), ctypes.byref(c), 0x104, None, ctypes.c_float(0.9), B.RULE_TOPP, 0, 0,
               0x300, ws, None) == B.EALIGN                      # misaligned scores
    assert sel(ctypes.byref(d), ctypes.byref(c), 0x100, 0x204, ctypes.c_float(0.9), B.RULE_TOPP, 0, 0,
               0x300, ws, None) == B.EALIGN                      # misaligned tau
    assert sel(ctypes.byref(d), ctypes.byref(c), 0x100, None, ctypes.c_float(0.0), B.RULE_TOPP, 0, 0,
               0x300, ws, None) == B.EINVAL                      # p out of range
    assert sel(ctypes.byref(d), ctypes.byref(c), 0x100, None, ctypes.c_float(0.9), B.RULE_TOPK, 0, 0,
               0x300, ws, None) == B.EINVAL                      # k out of range
    assert sel(ctypes.byref(d), ctypes.byref(c), 0x100, None, ctypes.c_float(0.9), 7, 1, 0,
               0x300, ws, None) == B.EINVAL                      # unknown rule
    assert sel(ctypes.byref(d), ctypes.byref(c), 0x100, None, ctypes.c_float(0.9), B.RULE_TOPP, 0, 3,
               0x300, ws, None) == B.EINVAL                      # unknown select mode
    assert lib.hardkv_flatten_sum(ctypes.byref(d), ctypes.byref(c), None, 0x200, None) == B.EINVAL
    assert lib.hardkv_flatten_sum(ctypes.byref(d), ctypes.byref(c), 0x100, 0x204, None) == B.EALIGN
    bad = desc(dtype=9)
    assert lib.hardkv_condense(ctypes.byref(bad), ctypes.byref(c), ws, None) == B.EDTYPE
    assert lib.hardkv_decode_step(ctypes.byref(d), ctypes.byref(c), None, ws, None) == B.EINVAL
    args = B.StepArgs(0x100, 0x200, 0x300, None, ctypes.c_float(2.0), 0, None, 0x400, None)
    assert lib.hardkv_decode_step(ctypes.byref(d), ctypes.byref(c), ctypes.byref(args), ws,
                                  None) == B.EINVAL
    assert lib.hardkv_decode_step_host(ctypes.byref(d), ctypes.byref(c), None, ws, None) == B.EINVAL


def test_paged_cache_validates(lib):
    """The paged compact tier: k_sp / v_sp may be NULL, every pool pointer is required and
    aligned, and the pool must be addressable by the 29-bit row codes."""
    d = desc()
    ws = ctypes.c_void_p(0x7000000)

    def append(c, k_new=0x100):
        return lib.hardkv_append(ctypes.byref(d), ctypes.byref(c), k_new, 0x200, ws, None)

    # a valid paged cache gets past the cache check: the misaligned k_new decides
    c = _fake_cache(paged=True)
    c.k_sp = c.v_sp = None
    assert append(c, k_new=0x104) == B.EALIGN
    assert append(_fake_cache(null="k_sp")) == B.EINVAL  # contiguous tier needs k_sp
    for name in POOL_FIELDS:
        assert append(_fake_cache(paged=True, null=name)) == B.EINVAL, name
        assert append(_fake_cache(paged=True, misalign=name)) == B.EALIGN, name
    for blocks in (0, -1, (1 << 29) // B.PAGE_ROWS, 1 << 62):
        c = _fake_cache(paged=True)
        c.pool_blocks = blocks
        assert append(c) == B.EINVAL, blocks
    c = _fake_cache(paged=True)
    c.pool_blocks = (1 << 29) // B.PAGE_ROWS - 1
    assert append(c, k_new=0x104) == B.EALIGN


def test_strerror(lib):
    for code in (B.OK, B.EINVAL, B.EALIGN, B.EDTYPE, B.ECAP, B.ECUDA, 12345):
        assert isinstance(B.strerror(code), str) and B.strerror(code)


def test_host_entry_validates_before_any_copy(lib):
    """hardkv_decode_step_host checks p, the select mode and the mask before its first
    copy: a bad argument returns its own code (on a machine without a GPU a copy would
    have failed with HARDKV_ECUDA instead)."""
    import numpy as np
    d = desc(batch=2, sparse_cap=100, ring_rows=1024, dense_window=64, condensed_slots=32)
    c = _fake_cache()
    ws = ctypes.c_void_p(0x7000000)
    q = np.zeros((2, 32, 128), np.uint16)
    kv = np.zeros((2, 8, 128), np.uint16)
    out = np.zeros((2, 32, 128), np.float32)
    tau = np.ones((2, 8), np.float32)

    def call(p=0.9, mode=0, mask=None, tau_ptr=None):
        a = B.StepArgs(q.ctypes.data, kv.ctypes.data, kv.ctypes.data, tau_ptr, ctypes.c_float(p),
                       mode, mask, out.ctypes.data, None)
        return lib.hardkv_decode_step_host(ctypes.byref(d), ctypes.byref(c), ctypes.byref(a), ws,
                                           None)

    for p in (0.0, 1.5, float("nan")):
        assert call(p=p) == B.EINVAL
        assert call(p=p, tau_ptr=tau.ctypes.data) == B.EINVAL
    assert call(mode=7) == B.EINVAL
    assert call(mask=0x1004) == B.EALIGN
    a = B.StepArgs(None, kv.ctypes.data, kv.ctypes.data, None, ctypes.c_float(0.9), 0, None,
                   out.ctypes.data, None)
    assert lib.hardkv_decode_step_host(ctypes.byref(d), ctypes.byref(c), ctypes.byref(a), ws,
                                       None) == B.EINVAL


def test_selection_rules_validate(lib):
    """Top-k wants 1 <= k <= Cap; the fused step's rule and calibration fields are checked."""
    d = desc()
    c = _fake_cache()
    ws = ctypes.c_void_p(0x7000000)
    for k in (0, -3, d.sparse_cap + 1):
        assert lib.hardkv_score_topk(ctypes.byref(d), ctypes.byref(c), 0x100, k, 0, 0x300, ws,
                                     None) == B.EINVAL
    assert lib.hardkv_score_topk(ctypes.byref(d), ctypes.byref(c), 0x100, 10, 9, 0x300, ws,
                                 None) == B.EINVAL
    assert lib.hardkv_score_calibrate_entropy_topp(ctypes.byref(d), ctypes.byref(c), 0x100,
                                                   ctypes.c_float(1.5), 0, 0x300, None, ws,
                                                   None) == B.EINVAL
    assert lib.hardkv_score_calibrate_entropy_topp(ctypes.byref(d), ctypes.byref(c), 0x100,
                                                   ctypes.c_float(0.9), 0, 0x300, 0x404, ws,
                                                   None) == B.EALIGN
    for rule, k, cal in ((2, 0, 0), (B.RULE_TOPK, 0, 0), (B.RULE_TOPK, d.sparse_cap + 1, 0),
                         (B.RULE_TOPP, 0, 5)):
        a = B.StepArgs(0x100, 0x200, 0x300, None, ctypes.c_float(0.9), 0, None, 0x400, None,
                       rule, k, cal, None)
        assert lib.hardkv_decode_step(ctypes.byref(d), ctypes.byref(c), ctypes.byref(a), ws,
                                      None) == B.EINVAL
