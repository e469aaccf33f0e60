"""The allocation-free entry point hardkv_score_calibrate_topp_static, called through
the C ABI, gives the same selection masks as hardkv_score_calibrate_topp with a
caller workspace, on two calls in a row with different queries (its built-in scratch
keeps the previous call's contents, which must not leak into the next result).

It exists for callers that cannot allocate device memory for a workspace (a plugin
whose host framework owns all device memory, code running under a stream capture that
forbids allocation). This file is collected last so a stop-at-first-failure run has
already run every other test; it builds its own state, so it also passes alone."""
import ctypes

import pytest
import torch

from attention_kv_head_b200 import binding as B
from attention_kv_head_b200 import synth
from attention_kv_head_b200.cache import DecodeCache
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def static_call(dc, q, p, mask, select_mode=B.SELECT_ALL):
    lib = B.load()
    return lib.hardkv_score_calibrate_topp_static(
        ctypes.byref(dc.desc), ctypes.byref(dc.cstruct), q.data_ptr(), None, ctypes.c_float(p),
        select_mode, mask.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name", ["bf16", "f32"])
def test_static_scratch_matches_workspace_entry_on_two_calls(name):
    w = synth.small(batch=3) if name == "bf16" else synth.small(dtype=synth.F32, batch=2)
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st)
    for t in (0, 1):
        (q, k, v), _ = U.upload_step(dc, w, st, t)
        dc.append(k, v)
        m_static = dc.new_mask()
        assert static_call(dc, q, w.p, m_static) == B.OK
        m_ws = dc.new_mask()
        dc.score_calibrate_topp(q, w.p, m_ws)
        torch.cuda.synchronize()
        assert torch.equal(m_static, m_ws), f"call {t}"
        assert int(m_static.count_nonzero()) > 0


def test_static_scratch_rejects_problems_beyond_its_size():
    lib = B.load()
    limit = lib.hardkv_static_scratch_bytes()
    assert limit == 32 << 20
    w = synth.WORKLOADS["stress64k"]   # 16 x 8 x 64576 fp32 scores > 32 MiB
    d = B.Desc(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.dense_window,
               w.condensed_slots, w.n_sink, w.sparse_cap, w.derived_ring_rows(), B.BF16,
               w.condense_mode)
    fake = B.Cache(*[0x10000 * (i + 1) for i in range(len(B.Cache._fields_))])
    rc = lib.hardkv_score_calibrate_topp_static(ctypes.byref(d), ctypes.byref(fake), 0x100, None,
                                                ctypes.c_float(0.9), 0, 0x200, None)
    assert rc == B.ESCRATCH
    assert "scratch" in B.strerror(rc)
