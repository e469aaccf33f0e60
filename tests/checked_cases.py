"""Workloads run by both the normal and the bounds-checked library (tests/test_gpu_checked.py).

`run_cases(path)` runs every case with whatever library `binding.load()` gives this
process and saves, per case, every step's output, mask, kept counts, indices and the
final status words to one .npz file. Importable; also runnable as
`python -m tests.checked_cases OUT.npz` (the checked build is selected by the
HARDKV_CHECKED=1 environment variable before the library is loaded).
"""
import sys

import numpy as np
import torch

from attention_kv_head_b200 import binding as B
from attention_kv_head_b200 import synth
from attention_kv_head_b200.cache import DecodeCache


def _tab(w):
    return w.batch * w.n_kv_heads * (-(-w.sparse_cap // B.PAGE_ROWS))


def cases():
    mti = B.LayoutPolicy(B.LAYOUT_MTI, -1, 96, 400, 0.5)
    small = synth.small(condense_mode=synth.MERGE, steps=20, batch=3, context=300, p=0.8,
                        temp_range=(0.3, 6.0))
    f32 = synth.small(dtype=synth.F32, n_q_heads=4, n_kv_heads=2, head_dim=64, steps=8)
    ragged = synth.small(batch=5, context=None, len_range=(150, 700), sparse_cap=120, steps=8)
    long_rows = synth.small(batch=2, n_kv_heads=1, n_q_heads=4, context=None,
                            len_range=(44000, 45500), sparse_cap=48000, dense_window=64,
                            condensed_slots=32, steps=2)
    big = synth.WORKLOADS["llama8b_8k"].with_(steps=1)
    return [
        ("merge_mti_moved", small, dict(layout=mti), None, "moved"),
        ("f32_d64", f32, {}, None, "all"),
        ("paged_mti", small, dict(layout=mti), _tab(small), "moved"),
        ("paged_short", small, {}, _tab(small) // 4, "all"),
        ("topk_ragged", ragged, dict(rule=B.RULE_TOPK, top_k=60), None, "all"),
        ("entropy", f32, dict(calibration=B.CAL_ENTROPY), None, "all"),
        ("long_rows", long_rows, {}, None, "all"),
        ("llama8b_8k", big, {}, None, "all"),
    ]


def run_cases(path):
    res = {}
    for name, w, kw, pool, select in cases():
        st = synth.initial_state(w)
        dc = DecodeCache.from_state(st, pool_blocks=pool)
        outs, masks, kept, idx = [], [], [], []
        for t in range(w.steps):
            qr, _ = synth.queries(w, t)
            kr, _, vr, _ = synth.step_kv(w, st.lens, t)
            q, k, v = dc.to_dev(qr), dc.to_dev(kr), dc.to_dev(vr)
            mask = dc.new_mask()
            out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
            mode = B.SELECT_MOVED if (select == "moved" and t > 0) else B.SELECT_ALL
            dc.step(q, k, v, out, synth.p_values(w)[0], mask=mask, select_mode=mode, **kw)
            torch.cuda.synchronize()
            outs.append(out.cpu().numpy())
            masks.append(mask.cpu().numpy())
            kept.append(dc.n_kept.cpu().numpy())
            idx.append(dc.sp_idx.cpu().numpy())
        # the standalone calls too: selection on the library's scores, regularization
        # from the mask, attention, and the sum form of the index
        q = dc.to_dev(synth.queries(w, w.steps)[0])
        mask = dc.new_mask()
        dc.score_calibrate_topp(q, synth.p_values(w)[0], mask)
        dc.regularize(mask)
        out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
        dc.decode_attn(q, out)
        offsets, flat = dc.flatten_sum()
        torch.cuda.synchronize()
        n_total = int(offsets[-1].item())
        res[name + "/out"] = np.stack(outs)
        res[name + "/mask"] = np.stack(masks)
        res[name + "/kept"] = np.stack(kept)
        res[name + "/idx"] = np.stack(idx)
        res[name + "/standalone_out"] = out.cpu().numpy()
        res[name + "/offsets"] = offsets.cpu().numpy()
        res[name + "/flat"] = flat[:n_total].cpu().numpy()
        res[name + "/status"] = dc.read_status()
    np.savez(path, **res)


def run_corrupted_table():
    """CHECKED BUILD ONLY (its bounds checks are what make this input safe): a paged cache
    after one valid step, then one head's first block-table entry pointed past the pool,
    then a standalone attention. Every read of that head's compact rows is checked
    against the pool size, so the rows are skipped and HARDKV_DEV_CHECK is set. Returns
    the status flags."""
    assert B.LIB_PATH.endswith("libhardkv_checked.so"), "only for the checked build"
    w = synth.small(batch=2, context=300, p=0.9)
    st = synth.initial_state(w)
    dc = DecodeCache.from_state(st, pool_blocks=_tab(w))
    qr, _ = synth.queries(w, 0)
    kr, _, vr, _ = synth.step_kv(w, st.lens, 0)
    q, k, v = dc.to_dev(qr), dc.to_dev(kr), dc.to_dev(vr)
    out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float32, device=dc.device)
    dc.step(q, k, v, out, w.p, mask=dc.new_mask())
    torch.cuda.synchronize()
    assert dc.read_status()[B.ST_FLAGS] == 0 and int(dc.blk_cnt[0, 0].item()) > 0
    dc.blk_tab[0, 0, 0] = dc.pool_blocks + 1000   # past the pool
    dc.decode_attn(q, out)
    torch.cuda.synchronize()
    return int(dc.read_status()[B.ST_FLAGS])


if __name__ == "__main__":
    if sys.argv[1] == "--corrupted-table":
        print("FLAGS", run_corrupted_table())
    else:
        run_cases(sys.argv[1])
