"""The bounds-checked build (libhardkv_checked.so, -DHARDKV_CHECKED) in place of a
memory sanitizer: every checked index of the kernels (ring, compact and pool rows,
Condensed slots, score, mask, index and flat-list slots, pool bookkeeping) is tested
before its access, and a failure sets HARDKV_DEV_CHECK and skips the access.

The same workloads (tests/checked_cases.py: MERGE with the MTI layout and reselection
on move, fp32, the paged tier with an ample and a short pool, top-k on ragged lengths,
entropy calibration, rows longer than the top-p cache, llama8b_8k at full size, and
the standalone entry points) run once on the checked build in a subprocess and once
on the normal build here: no check may fire, and every result must be identical."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from attention_kv_head_b200 import binding as B
from attention_kv_head_b200 import build as Bd

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_checked_build_agrees_and_no_check_fires(tmp_path):
    Bd.build()
    assert os.path.exists(Bd.LIB_CHECKED)
    checked = tmp_path / "checked.npz"
    env = dict(os.environ, HARDKV_CHECKED="1")
    r = subprocess.run([sys.executable, "-m", "tests.checked_cases", str(checked)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    from tests import checked_cases
    normal = tmp_path / "normal.npz"
    checked_cases.run_cases(str(normal))
    a, b = np.load(checked), np.load(normal)
    assert sorted(a.files) == sorted(b.files)
    for key in a.files:
        if key.endswith("/status"):
            sa, sb = a[key].view(np.uint32), b[key].view(np.uint32)
            assert not sa[B.ST_FLAGS] & B.DEV_CHECK, key        # no index out of range
            assert np.array_equal(sa, sb), (key, sa, sb)        # same flags and counters
        else:
            assert np.array_equal(a[key], b[key]), key          # bit-identical results


def test_checked_build_catches_a_table_entry_past_the_pool():
    """The checked build turns a block-table entry past the pool into HARDKV_DEV_CHECK
    (the reads it would cause are skipped). Runs only in a subprocess on the checked
    build: the normal build trusts the caller's table."""
    Bd.build()
    env = dict(os.environ, HARDKV_CHECKED="1")
    r = subprocess.run([sys.executable, "-m", "tests.checked_cases", "--corrupted-table"], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    flags = int(r.stdout.split("FLAGS")[-1].split()[0])
    assert flags & B.DEV_CHECK, flags
