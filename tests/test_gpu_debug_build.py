"""libgqa_debug.so: the library with device-side index checks compiled in.

Every index a kernel derives before it reads or writes (a cache row, a
partial-record slot, a head, a weight row) is checked against its buffer in
that build; a failed check skips the access and sets GQA_ERR_INDEX in the
status word, and nothing traps.  The tests run a cross-section of the parity
suite against the debug build in a child process (the binding picks the
library at import from GQA_LIB); every test there reads the status word, so
any check that fires fails it.  A second test shows that a check does fire:
a hook of the debug build declares one partial record fewer than a call over
full-length sequences writes, so the last record's write is skipped (it would
still have been inside the workspace) and the status reports GQA_ERR_INDEX; the release
build ignores the hook.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SUBSET = [
    "tests/test_gpu_decode.py::test_bf16_group_sizes",
    "tests/test_gpu_decode.py::test_f32_sweep",
    "tests/test_gpu_decode.py::test_forced_split_counts",
    "tests/test_gpu_decode.py::test_seqlens_out_of_range_are_clamped_and_flagged",
    "tests/test_gpu_decode.py::test_llama2_7b_decode_full",
    "tests/test_gpu_decode_tc.py",
    "tests/test_gpu_prefill.py::test_prefill_small",
    "tests/test_gpu_prefill.py::test_prefill_group_sizes_and_head_dims",
    "tests/test_gpu_window.py::test_decode_window",
    "tests/test_gpu_window.py::test_prefill_window",
    "tests/test_gpu_meanpool.py",
    "tests/test_gpu_qkv.py",
    "tests/test_gpu_layer.py::test_layer_decode_step_small",
]


def _child(args, extra_env, timeout=900):
    env = dict(os.environ)
    env["GQA_LIB"] = "debug"
    env.update(extra_env)
    return subprocess.run([sys.executable, *args], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


def test_parity_subset_passes_with_index_checks():
    r = _child(["-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu", *SUBSET], {})
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


PROBE = r"""
import os, torch
import kv_cache_decode_04_b200 as gqa
import gqa_inputs as gi
assert os.path.basename(gqa.LIB_PATH) == os.environ["EXPECT_LIB"], gqa.LIB_PATH
torch.cuda.set_device(0)
x = gi.decode_inputs(4, 16, 4, 128, 300, torch.bfloat16, seed=5)
out = gqa.decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(), x.scale)
try:
    gqa.get_status()
    print("STATUS OK")
except gqa.GQAError as e:
    print("STATUS", e.code)
"""


def test_index_check_fires_and_is_reported():
    hook = {"GQA_DEBUG_DECLARE_FEWER_RECORDS": "1"}
    r = _child(["-c", PROBE], dict(hook, EXPECT_LIB="libgqa_debug.so"), timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "STATUS -8" in r.stdout, r.stdout
    env = dict(hook, EXPECT_LIB="libgqa.so", GQA_LIB="release")
    r = _child(["-c", PROBE], env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "STATUS OK" in r.stdout, r.stdout
