"""Canary guards and the bounds-checked build: stand-ins for a memory checker.

compute-sanitizer does not run on this pool, so two cheaper checks stand in
for it.  (1) Every part of a cache's single allocation is followed by a 4 KB
guard of 0xA5 bytes; after the whole path has run on assorted shapes every
guard must be intact, and a byte planted in a guard (inside the allocation,
by the test) must be reported with the part it follows.  (2) The
bounds-checked library (STAR_LIB=checked) checks every global index its
kernels compute for a store against its buffer and reports a bad one through
the error word; the parity suites of the small cases run on it in a child
process and must pass with the error word clear.
"""

import os
import subprocess
import sys

import pytest
import torch

from block_sparse_long_phase_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SHAPES = [
    dict(),
    dict(L=1000, b=256, b_a=100, lq=7, T=3),
    dict(L=301, b=2, b_a=1, lq=3, T=2),
    dict(B=2, Hq=16, Hkv=2, D=128, L=700, b=128, b_a=64, lq=9, T=2),
]


@pytest.mark.parametrize("kv_fp8", [False, True])
@pytest.mark.parametrize("i", range(len(SHAPES)))
def test_guards_stay_intact(i, kv_fp8):
    from block_sparse_long_phase_b200 import StarCache
    w = wl.get("tiny").with_(**SHAPES[i])
    x = {k: v.cuda() for k, v in wl.make_inputs(w, "cpu").items()}
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T + 1, w.scale, kv_fp8=kv_fp8)
    cache.star_ctx_encode_fp32(x["Qc"], x["Kc"], x["Vc"])
    cache.star_query_prefill_partials(x["Qq"], x["Kq"], x["Vq"])
    cache.reset_query()
    cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    for t in range(w.T):
        cache.star_decode_step_partials(x["qd"][t], x["kd"][t], x["vd"][t])
    cache.star_partial_attend(x["qd"][0], 0, cache.num_segments - 1, x["kd"][0], x["vd"][0])
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    assert cache.check_guards() == (-1, "")
    cache.close()


def test_a_planted_overwrite_is_reported():
    """A byte written just past the context K array (inside the allocation,
    in the guard that follows it) is reported as guard 0, after context K."""
    from block_sparse_long_phase_b200 import StarCache
    from block_sparse_long_phase_b200.api import _view_from_ptr
    w = wl.get("tiny")
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq, w.scale)
    assert cache.check_guards() == (-1, "")
    last = cache.segment(cache.num_segments - 2)
    end = last.k + w.B * w.Hkv * last.len * w.D * 2          # first byte past the context K array
    past = _view_from_ptr((end + 255) // 256 * 256 + 100, 1, "|u1", torch.device("cuda"))
    past.fill_(0)
    torch.cuda.synchronize()
    idx, what = cache.check_guards()
    assert idx == 0 and "context K" in what, (idx, what)
    cache.close()


def test_parity_suites_pass_on_the_bounds_checked_build():
    lib = os.path.join(ROOT, "block_sparse_long_phase_b200", "lib", "libstar_checked.so")
    assert os.path.exists(lib), "build the checked variant first (build(checked=True))"
    env = dict(os.environ, STAR_LIB="checked")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_parity.py::test_small_cases_every_element",
           "tests/test_gpu_short_blocks.py", "tests/test_gpu_fp8.py::test_fp8_small_cases",
           "tests/test_gpu_partials.py", "tests/test_gpu_sharded.py"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    # the child really ran on the checked library
    chk = subprocess.run([sys.executable, "-c",
                          "from block_sparse_long_phase_b200 import _abi; print(_abi.LIB_PATH)"],
                         cwd=ROOT, env=env, capture_output=True, text=True)
    assert chk.stdout.strip().endswith("libstar_checked.so")
