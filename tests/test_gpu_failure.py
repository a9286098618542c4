"""Failure paths on the GPU, made without a GPU fault.

A bounded wait that runs out: the self-test kernel waits, with the pipelined
kernels' own bounded mbarrier wait, on a barrier nothing completes; the wait
must give up, the kernel must report it and return, and the context must stay
usable.  A failed allocation: the STAR_FAULT_INJECT test hook makes the
cache's one cudaMalloc fail; creation must return STAR_ENOMEM and a later
creation must work.  After each, a small phase 1 is checked against the
oracle.
"""

import ctypes
import time

import numpy as np
import pytest
import torch

from block_sparse_long_phase_b200 import workloads as wl
from oracle import star_oracle as so

pytestmark = pytest.mark.gpu


def small_phase1_matches_the_oracle():
    from block_sparse_long_phase_b200 import StarCache
    w = wl.get("tiny")
    cpu = wl.make_inputs(w, "cpu", with_decode=False)
    x = {k: v.cuda() for k, v in cpu.items()}
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq, w.scale)
    O, LSE = cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    Oref, Lref = so.ctx_encode(cpu["Qc"], cpu["Kc"], cpu["Vc"], w.b, w.b_a, w.scale)
    err = np.abs(O.double().cpu().numpy() - Oref)
    assert err.max() <= 1e-2 and err.mean() <= 1e-3
    assert np.abs(LSE.double().cpu().numpy() - Lref).max() <= 1e-3
    cache.close()


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    from block_sparse_long_phase_b200 import _abi
    lib = _abi.load()
    torch.cuda.init()
    for polls in (1, 1000):
        gave_up = ctypes.c_int(0)
        t0 = time.perf_counter()
        rc = lib.star_selftest_wait_timeout(polls, ctypes.byref(gave_up), None)
        dt = time.perf_counter() - t0
        assert rc == _abi.STAR_OK, lib.star_last_error()
        assert gave_up.value == 1, "the wait on a barrier nothing completes did not give up"
        assert dt < 5.0
    small_phase1_matches_the_oracle()


def test_injected_allocation_failure_leaves_the_library_usable(monkeypatch):
    from block_sparse_long_phase_b200 import StarCache
    from block_sparse_long_phase_b200._abi import StarError, STAR_ENOMEM
    monkeypatch.setenv("STAR_FAULT_INJECT", "alloc")
    with pytest.raises(StarError) as e:
        StarCache(1, 4, 2, 64, 1024, 256, 256, 8)
    assert e.value.code == STAR_ENOMEM
    monkeypatch.delenv("STAR_FAULT_INJECT")
    small_phase1_matches_the_oracle()
