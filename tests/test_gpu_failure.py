"""Failure detection on the GPU without a GPU fault: a bounded device-side
wait that runs out is reported as KVPOP_ERR_TIMEOUT, the kernel returns, and
the context and the cache stay usable.

The failure is injected through the test build of the library (compiled with
KVPOP_TEST_HOOKS; its decode kernel's merge-queue waits give up after 50 ms):
one consumer warp finishes its work but never reports that it is done, so its
CTA's merge helpers wait for a report that never comes.  That wait is on
shared memory only, with no copy in flight; no TMA or mbarrier wait is made
to run out."""
import os
import time

import numpy as np
import pytest
import torch

import kvpop_workloads as wl

pytestmark = pytest.mark.gpu

gh = pytest.importorskip("gpu_harness")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _hooks_library():
    import importlib.util
    import fixed_budget_kv_kvpop_b200 as kp
    spec = importlib.util.spec_from_file_location(
        "kvpop_build", os.path.join(ROOT, "fixed_budget_kv_kvpop_b200", "csrc", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return kp.load_library(mod.build_test_hooks())


def test_merge_wait_runs_out_reports_timeout_and_recovers():
    _need_gpu()
    import fixed_budget_kv_kvpop_b200 as kp
    lib2 = _hooks_library()
    w = wl.Workload("failure_case", batch=2, n_layers=1, n_q_heads=8, n_kv_heads=2, head_dim=128, dtype="bf16",
                    sinks=4, window=16, topk=40, delay=0, prefill=100, decode=8, scorer_hidden=64,
                    heavy_hitter_frac=0.02)
    fail_step = 3
    seen = {}

    def hook(cache, i, when):
        if i == fail_step and when == "before":
            cache.set_test_hook(1)
            seen["t0"] = time.perf_counter()
        if i == fail_step and when == "after":
            st, bits = cache.get_error()          # synchronises: the kernel has returned
            seen["dt"] = time.perf_counter() - seen["t0"]
            seen["status"], seen["bits"] = st, bits
            cache.set_test_hook(0)
            cache.clear_error()
        elif when == "after":
            st, bits = cache.get_error()
            assert st == kp.KVPOP_OK, (i, st, bits)

    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, library=lib2, step_hook=hook)
    assert seen["status"] == kp.KVPOP_ERR_TIMEOUT, seen
    assert seen["bits"] & kp.KVPOP_DEVERR_TIMEOUT, seen
    assert seen["dt"] < 30.0, seen                 # the bounded wait gave up; nothing hung
    # every step after the failure (and before it) matches the oracle: the
    # timed-out wait came after all merges of its step, so the cache stayed
    # consistent; the failing step's outputs are undefined by the API
    steps = [i for i in range(w.decode) if i != fail_step]
    for unit in range(w.batch * w.n_kv_heads):
        gh.check_unit(run, 0, unit, exact_slots=False, atol=gh.BF16_ATOL, steps_to_check=steps)
    # a fresh cache of the test build runs clean
    fresh = gh.run_gpu(w, n_layers=1, n_steps=4, library=lib2)
    for unit in range(w.batch * w.n_kv_heads):
        gh.check_unit(fresh, 0, unit, exact_slots=False, atol=gh.BF16_ATOL)


def test_production_build_has_no_hook():
    """The library the product loads refuses the hook and changes nothing."""
    _need_gpu()
    import fixed_budget_kv_kvpop_b200 as kp
    w = wl.TINY.replace(prefill=20, decode=4)
    run = gh.run_gpu(w, n_layers=1, n_steps=2)
    with pytest.raises(kp.KVPopError):
        run.cache.set_test_hook(1)
