"""kvpop_decode_step_noalloc: the decode step for callers that cannot allocate
device memory (a plugin whose host engine plans every device byte itself, or
a decode loop that must not risk the device-wide synchronisation of
cudaMalloc/cudaFree).  Its split-K scratch lives in the library's static
16 MiB device buffer, so it must give what kvpop_decode_step gives.

This file is collected last, so a run that stops at its first failure has
run every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

import fixed_budget_kv_kvpop_b200 as kp
import kvpop_workloads as wl


def test_noalloc_rejects_null_arguments():
    assert kp.lib.kvpop_decode_step_noalloc(None, 0, None, None, None, None, None, None) == kp.KVPOP_ERR_INVALID_ARG
    assert kp.lib.kvpop_status_string(kp.KVPOP_ERR_SCRATCH_LIMIT).decode() != "unknown status"


def _noalloc_need(units, G, d):
    a256 = lambda x: (x + 255) // 256 * 256
    return a256(units * 64 * G * d * 4) + a256(units * 64 * G * 2 * 4) + a256(units * 4)


def test_scratch_limit_formula_matches_header():
    """The documented need (G = 4, d = 128) fits up to 126 units."""
    assert _noalloc_need(126, 4, 128) <= kp.KVPOP_NOALLOC_SCRATCH_BYTES < _noalloc_need(127, 4, 128)


def _cache(w, weights):
    w1, b1, w2, b2 = weights
    cfg = kp.make_config(batch=w.batch, n_layers=w.n_layers, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                         head_dim=w.head_dim, sinks=w.sinks, window=w.window, topk=w.topk, delay=w.delay,
                         max_prefill_chunk=max(w.prefill, 1), dtype=w.dtype, scorer_hidden=w.scorer_hidden,
                         w1=w1, b1=b1, w2=w2, b2=b2, debug_checks=True)
    return kp.KVPopCache(cfg, device="cuda", keepalive=weights)


@pytest.mark.gpu
def test_noalloc_matches_decode_step_on_consecutive_calls():
    """Two identical caches: one stepped by kvpop_decode_step, the other by
    kvpop_decode_step_noalloc, two steps of two layers (four calls in a row
    that share the static buffer).  Long caches split each unit over many
    warps, so the partials and tickets in the static buffer are exercised.
    Outputs agree within the bf16 tolerance of the parity tests; slot maps,
    scores and device error words are identical."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gpu_harness import BF16_ATOL
    w = wl.Workload("noalloc_case", batch=4, n_layers=2, n_q_heads=32, n_kv_heads=8, head_dim=128, dtype="bf16",
                    sinks=4, window=64, topk=956, delay=0, prefill=2048, decode=2, scorer_hidden=64,
                    heavy_hitter_frac=0.02)
    assert _noalloc_need(w.batch * w.n_kv_heads, w.group, w.head_dim) <= kp.KVPOP_NOALLOC_SCRATCH_BYTES
    weights = tuple(t.cuda() for t in wl.scorer_weights(w))
    ref, alt = _cache(w, weights), _cache(w, weights)
    for layer in range(w.n_layers):
        k, v = (t.cuda() for t in wl.prompt_kv(w, layer))
        ref.prefill(layer, k, v)
        alt.prefill(layer, k, v)
    for step in range(w.decode):
        for layer in range(w.n_layers):
            q, kn, vn = (t.cuda() for t in wl.decode_inputs(w, layer, step))
            o_ref, o_alt = torch.empty_like(q), torch.empty_like(q)
            ref.decode_step(layer, q, kn, vn, o_ref)
            alt.decode_step_noalloc(layer, q, kn, vn, o_alt)
            torch.cuda.synchronize()
            assert torch.isfinite(o_alt.float()).all()
            np.testing.assert_allclose(o_alt.double().cpu().numpy(), o_ref.double().cpu().numpy(),
                                       rtol=0, atol=BF16_ATOL, err_msg=f"step {step} layer {layer}")
            p_ref, s_ref, st_ref = ref.inspect(layer)
            p_alt, s_alt, st_alt = alt.inspect(layer)
            np.testing.assert_array_equal(p_alt, p_ref)
            np.testing.assert_array_equal(s_alt, s_ref)
            np.testing.assert_array_equal(st_alt, st_ref)
    assert ref.get_error() == (kp.KVPOP_OK, 0)
    assert alt.get_error() == (kp.KVPOP_OK, 0)


@pytest.mark.gpu
def test_noalloc_rejects_a_problem_beyond_the_static_buffer():
    """136 units at G = 4, d = 128 need more than 16 MiB: the call returns
    KVPOP_ERR_SCRATCH_LIMIT, enqueues nothing, and the layer then steps
    normally through kvpop_decode_step."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = wl.Workload("noalloc_limit", batch=17, n_layers=1, n_q_heads=32, n_kv_heads=8, head_dim=128,
                    dtype="bf16", sinks=2, window=8, topk=6, delay=0, prefill=24, decode=1, scorer_hidden=64)
    assert _noalloc_need(w.batch * w.n_kv_heads, w.group, w.head_dim) > kp.KVPOP_NOALLOC_SCRATCH_BYTES
    weights = tuple(t.cuda() for t in wl.scorer_weights(w))
    cache = _cache(w, weights)
    k, v = (t.cuda() for t in wl.prompt_kv(w, 0))
    cache.prefill(0, k, v)
    q, kn, vn = (t.cuda() for t in wl.decode_inputs(w, 0, 0))
    out = torch.empty_like(q)
    st = kp.lib.kvpop_decode_step_noalloc(cache.handle, 0, q.data_ptr(), kn.data_ptr(), vn.data_ptr(),
                                          out.data_ptr(), None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == kp.KVPOP_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert cache.inspect(0)[2][0][0] == w.prefill    # position counter untouched
    cache.decode_step(0, q, kn, vn, out)
    assert cache.inspect(0)[2][0][0] == w.prefill + 1
    assert cache.get_error() == (kp.KVPOP_OK, 0)
