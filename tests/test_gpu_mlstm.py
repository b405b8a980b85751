"""Parity of the stateful mLSTM scorer with delayed readout (CUDA, through the
C ABI) with the CPU oracle (unit_scores_mlstm; KVpop page §A, §E.3, §E.4):
the long-range slots' fp32 scores within 1e-4 relative of the oracle's, the
long-range sets equal up to near-ties, and attention outputs within the
dtype's tolerance at every decode step, over chunked prefills, staging rings
(D > 0), temporal decay, both split and fused decode entry points."""
import numpy as np
import pytest
import torch

import kvpop_workloads as wl

pytestmark = pytest.mark.gpu

gh = pytest.importorskip("gpu_harness")


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check_scores(run, layer):
    """Every occupied long-range slot's fp32 score against the oracle's."""
    w = run.w
    pos, score, _ = run.cache.inspect(layer)
    base = w.sinks + w.window + w.delay
    n = 0
    for unit in range(w.batch * w.n_kv_heads):
        k_all, v_all, _ = gh.unit_inputs(run, layer, unit)
        ref = gh.unit_scores(run, layer, unit, k_all, v_all)
        tol = gh.score_tol(ref, ref)
        for sl in range(base, pos.shape[1]):
            if pos[unit, sl] >= 0:
                j = int(pos[unit, sl])
                assert np.isfinite(ref[j]), (unit, sl, j)
                assert abs(float(score[unit, sl]) - ref[j]) <= tol[j], (unit, sl, j, float(score[unit, sl]), ref[j])
                n += 1
    return n


@pytest.mark.parametrize("dtype,d,hq,hkv,S,W,D,K,p,dv", [
    ("f32", 64, 4, 2, 4, 16, 0, 44, 8, 8),       # the tiny workload's shape
    ("bf16", 128, 8, 2, 4, 16, 0, 40, 16, 16),
    ("bf16", 128, 8, 2, 2, 8, 5, 20, 16, 16),     # staging ring: scored D steps after leaving the window
    ("bf16", 64, 8, 2, 3, 10, 2, 25, 4, 24),      # dv above 16
    ("f32", 64, 4, 2, 0, 1, 0, 7, 1, 1),          # no sinks, window 1, one-dimensional projections
])
def test_mlstm_scores_sets_and_outputs(dtype, d, hq, hkv, S, W, D, K, p, dv):
    _need_gpu()
    w = wl.Workload(f"mlstm_{dtype}_d{d}_s{S}w{W}d{D}k{K}_p{p}v{dv}", batch=2, n_layers=1, n_q_heads=hq,
                    n_kv_heads=hkv, head_dim=d, dtype=dtype, sinks=S, window=W, topk=K, delay=D, prefill=90,
                    decode=40, scorer_hidden=64, heavy_hitter_frac=0.02 if dtype == "bf16" else 0.0)
    chunks = [33, 57]
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, chunks=chunks, mlstm_dims=(p, dv))
    atol = gh.F32_ATOL if dtype == "f32" else gh.BF16_ATOL
    for unit in range(w.batch * w.n_kv_heads):
        gh.check_unit(run, 0, unit, exact_slots=False, atol=atol, chunks=chunks)
    assert _check_scores(run, 0) == w.batch * w.n_kv_heads * K


def test_mlstm_split_append_attend_and_decay():
    """kvpop_decode_append + kvpop_decode_attend with the mLSTM scorer, two
    layers with different temporal decay: the same retention and outputs as
    the oracle's decayed static priorities."""
    _need_gpu()
    w = wl.Workload("mlstm_split", batch=2, n_layers=2, n_q_heads=8, n_kv_heads=2, head_dim=128, dtype="bf16",
                    sinks=4, window=12, topk=30, delay=3, prefill=70, decode=30, scorer_hidden=64,
                    heavy_hitter_frac=0.02)
    lg = -np.array([[0.01, 0.0], [0.1, 0.002]], np.float32)
    run = gh.run_gpu(w, n_layers=2, n_steps=w.decode, layers_to_keep=(0, 1), split=True, log_decay=lg,
                     mlstm_dims=(16, 16))
    for layer in (0, 1):
        for unit in range(w.batch * w.n_kv_heads):
            gh.check_unit(run, layer, unit, exact_slots=False, atol=gh.BF16_ATOL)
        assert _check_scores(run, layer) > 0


def test_mlstm_decode_from_empty_cache():
    """No prompt: the state starts at zero and every token is scored by the
    decode steps' own kernel."""
    _need_gpu()
    w = wl.Workload("mlstm_empty", batch=2, n_layers=1, n_q_heads=4, n_kv_heads=2, head_dim=64, dtype="f32",
                    sinks=2, window=6, topk=10, delay=2, prefill=0, decode=50, scorer_hidden=32)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, mlstm_dims=(8, 8))
    for unit in range(4):
        gh.check_unit(run, 0, unit, exact_slots=False, atol=gh.F32_ATOL, chunks=[])


def test_mlstm_target_shape_sampled_units():
    """The 87.5%-compression Qwen3-4B shape (prompt 8192, B = 1024, G = 4,
    bf16) with the mLSTM scorer (p = dv = 16) on 4 rows x 8 KV heads, one
    layer, 4 decode steps: sampled units against the oracle at every step."""
    _need_gpu()
    w = wl.QWEN3_4B_CR88.replace(name="mlstm_target_case", batch=4, n_layers=1, decode=4)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, gen_device="cuda", debug=False, mlstm_dims=(16, 16))
    units = w.batch * w.n_kv_heads
    for unit in (0, units // 2 + 1, units - 1):
        gh.check_unit(run, 0, unit, exact_slots=False, atol=gh.BF16_ATOL)


def test_mlstm_rejected_by_prefill_attention():
    """The parallel prefill attention takes the stateless scorers only."""
    _need_gpu()
    import fixed_budget_kv_kvpop_b200 as kp
    w = wl.TINY
    packed = wl.mlstm_weights(w, 4, 4).cuda()
    cfg = kp.make_config(batch=1, n_layers=1, n_q_heads=4, n_kv_heads=2, head_dim=64, sinks=4, window=16, topk=44,
                         max_prefill_chunk=8, dtype="f32", scorer="mlstm", mlstm_p=4, mlstm_dv=4, mlstm_w=packed)
    cache = kp.KVPopCache(cfg, keepalive=(packed,))
    with pytest.raises(kp.KVPopError):
        cache.prefill_attention_workspace_bytes(32)
