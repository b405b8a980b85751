"""Parity of the CUDA path (through the C ABI) with the CPU oracle."""
import numpy as np
import pytest
import torch

import kvpop_workloads as wl

pytestmark = pytest.mark.gpu

gh = pytest.importorskip("gpu_harness")


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_tiny_workload_full_run_matches_oracle():
    """The tiny fp32 workload end to end: 128-token prefill, 128 decode steps,
    MLP scorer on the GPU; outputs within fp32 tolerance at every step, GPU
    scores within 1e-4 relative, long-range sets equal (up to near-ties)."""
    _need_gpu()
    w = wl.TINY
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode)
    for unit in range(w.batch * w.n_kv_heads):
        gh.check_unit(run, 0, unit, exact_slots=False, atol=gh.F32_ATOL)


@pytest.mark.parametrize("dtype,d,hq,hkv", [("f32", 64, 4, 2), ("bf16", 64, 8, 2), ("bf16", 128, 8, 2),
                                            ("bf16", 128, 4, 4), ("bf16", 64, 16, 2)])
@pytest.mark.parametrize("S,W,D,K", [(4, 16, 0, 44), (2, 8, 5, 20), (0, 1, 0, 7), (3, 4, 0, 0)])
def test_external_scores_bit_exact_slots(dtype, d, hq, hkv, S, W, D, K):
    """Identical (tie-heavy) score arrays on both sides: the slot -> position
    map must equal the oracle's slot simulator bit for bit at every step."""
    _need_gpu()
    w = wl.Workload("ext_case", batch=3, n_layers=2, n_q_heads=hq, n_kv_heads=hkv, head_dim=d, dtype=dtype,
                    sinks=S, window=W, topk=K, delay=D, prefill=57, decode=40, scorer_hidden=32,
                    heavy_hitter_frac=0.02 if dtype == "bf16" else 0.0)
    run = gh.run_gpu(w, n_layers=2, n_steps=w.decode, external=True, tie_levels=3, layers_to_keep=(1,))
    atol = gh.F32_ATOL if dtype == "f32" else gh.BF16_ATOL
    for unit in range(w.batch * w.n_kv_heads):
        gh.check_unit(run, 1, unit, exact_slots=True, atol=atol)


@pytest.mark.parametrize("chunks", [[10, 30, 17], [1] * 12 + [45], [56, 1]])
def test_chunked_prefill_bit_exact(chunks):
    """Prefill in chunks: survivors keep their slots, newcomers fill free or
    vacated slots in ascending order; then decode continues exactly."""
    _need_gpu()
    w = wl.Workload("chunk_case", batch=2, n_layers=1, n_q_heads=8, n_kv_heads=2, head_dim=128, dtype="bf16",
                    sinks=3, window=6, topk=9, delay=2, prefill=sum(chunks), decode=20, scorer_hidden=64)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, external=True, tie_levels=2, chunks=chunks)
    for unit in range(w.batch * w.n_kv_heads):
        gh.check_unit(run, 0, unit, exact_slots=True, atol=gh.BF16_ATOL, chunks=chunks)


def test_budget_covering_context_is_dense_attention():
    """Budget >= context: every token is attended (dense causal attention)."""
    _need_gpu()
    w = wl.Workload("dense_case", batch=2, n_layers=1, n_q_heads=8, n_kv_heads=2, head_dim=128, dtype="bf16",
                    sinks=4, window=32, topk=300, delay=0, prefill=100, decode=60, scorer_hidden=64,
                    heavy_hitter_frac=0.02)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode)
    for unit in range(4):
        res = gh.check_unit(run, 0, unit, exact_slots=False, atol=gh.BF16_ATOL)
        assert res.attended_counts == [w.prefill + i + 1 for i in range(w.decode)]


def test_decode_from_empty_cache():
    """No prompt at all: sinks, window and long-range slots fill during decode."""
    _need_gpu()
    w = wl.Workload("empty_case", batch=2, n_layers=1, n_q_heads=4, n_kv_heads=2, head_dim=64, dtype="f32",
                    sinks=4, window=8, topk=10, delay=3, prefill=0, decode=50, scorer_hidden=32)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, external=True, tie_levels=3)
    for unit in range(4):
        gh.check_unit(run, 0, unit, exact_slots=True, atol=gh.F32_ATOL, chunks=[])


def test_many_segments_per_unit_merge():
    """Few units with long caches: each unit's slots are split over many
    consumer warps, so the split-K merge (atomic ticket, LSE combine) runs."""
    _need_gpu()
    w = wl.Workload("merge_case", batch=1, n_layers=1, n_q_heads=8, n_kv_heads=2, head_dim=128, dtype="bf16",
                    sinks=4, window=64, topk=1980, delay=0, prefill=2600, decode=6, scorer_hidden=64,
                    heavy_hitter_frac=0.02)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode)
    for unit in range(2):
        gh.check_unit(run, 0, unit, exact_slots=False, atol=gh.BF16_ATOL)


def test_nonfinite_free_outputs_and_rows_hold_tokens():
    """Every occupied slot row holds exactly the k/v of the token its position
    says (checks the in-place copies of append, staging move and replace)."""
    _need_gpu()
    w = wl.Workload("rows_case", batch=2, n_layers=1, n_q_heads=8, n_kv_heads=2, head_dim=128, dtype="bf16",
                    sinks=2, window=5, topk=11, delay=3, prefill=40, decode=25, scorer_hidden=64)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, external=True, tie_levels=4)
    rows = run.cache.kv_rows(0).cpu()
    pos, _, state = run.cache.inspect(0)
    for unit in range(4):
        k_all, v_all, _ = gh.unit_inputs(run, 0, unit)
        for slot, p in enumerate(pos[unit]):
            if p < 0:
                continue
            r = rows[unit, slot].view(torch.bfloat16).double().numpy()
            np.testing.assert_array_equal(r[:128], k_all[p])
            np.testing.assert_array_equal(r[128:], v_all[p])
        assert state[unit][0] == w.prefill + w.decode
    for o in run.outs[0]:
        assert torch.isfinite(o).all()


@pytest.mark.parametrize("S,W,D,K", [(4, 16, 0, 44), (2, 8, 5, 20), (0, 1, 0, 7), (2, 3, 1, 6)])
def test_split_append_attend_matches_fused_step(S, W, D, K):
    """kvpop_decode_append + kvpop_decode_attend (two launches) and the fused
    kvpop_decode_step agree: identical slot maps, outputs equal up to fp32
    summation order."""
    _need_gpu()
    w = wl.Workload("split_case", batch=2, n_layers=1, n_q_heads=8, n_kv_heads=2, head_dim=128, dtype="bf16",
                    sinks=S, window=W, topk=K, delay=D, prefill=50, decode=30, scorer_hidden=64,
                    heavy_hitter_frac=0.02)
    a = gh.run_gpu(w, n_layers=1, n_steps=w.decode)
    b = gh.run_gpu(w, n_layers=1, n_steps=w.decode, split=True)
    for i in range(w.decode + 1):
        np.testing.assert_array_equal(a.slot_pos[0][i], b.slot_pos[0][i])
    for i in range(w.decode):
        np.testing.assert_allclose(a.outs[0][i].numpy(), b.outs[0][i].numpy(), rtol=0, atol=1.6e-2)
    for unit in range(4):
        gh.check_unit(b, 0, unit, exact_slots=False, atol=gh.BF16_ATOL)


@pytest.mark.parametrize("external", [True, False])
def test_team_decision_with_several_key_batches(external):
    """Two units (fewer than CTAs): a CTA's four decider warps share each
    decision, and with K = 2100 each warp scans 525 long-range keys in two
    batches of loads.  Prompt 2400 (the long-range set full), 6 decode
    steps; slot maps bit-exact against the slot simulator with tie-heavy
    caller scores, exact fp32 scores with the MLP."""
    _need_gpu()
    w = wl.Workload("team_case", batch=1, n_layers=1, n_q_heads=8, n_kv_heads=2, head_dim=128, dtype="bf16",
                    sinks=4, window=16, topk=2100, delay=0, prefill=2400, decode=6, scorer_hidden=64,
                    heavy_hitter_frac=0.02)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, external=external, tie_levels=3 if external else 0)
    for unit in range(2):
        gh.check_unit(run, 0, unit, exact_slots=external, atol=gh.BF16_ATOL)
    if not external:
        pos, score, _ = run.cache.inspect(0)
        base = w.sinks + w.window + w.delay
        for unit in range(2):
            k_all, v_all, _ = gh.unit_inputs(run, 0, unit)
            ref = gh.unit_scores(run, 0, unit, k_all, v_all)
            got = [(int(pos[unit, sl]), float(score[unit, sl])) for sl in range(base, pos.shape[1]) if pos[unit, sl] >= 0]
            assert len(got) == w.topk
            assert all(np.float32(ref[p_]) == s_ for p_, s_ in got), f"unit {unit}: scores differ"


def test_mlp_scores_match_oracle_exactly_in_fp32():
    """The scorer accumulates in fp64 and rounds once, so the long-range slots'
    fp32 scores equal the oracle's float64-then-float32 scores."""
    _need_gpu()
    w = wl.Workload("score_case", batch=2, n_layers=1, n_q_heads=8, n_kv_heads=2, head_dim=128, dtype="bf16",
                    sinks=4, window=16, topk=40, delay=2, prefill=120, decode=24, scorer_hidden=64,
                    heavy_hitter_frac=0.02)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode)
    pos, score, _ = run.cache.inspect(0)
    base = w.sinks + w.window + w.delay
    n_exact = n_total = 0
    for unit in range(4):
        k_all, v_all, _ = gh.unit_inputs(run, 0, unit)
        ref = gh.unit_scores(run, 0, unit, k_all, v_all)
        for sl in range(base, pos.shape[1]):
            if pos[unit, sl] >= 0:
                n_total += 1
                n_exact += int(np.float32(ref[pos[unit, sl]]) == score[unit, sl])
    assert n_total == 4 * w.topk
    assert n_exact == n_total, f"{n_total - n_exact} of {n_total} scores differ from the oracle's fp32 value"


@pytest.mark.parametrize("external,S,W,D,K", [(True, 4, 16, 0, 44), (True, 2, 3, 2, 9), (False, 4, 16, 0, 44),
                                              (False, 2, 8, 5, 20)])
def test_temporal_decay_matches_oracle(external, S, W, D, K):
    """Temporal decay (per-head ln gamma, different per layer and head):
    with identical caller scores the slot maps equal the oracle's bit for
    bit; with the MLP scorer the long-range slots' fp32 priorities equal the
    oracle's exactly.  Outputs match at every step.  Includes a chunked
    prefill, so prompt tokens and decode tokens both take the priority."""
    _need_gpu()
    w = wl.Workload("decay_case", batch=2, n_layers=2, n_q_heads=8, n_kv_heads=2, head_dim=128, dtype="bf16",
                    sinks=S, window=W, topk=K, delay=D, prefill=90, decode=40, scorer_hidden=64,
                    heavy_hitter_frac=0.02)
    lg = -np.array([[0.003, 0.04], [0.0, 0.2]], np.float32)   # [L][Hkv]; includes no decay (0)
    chunks = [30, 60]
    run = gh.run_gpu(w, n_layers=2, n_steps=w.decode, external=external, tie_levels=3 if external else 0,
                     layers_to_keep=(0, 1), chunks=chunks, log_decay=lg)
    for layer in (0, 1):
        for unit in range(w.batch * w.n_kv_heads):
            gh.check_unit(run, layer, unit, exact_slots=external, atol=gh.BF16_ATOL, chunks=chunks)
    if not external:
        base = S + W + D
        for layer in (0, 1):
            pos, score, _ = run.cache.inspect(layer)
            for unit in range(w.batch * w.n_kv_heads):
                k_all, v_all, _ = gh.unit_inputs(run, layer, unit)
                pr = gh.unit_scores(run, layer, unit, k_all, v_all)
                for sl in range(base, pos.shape[1]):
                    if pos[unit, sl] >= 0:
                        assert np.float32(pr[pos[unit, sl]]) == score[unit, sl], (layer, unit, sl)


@pytest.mark.parametrize("dtype,d,hq,hkv", [("bf16", 128, 8, 2), ("f32", 64, 4, 2)])
def test_linear_scorer_matches_oracle(dtype, d, hq, hkv):
    """Stateless headwise linear scorer (scorer_hidden = 0): GPU scores of
    the long-range tokens equal the oracle's float64-then-float32 scores
    exactly, sets and outputs match at every step, over a chunked prefill
    and decode with a staging ring."""
    _need_gpu()
    w = wl.Workload("linear_case", batch=2, n_layers=1, n_q_heads=hq, n_kv_heads=hkv, head_dim=d, dtype=dtype,
                    sinks=3, window=10, topk=30, delay=2, prefill=100, decode=30, scorer_hidden=0,
                    heavy_hitter_frac=0.02 if dtype == "bf16" else 0.0)
    chunks = [37, 63]
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, chunks=chunks)
    atol = gh.F32_ATOL if dtype == "f32" else gh.BF16_ATOL
    pos, score, _ = run.cache.inspect(0)
    base = w.sinks + w.window + w.delay
    for unit in range(w.batch * w.n_kv_heads):
        gh.check_unit(run, 0, unit, exact_slots=False, atol=atol, chunks=chunks)
        k_all, v_all, _ = gh.unit_inputs(run, 0, unit)
        ref = gh.unit_scores(run, 0, unit, k_all, v_all)
        for sl in range(base, pos.shape[1]):
            assert pos[unit, sl] >= 0
            assert np.float32(ref[pos[unit, sl]]) == score[unit, sl], (unit, sl)


def test_full_size_target_config_sampled_units():
    """The 87.5%-compression target shape at full size (64 rows x 8 KV heads,
    prompt 8192, B = 1024 = 4 + 128 + 892, G = 4, bf16, MLP scorer), one
    layer, in the launch configuration bench.py times (one CTA per SM, 10
    consumer + 2 decider warps, 64 tiles per unit split over ~3 warps).
    Prefill plus 4 fused decode steps; three sampled units (first, middle,
    last) checked against the oracle at every step: outputs, long-range sets
    and exact fp32 scores."""
    _need_gpu()
    w = wl.QWEN3_4B_CR88.replace(name="full_size_case", n_layers=1, decode=4)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, gen_device="cuda", debug=False)
    units = w.batch * w.n_kv_heads
    for unit in (0, units // 2 + 3, units - 1):
        gh.check_unit(run, 0, unit, exact_slots=False, atol=gh.BF16_ATOL)
    pos, score, state = run.cache.inspect(0)
    base = w.sinks + w.window + w.delay
    assert (pos[:, base:] >= 0).all()                       # every long-range slot filled
    assert (state[:, 0] == w.prefill + w.decode).all()     # every unit advanced


def test_full_size_cr75_sampled_units():
    """The 75%-compression Qwen3-4B shape at full size (16 rows x 8 KV heads,
    prompt 8192, B = 2048 = 4 + 128 + 1916, G = 4, bf16, MLP scorer), one
    layer, bench.py's launch configuration.  Prefill plus 4 fused decode
    steps; first, middle and last units against the oracle at every step:
    outputs, long-range sets and exact fp32 scores."""
    _need_gpu()
    w = wl.QWEN3_4B_CR75.replace(name="full_size_cr75_case", n_layers=1, decode=4)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, gen_device="cuda", debug=False)
    units = w.batch * w.n_kv_heads
    for unit in (0, units // 2 + 3, units - 1):
        gh.check_unit(run, 0, unit, exact_slots=False, atol=gh.BF16_ATOL)
    pos, score, state = run.cache.inspect(0)
    base = w.sinks + w.window + w.delay
    assert (pos[:, base:] >= 0).all()
    assert (state[:, 0] == w.prefill + w.decode).all()


def test_full_size_8b_delayed_scoring_sampled_units():
    """The Qwen3-8B shape with delayed scoring at full size (32 rows x 8 KV
    heads, prompt 32768, B = 4096 = 4 + 256 + 3836 plus a D = 32 staging ring,
    G = 4, bf16, MLP scorer), one layer.  Prefill plus 4 fused decode steps;
    first, middle and last units against the oracle at every step, including
    the staged tokens being attended and scored 32 steps after they leave the
    window."""
    _need_gpu()
    w = wl.QWEN3_8B_D32.replace(name="full_size_8b_case", n_layers=1, decode=4)
    run = gh.run_gpu(w, n_layers=1, n_steps=w.decode, gen_device="cuda", debug=False)
    units = w.batch * w.n_kv_heads
    for unit in (0, units // 2 + 3, units - 1):
        res = gh.check_unit(run, 0, unit, exact_slots=False, atol=gh.BF16_ATOL)
        assert res.attended_counts == [w.budget + w.delay] * w.decode
    pos, score, state = run.cache.inspect(0)
    base = w.sinks + w.window + w.delay
    assert (pos[:, base:] >= 0).all()
    assert (pos[:, w.sinks + w.window:base] >= 0).all()     # the staging ring is full
    assert (state[:, 0] == w.prefill + w.decode).all()
