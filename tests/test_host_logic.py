"""Host-side logic checked on the CPU: the decode kernel's split-K work
decomposition (restated from kvpop_internal.cuh) covers every tile exactly
once and never gives a unit more partials than the scratch holds."""
import random

import pytest

K_MAX_SEG = 64


def seg_lo(w, total, nw):
    return (w * total) // nw


def warp_of_tile(x, total, nw):
    return ((x + 1) * nw - 1) // total


def active_warps(total, tpu, launched):
    nw = min(launched, total)
    min_tiles = max(1, (tpu + K_MAX_SEG - 2) // (K_MAX_SEG - 1))
    cap = max(1, total // min_tiles)
    return min(nw, cap)


def _check(units, tpu, launched):
    total = units * tpu
    nw = active_warps(total, tpu, launched)
    assert 1 <= nw <= launched
    owner = []
    for w in range(nw):
        lo, hi = seg_lo(w, total, nw), seg_lo(w + 1, total, nw)
        assert hi > lo, "every active warp gets at least one tile"
        owner += [w] * (hi - lo)
    assert len(owner) == total
    for x in (0, total - 1, total // 2, random.randrange(total)):
        assert warp_of_tile(x, total, nw) == owner[x]
    for u in range(units):
        first, last = owner[u * tpu], owner[u * tpu + tpu - 1]
        assert warp_of_tile(u * tpu, total, nw) == first
        assert warp_of_tile(u * tpu + tpu - 1, total, nw) == last
        assert last - first + 1 <= K_MAX_SEG


@pytest.mark.parametrize("units", [1, 2, 3, 8, 16, 64, 128, 512])
@pytest.mark.parametrize("tpu", [1, 2, 5, 63, 64, 65, 127, 128, 129, 257, 512])
def test_decode_work_split(units, tpu):
    random.seed(units * 1000 + tpu)
    for launched in (8, 9 * 8, 148 * 8, 1184):
        _check(units, tpu, launched)


def test_prefill_attention_flop_count():
    """bench.py's flop count of one prefill-attention call: 4 d flops per
    attended (position, query head) pair, position q attending min(q + 1, B + D)
    tokens; checked against the sum written out for a small shape and the
    closed form sum_{q<B'} (q + 1) + (n - B') B' for the target shape."""
    import bench
    import kvpop_workloads as wl
    small = wl.TINY.replace(prefill=30)          # B + D = 4 + 16 + 44 = 64 > 30: every position dense
    assert bench.prefill_attention_flops(small) == 4.0 * 64 * sum(q + 1 for q in range(30)) * 4 * 1
    w = wl.QWEN3_4B_CR88.replace(n_layers=1)
    Bp = w.sinks + w.window + w.delay + w.topk
    n = w.prefill
    pairs = Bp * (Bp + 1) // 2 + (n - Bp) * Bp
    assert bench.prefill_attention_flops(w) == 4.0 * w.head_dim * pairs * w.n_q_heads * w.batch


def test_bench_arguments(monkeypatch):
    """Default steps stay unset until the chosen path fills them in (200 decode
    steps, 10 prefill-attention calls); the prefill-attention options parse."""
    import sys
    import bench
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    a = bench.parse_args()
    assert a.path == "decode" and a.steps is None and a.pa_batch == 0
    monkeypatch.setattr(sys, "argv", ["bench.py", "--path", "prefill-attention", "--pa-batch", "4", "--steps", "2"])
    a = bench.parse_args()
    assert a.path == "prefill-attention" and a.pa_batch == 4 and a.steps == 2


def test_sweep_plan_covers_the_grid_and_bounds_memory():
    """Every (budget, batch) point of the bandwidth sweep is planned once;
    the 36-layer cache is kept whole where it fits under the cap, and the
    points where it does not (b256 x B8192 = 309 GB is larger than HBM) run
    fewer layers, each point's cache within the cap; the prompt fills the
    long-range slots (prompt - W - S >= K)."""
    import bench
    import kvpop_workloads as wl
    plan = bench.sweep_plan()
    assert {(p["budget"], p["batch"]) for p in plan} == {(B, b) for B in wl.SWEEP_BUDGETS
                                                           for b in wl.SWEEP_BATCHES}
    assert len(plan) == len(wl.SWEEP_BUDGETS) * len(wl.SWEEP_BATCHES)
    for p in plan:
        w = p["workload"]
        per_layer = bench.attention_bytes(w)
        assert 1 <= p["layers"] <= 36 and w.n_layers == p["layers"]
        assert p["layers"] == 36 or per_layer * (p["layers"] + 1) > bench.SWEEP_CACHE_CAP
        assert per_layer * p["layers"] <= bench.SWEEP_CACHE_CAP
        assert p["prompt"] - w.window - w.sinks >= w.topk
        assert w.budget == p["budget"] and w.batch == p["batch"]
    big = [p for p in plan if p["budget"] == 8192 and p["batch"] == 256][0]
    assert big["full_cache_gb"] > 180 and big["layers"] < 36
    small = [p for p in plan if p["budget"] == 512 and p["batch"] == 1][0]
    assert small["layers"] == 36


def test_dtype_names_are_explicit():
    """make_config accepts only known element-type names; a typo raises
    instead of silently building a bf16 cache."""
    import torch
    import fixed_budget_kv_kvpop_b200 as kp
    for name in ("f32", "float32", "fp32", torch.float32):
        assert kp.dtype_code(name) == kp.KVPOP_DTYPE_F32
    for name in ("bf16", "bfloat16", torch.bfloat16):
        assert kp.dtype_code(name) == kp.KVPOP_DTYPE_BF16
    for bad in ("float", "fp16", "bf 16", torch.float16, None):
        with pytest.raises(ValueError):
            kp.dtype_code(bad)


def test_tensor_checks_reject_host_tensors():
    """The binding checks every tensor before passing its address on: a
    host tensor, a wrong dtype, shape or layout raises ValueError."""
    import torch
    import fixed_budget_kv_kvpop_b200 as kp
    dev = torch.device("cuda", 0)
    with pytest.raises(ValueError, match="cuda"):
        kp.check_tensor(torch.zeros(2, 3), "q", (2, 3), torch.float32, dev)
    with pytest.raises(ValueError, match="torch.Tensor"):
        kp.check_tensor([1.0], "q", (1,), torch.float32, dev)
    meta = torch.empty(2, 3, device="meta")
    with pytest.raises(ValueError):
        kp.check_tensor(meta, "q", (2, 3), torch.float32, dev)
