"""Parity of the parallel sparse prefill attention (CUDA, through the C ABI)
with the CPU oracle: running cutoffs bit-exact, outputs and log-normalisers
within the dtype's tolerance, on seeded inputs of several tiles with ragged
tails, and the edge cases of the mask (nothing eligible, K = 0, K covering the
prompt, one token); and the fused whole-prompt call
(kvpop_prefill_with_attention) bit for bit against kvpop_prefill followed by
kvpop_prefill_attention."""
import numpy as np
import pytest
import torch

import kvpop_workloads as wl
from oracle import kvpop_oracle as orc

pytestmark = pytest.mark.gpu

gh = pytest.importorskip("gpu_harness")

LSE_ATOL = {"f32": 1e-4, "bf16": 1e-3}   # fp32 sums of at most a few thousand terms


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


class PaRun:
    pass


def run_prefill_attention(w, n, *, external=False, tie_levels=0, log_decay=None, layer=0, master=0,
                          gen_device="cpu", with_lse=True, out_offset=0):
    """One prefill-attention call for `layer` of a one-layer-per-call cache
    (out_offset: the output starts that many elements into its allocation)."""
    import fixed_budget_kv_kvpop_b200 as kp
    n_layers = layer + 1
    weights = None
    if not external:
        wshape = w.replace(n_layers=n_layers, scorer_hidden=max(w.scorer_hidden, 1))
        weights = tuple(t.cuda() for t in wl.scorer_weights(wshape, master=master))
    dec = None if log_decay is None else torch.tensor(np.asarray(log_decay, np.float32), device="cuda")
    cache = gh.build_cache(w, n_layers, external, weights, max_chunk=1, debug=True, log_decay=dec)
    k, v = wl.prompt_kv(w, layer, n_tokens=n, master=master, device=gen_device)
    q = wl.prompt_queries(w, layer, n, master=master, device=gen_device)
    k, v, q = k.cuda(), v.cuda(), q.cuda()
    ext = None
    if external:
        ext = wl.external_scores(w, layer, n, master=master, device=gen_device, tie_levels=tie_levels).cuda()
    out = torch.full((q.numel() + out_offset,), float("nan"), dtype=q.dtype, device="cuda")[out_offset:].view(q.shape)
    lse = torch.full((w.batch, w.n_q_heads, n), float("nan"), device="cuda") if with_lse else None
    ws = torch.empty(cache.prefill_attention_workspace_bytes(n), dtype=torch.uint8, device="cuda")
    cache.prefill_attention(layer, q, k, v, out, lse, ws, ext)
    torch.cuda.synchronize()
    st, bits = cache.get_error()
    assert st == 0, f"device error status {st} bits {bits}"
    units = w.batch * w.n_kv_heads
    r = PaRun()
    r.w, r.n, r.layer, r.cache, r.weights = w, n, layer, cache, weights
    r.q, r.k, r.v, r.ext, r.out, r.lse = q, k, v, ext, out, lse
    r.cut = ws[:units * n * 4].view(torch.int32).reshape(units, n).cpu().numpy() if n > 0 else None
    r.log_decay = None if log_decay is None else np.asarray(log_decay, np.float32)
    return r


def unit_view(r, unit):
    w = r.w
    b, h = divmod(unit, w.n_kv_heads)
    G = w.group
    k = r.k[b, h].double().cpu().numpy()
    v = r.v[b, h].double().cpu().numpy()
    q = r.q[b, h * G:(h + 1) * G].double().cpu().numpy().transpose(1, 0, 2)   # [n][G][d]
    out = r.out[b, h * G:(h + 1) * G].double().cpu().numpy().transpose(1, 0, 2)
    lse = None if r.lse is None else r.lse[b, h * G:(h + 1) * G].double().cpu().numpy().T
    if r.ext is not None:
        s = orc.ranking_score(r.ext[b, h].double().cpu().numpy())
    else:
        w1, b1, w2, b2 = (t.double().cpu().numpy() for t in r.weights)
        if w.scorer_hidden == 0:
            s = orc.unit_scores_linear(k, v, w1[r.layer, h, 0], b2[r.layer, h])
        else:
            s = orc.unit_scores_mlp(k, v, w1[r.layer, h], b1[r.layer, h], w2[r.layer, h], b2[r.layer, h])
    if r.log_decay is not None:
        s = orc.decayed_priority(s, w.window, w.delay, float(r.log_decay[r.layer, h]))
    return k, v, q, out, lse, s


def check_all_rows(r, units=None, atol=None):
    w = r.w
    atol = atol if atol is not None else (gh.F32_ATOL if w.dtype == "f32" else gh.BF16_ATOL)
    for unit in (range(w.batch * w.n_kv_heads) if units is None else units):
        k, v, q, out, lse, s = unit_view(r, unit)
        cut = orc.running_cutoffs(s, r.n, w.sinks, w.window, w.delay, w.topk)
        assert list(r.cut[unit]) == cut, f"unit {unit}: cutoffs differ"
        ref, ref_lse, _ = orc.prefill_attention(q, k, v, s, w.sinks, w.window, w.delay, w.topk)
        np.testing.assert_allclose(out, ref, rtol=0, atol=atol, err_msg=f"unit {unit}")
        if lse is not None:
            np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=LSE_ATOL[w.dtype], err_msg=f"unit {unit} lse")


def _case(dtype, d, hq, hkv, *, S, W, D, K, hidden, batch=1):
    return wl.Workload(f"pa_{dtype}_d{d}_g{hq // hkv}_s{S}w{W}d{D}k{K}_h{hidden}", batch=batch, n_layers=1,
                       n_q_heads=hq, n_kv_heads=hkv, head_dim=d, dtype=dtype, sinks=S, window=W, topk=K,
                       delay=D, prefill=0, decode=0, scorer_hidden=hidden, heavy_hitter_frac=0.02)


def test_tiny_shape_mlp_scorer():
    """The tiny workload's shape (fp32, d 64, G 2, S 4, W 16, K 44, MLP 32):
    300 prompt positions = 9 full query tiles of 32 plus a ragged one."""
    _need_gpu()
    r = run_prefill_attention(wl.TINY.replace(prefill=0), 300)
    check_all_rows(r)


@pytest.mark.parametrize("dtype,d,hq,hkv,S,W,D,K,hidden,n,ties", [
    ("bf16", 128, 8, 2, 4, 16, 0, 40, 64, 500, 2),
    ("bf16", 128, 8, 2, 2, 12, 5, 30, 64, 333, 0),
    ("bf16", 64, 16, 2, 1, 8, 0, 20, 32, 257, 3),
    ("f32", 64, 2, 2, 0, 4, 3, 50, 32, 401, 1),
    ("bf16", 64, 8, 8, 4, 32, 0, 64, 64, 190, 0),
])
def test_external_scores_with_ties(dtype, d, hq, hkv, S, W, D, K, hidden, n, ties):
    """Caller scores (quantised so that equal scores are common): cutoffs
    bit-exact under the (score, -position) order, outputs and normalisers."""
    _need_gpu()
    w = _case(dtype, d, hq, hkv, S=S, W=W, D=D, K=K, hidden=hidden)
    r = run_prefill_attention(w, n, external=True, tie_levels=ties)
    check_all_rows(r)


@pytest.mark.parametrize("dtype,d,hq,hkv,S,W,D,K,hidden,n", [
    ("bf16", 128, 8, 2, 4, 16, 0, 40, 64, 400),
    ("bf16", 128, 4, 1, 3, 10, 4, 25, 64, 300),
    ("f32", 64, 4, 2, 2, 8, 0, 30, 0, 280),
    ("bf16", 64, 8, 2, 4, 16, 2, 20, 128, 220),
])
def test_gpu_scorer(dtype, d, hq, hkv, S, W, D, K, hidden, n):
    """The scores come from the library's own scorer (MLP of hidden 64 / 128,
    or the linear scorer), as kvpop_prefill computes them."""
    _need_gpu()
    w = _case(dtype, d, hq, hkv, S=S, W=W, D=D, K=K, hidden=hidden, batch=2)
    r = run_prefill_attention(w, n)
    check_all_rows(r)


def test_output_rows_16_byte_aligned():
    """An output buffer that is 16- but not 32-byte aligned (the tensor-core
    kernel then writes 16 bytes per store instead of 32): same parity."""
    _need_gpu()
    w = _case("bf16", 128, 8, 2, S=4, W=16, D=0, K=40, hidden=64, batch=2)
    r = run_prefill_attention(w, 333, out_offset=8)
    assert r.out.data_ptr() % 32 == 16
    check_all_rows(r)


def test_temporal_decay():
    """Ranking by the decayed static priority (ln gamma per KV head)."""
    _need_gpu()
    w = _case("bf16", 128, 8, 2, S=4, W=16, D=0, K=40, hidden=64)
    r = run_prefill_attention(w, 350, log_decay=np.array([[-0.01, -0.2]], np.float32))
    check_all_rows(r)


@pytest.mark.parametrize("S,W,D,K,n", [
    (4, 16, 0, 40, 1),          # one token
    (4, 16, 0, 40, 19),         # nothing ever eligible (n <= S + W + D)
    (4, 16, 2, 40, 23),         # exactly one eligible token at the last position
    (4, 16, 0, 0, 150),         # K = 0: sinks + window only
    (4, 16, 0, 500, 150),       # K covers the prompt: dense causal attention
    (0, 1, 0, 1, 90),           # no sinks, window 1, one long-range slot
])
def test_mask_edge_cases(S, W, D, K, n):
    _need_gpu()
    w = _case("bf16", 128, 8, 2, S=S, W=W, D=D, K=K, hidden=64)
    r = run_prefill_attention(w, n, external=True, tie_levels=2)
    check_all_rows(r)
    if K >= n:
        # every row is plain causal attention
        qt = r.q.double().cpu()
        kt = r.k.double().cpu().repeat_interleave(w.group, dim=1)
        vt = r.v.double().cpu().repeat_interleave(w.group, dim=1)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
        np.testing.assert_allclose(r.out.double().cpu().numpy(), ref.numpy(), rtol=0, atol=gh.BF16_ATOL)


def test_attention_from_cutoffs_equals_the_full_call():
    """kvpop_prefill_attention_from_cutoffs (the attention stage alone, from
    the cutoffs a first call left in the workspace) returns the full call's
    outputs and normalisers bit for bit, and another query set over the same
    mask matches the oracle."""
    _need_gpu()
    w = _case("bf16", 128, 8, 2, S=4, W=16, D=0, K=40, hidden=64)
    r = run_prefill_attention(w, 300)
    ws = torch.empty(r.cache.prefill_attention_workspace_bytes(300), dtype=torch.uint8, device="cuda")
    out_full = torch.empty_like(r.q)
    lse_full = torch.empty_like(r.lse)
    r.cache.prefill_attention(0, r.q, r.k, r.v, out_full, lse_full, ws)
    out2 = torch.full_like(r.q, float("nan"))
    lse2 = torch.full_like(r.lse, float("nan"))
    r.cache.prefill_attention_from_cutoffs(0, r.q, r.k, r.v, out2, lse2, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_full, out2) and torch.equal(lse_full, lse2)
    q2 = wl.prompt_queries(w, 0, 300, master=5).cuda()
    r.cache.prefill_attention_from_cutoffs(0, q2, r.k, r.v, out2, lse2, ws)
    torch.cuda.synchronize()
    r.q, r.out, r.lse = q2, out2, lse2
    check_all_rows(r)


def test_repeat_call_is_deterministic_and_leaves_cache_alone():
    """Two calls give identical bits; the cache's position counter is untouched."""
    _need_gpu()
    w = _case("bf16", 128, 8, 2, S=4, W=16, D=0, K=40, hidden=64)
    r = run_prefill_attention(w, 200)
    first = r.out.clone()
    ws = torch.empty(r.cache.prefill_attention_workspace_bytes(200), dtype=torch.uint8, device="cuda")
    r.cache.prefill_attention(0, r.q, r.k, r.v, r.out, r.lse, ws)
    torch.cuda.synchronize()
    assert torch.equal(first, r.out)
    _, _, state = r.cache.inspect(0)
    assert (state[:, 0] == 0).all()


def test_full_size_target_shape_sampled_rows():
    """The 87.5%-compression target shape at full size (64 rows x 8 KV heads,
    prompt 8192, S 4 + W 128 + K 892, G 4, bf16, MLP scorer 64), in the launch
    configuration bench.py times.  Sampled units and positions: the mask each
    position gets from the GPU's cutoffs equals the oracle's attended set, and
    the output row and normaliser match attention over that set."""
    _need_gpu()
    w = wl.QWEN3_4B_CR88.replace(name="pa_full_size", n_layers=1, decode=0)
    n = w.prefill
    r = run_prefill_attention(w, n, gen_device="cuda")
    units = w.batch * w.n_kv_heads
    S, W, D, K = w.sinks, w.window, w.delay, w.topk
    rng = np.random.default_rng(7)
    for unit in (0, units // 2 + 3, units - 1):
        k, v, q, out, lse, s = unit_view(r, unit)
        c = r.cut[unit]
        rows = sorted(set([0, S, S + W, S + W + K + 3, n - 1] + list(rng.integers(0, n, 6))))
        for qp in rows:
            T = orc.running_topk(s, qp, S, W, D, K)
            A = orc.attended_positions(qp, S, W, D, T)
            m = qp - W - D
            gpu_set = sorted(set(range(min(S, qp + 1))) | set(range(max(S, m + 1), qp + 1)) |
                             {j for j in range(S, m + 1) if c[j] > m})
            assert gpu_set == A, (unit, qp)
            o, _ = orc.attention(q[qp], k[A], v[A])
            np.testing.assert_allclose(out[qp], o, rtol=0, atol=gh.BF16_ATOL, err_msg=f"unit {unit} q {qp}")
            np.testing.assert_allclose(lse[qp], orc.attention_lse(q[qp], k[A]), rtol=0, atol=LSE_ATOL["bf16"])
    assert torch.isfinite(r.out).all()


def _fenwick_cutoffs(s, n, S, W, D, K):
    import oracle_pins
    return oracle_pins._fenwick_cutoffs(s, n, S, W, D, K)


def _check_large_unit(r, unit, m_samples, rows, atol):
    """Cutoffs of one unit at a size the brute-force cutoffs cannot reach:
    equal to the pinned Fenwick-tree computation, and at sampled newest-
    eligible positions m the GPU's cutoffs give exactly the oracle's running
    top-k (j kept iff j <= m < c_j); sampled rows against the oracle's
    attention over its attended set."""
    w = r.w
    S, W, D, K = w.sinks, w.window, w.delay, w.topk
    k, v, q, out, lse, s = unit_view(r, unit)
    c = r.cut[unit]
    assert list(c) == _fenwick_cutoffs(s, r.n, S, W, D, K), f"unit {unit}: cutoffs differ from the Fenwick tree"
    for m in m_samples:
        kept = set(orc.running_topk(s, m + W + D, S, W, D, K))
        gpu = {j for j in range(S, m + 1) if c[j] > m}
        assert gpu == kept, (unit, m)
    for qp in rows:
        T = orc.running_topk(s, qp, S, W, D, K)
        A = orc.attended_positions(qp, S, W, D, T)
        o, _ = orc.attention(q[qp], k[A], v[A])
        np.testing.assert_allclose(out[qp], o, rtol=0, atol=atol, err_msg=f"unit {unit} q {qp}")
        if lse is not None:
            np.testing.assert_allclose(lse[qp], orc.attention_lse(q[qp], k[A]), rtol=0, atol=LSE_ATOL[w.dtype])


def test_cutoffs_from_the_register_sort():
    """4097 .. 8192 eligible tokens per unit: cutoff_kernel sorts the 8192
    rank keys with 16 per thread in registers (shuffles between lanes,
    shared memory only for strides of 512 and more).  Two units, 6,000 and
    8,324 prompt tokens (5,868 and 8,192 eligible), bf16 d 128 G 4, the 87.5%
    budget, caller scores with ties: every cutoff equal to the Fenwick tree,
    the running top-k at sampled positions, sampled rows."""
    _need_gpu()
    w = _case("bf16", 128, 8, 2, S=4, W=128, D=0, K=892, hidden=64)
    for n in (6000, 8324):
        r = run_prefill_attention(w, n, external=True, tie_levels=3, gen_device="cuda")
        rng = np.random.default_rng(n)
        m_last = n - 1 - w.window - w.delay
        ms = sorted(set([w.sinks, w.sinks + w.topk - 1, w.sinks + w.topk, m_last] +
                        list(rng.integers(w.sinks, m_last + 1, 4))))
        rows = sorted(set([0, n - 1] + list(rng.integers(0, n, 4))))
        for unit in range(2):
            _check_large_unit(r, unit, ms, rows, gh.BF16_ATOL)


def test_cutoffs_sorted_in_the_workspace():
    """More than 16,384 eligible tokens in a unit: cutoff_kernel sorts the
    rank keys in the caller's workspace instead of shared memory (bitmap
    still in shared memory).  One unit, 17,000 prompt tokens, bf16 d 128 G 4,
    the 87.5% budget (4 + 128 + 892), caller scores with ties."""
    _need_gpu()
    w = _case("bf16", 128, 4, 1, S=4, W=128, D=0, K=892, hidden=64)
    n = 17000
    r = run_prefill_attention(w, n, external=True, tie_levels=3, gen_device="cuda")
    rng = np.random.default_rng(3)
    m_last = n - 1 - w.window - w.delay
    ms = sorted(set([w.sinks, w.sinks + w.topk - 1, w.sinks + w.topk, m_last] +
                    list(rng.integers(w.sinks, m_last + 1, 8))))
    rows = sorted(set([0, n - 1, 16500] + list(rng.integers(0, n, 8))))
    _check_large_unit(r, 0, ms, rows, gh.BF16_ATOL)
    assert torch.isfinite(r.out).all()


def test_cutoffs_with_the_bitmap_in_the_workspace():
    """More than 131,072 eligible tokens in a unit: the sort keys (cutoff_kernel)
    and the walk's position bitmap (walk_kernel) both live in the workspace.  One unit of
    131,594 prompt tokens (131,572 eligible), fp32 d 64 G 2, S 4 + W 16 +
    D 2 + K 300, the library's MLP scorer."""
    _need_gpu()
    w = _case("f32", 64, 2, 1, S=4, W=16, D=2, K=300, hidden=32)
    n = 131072 + 22 + 500
    r = run_prefill_attention(w, n, gen_device="cuda")
    rng = np.random.default_rng(4)
    m_last = n - 1 - w.window - w.delay
    ms = sorted(set([w.sinks, w.sinks + w.topk, 131100, m_last] + list(rng.integers(w.sinks, m_last + 1, 4))))
    rows = sorted(set([0, n - 1, 131090] + list(rng.integers(0, n, 6))))
    _check_large_unit(r, 0, ms, rows, gh.F32_ATOL)
    assert torch.isfinite(r.out).all()


def test_bf16_prompt_above_65535_tokens():
    """A bf16 prompt of 66,236 tokens (one unit, G 4, d 128, S 4 + W 16 + D 2 +
    K 300): past 65,535 positions the tensor-core kernel keeps plain positions
    in its candidate lists and reads the cutoffs for the mask from global
    memory.  Cutoffs against the Fenwick tree and the running top-k at sampled
    positions, and sampled output rows."""
    _need_gpu()
    w = _case("bf16", 128, 4, 1, S=4, W=16, D=2, K=300, hidden=64)
    n = 65536 + 700
    r = run_prefill_attention(w, n, gen_device="cuda")
    rng = np.random.default_rng(5)
    m_last = n - 1 - w.window - w.delay
    ms = sorted(set([w.sinks, w.sinks + w.topk, 65600, m_last] + list(rng.integers(w.sinks, m_last + 1, 3))))
    rows = sorted(set([0, 65534, 65535, 65536, n - 1] + list(rng.integers(0, n, 5))))
    _check_large_unit(r, 0, ms, rows, gh.BF16_ATOL)
    assert torch.isfinite(r.out).all()


def test_full_size_8b_delayed_shape_sampled_rows():
    """The Qwen3-8B delayed-scoring shape at full size (32 rows x 8 KV heads,
    prompt 32768, S 4 + W 256 + D 32 + K 3836, G 4, bf16, MLP scorer): 32,476
    eligible tokens per unit, so every unit's cutoffs are sorted in the
    workspace.  Sampled units: cutoffs against the Fenwick tree and the
    oracle's running top-k at sampled positions, and sampled output rows."""
    _need_gpu()
    w = wl.QWEN3_8B_D32.replace(name="pa_full_size_8b", n_layers=1, decode=0)
    n = w.prefill
    r = run_prefill_attention(w, n, gen_device="cuda")
    units = w.batch * w.n_kv_heads
    rng = np.random.default_rng(8)
    m_last = n - 1 - w.window - w.delay
    for unit in (0, units - 1):
        ms = sorted(set([w.sinks, w.sinks + w.topk, m_last] + list(rng.integers(w.sinks, m_last + 1, 3))))
        rows = sorted(set([0, w.sinks + w.window + w.delay + w.topk + 5, n - 1] + list(rng.integers(0, n, 4))))
        _check_large_unit(r, unit, ms, rows, gh.BF16_ATOL)
    assert torch.isfinite(r.out).all()


def test_argument_errors_enqueue_nothing():
    """Misaligned or missing pointers, a short workspace and a bad layer are
    rejected before any work is enqueued; the output stays untouched."""
    _need_gpu()
    import fixed_budget_kv_kvpop_b200 as kp
    w = _case("bf16", 128, 8, 2, S=4, W=16, D=0, K=40, hidden=64)
    r = run_prefill_attention(w, 64)
    n = 64
    need = r.cache.prefill_attention_workspace_bytes(n)
    out = torch.full_like(r.q, 7.0)
    ws = torch.empty(need + 64, dtype=torch.uint8, device="cuda")
    lib, h = kp.lib, r.cache.handle

    def call(layer=0, q=r.q.data_ptr(), out_p=out.data_ptr(), ws_p=ws.data_ptr(), ws_n=need, n_tok=n):
        return lib.kvpop_prefill_attention(h, layer, q, r.k.data_ptr(), r.v.data_ptr(), n_tok, None, out_p, None,
                                           ws_p, ws_n, None)
    assert call(ws_n=need - 1) == kp.KVPOP_ERR_INVALID_ARG
    assert call(ws_p=ws.data_ptr() + 4) == kp.KVPOP_ERR_INVALID_ARG
    assert call(q=r.q.data_ptr() + 2) == kp.KVPOP_ERR_INVALID_ARG
    assert call(out_p=None) == kp.KVPOP_ERR_INVALID_ARG
    assert call(layer=1) == kp.KVPOP_ERR_INVALID_ARG
    assert call(n_tok=-1) == kp.KVPOP_ERR_INVALID_ARG
    assert call(n_tok=0) == kp.KVPOP_OK
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    assert call() == kp.KVPOP_OK
    torch.cuda.synchronize()
    assert torch.equal(out, r.out)


@pytest.mark.parametrize("dtype,d,hq,hkv,S,W,D,K,hidden,n,external,ties,decay", [
    ("bf16", 128, 8, 2, 4, 16, 0, 40, 64, 300, False, 0, None),
    ("bf16", 128, 8, 2, 2, 12, 3, 30, 64, 257, True, 2, None),
    ("f32", 64, 4, 2, 4, 16, 0, 44, 0, 200, False, 0, None),
    ("bf16", 64, 8, 2, 4, 16, 2, 20, 32, 180, False, 0, -0.05),
    ("bf16", 128, 8, 2, 4, 16, 0, 500, 64, 120, True, 1, None),   # fewer eligible tokens than K
])
def test_fused_prefill_matches_prefill_then_attention(dtype, d, hq, hkv, S, W, D, K, hidden, n, external, ties,
                                                      decay):
    """kvpop_prefill_with_attention (one scoring pass; long-range slots from
    the cutoffs) leaves bit for bit the cache kvpop_prefill builds (slot map,
    scores, rows, counters), returns bit for bit the outputs of
    kvpop_prefill_attention, and the decode steps after it agree bit for bit."""
    _need_gpu()
    w = _case(dtype, d, hq, hkv, S=S, W=W, D=D, K=K, hidden=hidden, batch=2)
    weights = None
    if not external:
        weights = tuple(t.cuda() for t in wl.scorer_weights(w.replace(scorer_hidden=max(hidden, 1))))
    dec = None if decay is None else torch.full((1, hkv), decay, dtype=torch.float32, device="cuda")
    caches = [gh.build_cache(w, 1, external, weights, max_chunk=n, debug=True, log_decay=dec) for _ in range(2)]
    k, v = (t.cuda() for t in wl.prompt_kv(w, 0, n_tokens=n))
    q = wl.prompt_queries(w, 0, n).cuda()
    steps = 3
    ext_all = wl.external_scores(w, 0, n + steps, tie_levels=ties).cuda() if external else None
    ext = ext_all[:, :, :n].contiguous() if external else None
    outs, lses = [], []
    for i, c in enumerate(caches):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((w.batch, w.n_q_heads, n), float("nan"), device="cuda")
        ws = torch.empty(c.prefill_attention_workspace_bytes(n), dtype=torch.uint8, device="cuda")
        if i == 0:
            c.prefill(0, k, v, ext)
            c.prefill_attention(0, q, k, v, out, lse, ws, ext)
        else:
            c.prefill_with_attention(0, q, k, v, out, lse, ws, ext)
        outs.append(out)
        lses.append(lse)
    torch.cuda.synchronize()
    for c in caches:
        st, bits = c.get_error()
        assert st == 0, (st, bits)
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(lses[0], lses[1])
    ia, ib = caches[0].inspect(0), caches[1].inspect(0)
    for xa, xb, what in zip(ia, ib, ("slot map", "scores", "state")):
        assert np.array_equal(xa, xb), what
    assert torch.equal(caches[0].kv_rows(0), caches[1].kv_rows(0))
    # with the MLP scorer some long-range slots must be in use, and they must be ascending
    base = S + W + D
    pos = ia[0].reshape(w.batch * w.n_kv_heads, -1)[:, base:]
    for row in pos:
        kept = [int(x) for x in row if x >= 0]
        assert kept == sorted(kept) and len(kept) == min(K, max(0, n - W - D - S))
    for i in range(steps):
        qd, kn, vn = wl.decode_inputs(w, 0, i)
        qd, kn, vn = qd.cuda(), kn.cuda(), vn.cuda()
        es = ext_all[:, :, n + i].contiguous() if external else None
        res = []
        for c in caches:
            o = torch.empty_like(qd)
            c.decode_step(0, qd, kn, vn, o, es)
            res.append(o)
        torch.cuda.synchronize()
        assert torch.equal(res[0], res[1]), f"decode step {i}"


def test_fused_prefill_rejects_a_used_layer():
    _need_gpu()
    import fixed_budget_kv_kvpop_b200 as kp
    w = _case("bf16", 128, 8, 2, S=4, W=16, D=0, K=40, hidden=64)
    r = run_prefill_attention(w, 64)
    k, v = r.k, r.v
    r.cache.prefill(0, k[:, :, :1].contiguous(), v[:, :, :1].contiguous())   # the layer has seen a token
    ws = torch.empty(r.cache.prefill_attention_workspace_bytes(64), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(r.q)
    with pytest.raises(kp.KVPopError):
        r.cache.prefill_with_attention(0, r.q, k, v, out, None, ws)
