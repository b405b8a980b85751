"""Pins of the CPU oracle against what the KVpop page and plain mathematics fix.

Each pin raises AssertionError on failure.  They are plain functions so that
test_oracle_pins.py runs them and test_oracle_mutations.py can check that a
planted mistake in the oracle makes at least one of them fail.
"""
import json
import math
import os

import numpy as np
import torch

from oracle import kvpop_oracle as orc

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def pin_mlp_hand_example():
    g = _load("mlp_hand_example.json")
    x = orc.head_input(np.array(g["k"]), np.array(g["v"]))
    s = orc.mlp_score(x, np.array(g["w1"]), np.array(g["b1"]), np.array(g["w2"]), g["b2"])
    assert abs(float(s) - g["score"]) < 1e-12, (float(s), g["score"])


def _trace(name):
    g = _load(name)
    S, W, D, K, P = g["S"], g["W"], g["D"], g["K"], g["P"]
    scores = g["scores"]
    st = orc.SlotState(S, W, D, K)
    st.append_chunk(P, scores)
    assert st.slot_pos == g["slot_map_after_prefill"], (st.slot_pos, g["slot_map_after_prefill"])
    for step in g["steps"]:
        q = step["q"]
        st.decode(scores)
        assert st.n_seen == q + 1
        T = orc.running_topk(scores, q, S, W, D, K)
        assert T == step["topk"], (q, T, step["topk"])
        assert orc.attended_positions(q, S, W, D, T) == step["attended"], (q, step["attended"])
        assert st.slot_pos == step["slot_map"], (q, st.slot_pos, step["slot_map"])


def pin_retention_trace_d0():
    _trace("retention_trace_s1_w2_d0_k2.json")


def pin_retention_trace_d1():
    _trace("retention_trace_s1_w2_d1_k1.json")


def pin_prefill_chunk_placement():
    g = _load("prefill_chunk_placement_s1_w1_k2.json")
    for mode in ("chunked", "single"):
        st = orc.SlotState(g["S"], g["W"], g["D"], g["K"])
        for n, expect in zip(g[mode]["chunks"], g[mode]["slot_map_after_chunk"]):
            st.append_chunk(n, g["scores"])
            assert st.slot_pos == expect, (mode, st.slot_pos, expect)
        assert st.topk_positions() == g["topk"]


def _rand_unit(seed, n_tokens, n_steps, G, d, tie_levels=0):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((n_tokens, d))
    v = rng.standard_normal((n_tokens, d))
    q = rng.standard_normal((n_steps, G, d))
    s = rng.standard_normal(n_tokens)
    if tie_levels:
        s = np.floor(s * tie_levels)
    return k, v, q, orc.ranking_score(s)


def pin_dense_when_budget_covers_context():
    """Budget >= context: the output is plain dense attention (torch SDPA, float64)."""
    S, W, D, K, P, n, G, d = 3, 5, 2, 64, 20, 30, 4, 16
    k, v, q, s = _rand_unit(1, P + n, n, G, d)
    res = orc.run_unit(k, v, q, s, S, W, D, K, P)
    for i in range(n):
        t = P + i
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q[i][:, None, :]), torch.tensor(k[None, :t + 1]),
            torch.tensor(v[None, :t + 1])).numpy()[:, 0, :]
        np.testing.assert_allclose(res.outputs[i], ref, rtol=1e-10, atol=1e-12)


def pin_budget_invariant_and_structure():
    """|sinks| + |window + staging| + |top-k| = B + D once the context is long enough;
    sinks are always kept; the recent block is exactly the last W + D positions;
    an evicted token never comes back; the long-range set is the brute-force top-K."""
    for (S, W, D, K) in [(4, 16, 0, 44), (2, 5, 3, 7), (0, 3, 0, 4), (1, 1, 0, 3)]:
        P, n = 40, 60
        k, v, q, s = _rand_unit(S * 100 + W, P + n, n, 2, 8, tie_levels=3)
        res = orc.run_unit(k, v, q, s, S, W, D, K, P)
        evicted = set()
        for i in range(n):
            t = P + i
            T = res.topk_sets[i + 1]
            A = orc.attended_positions(t, S, W, D, T)
            assert len(A) == res.attended_counts[i]
            if t + 1 >= S + W + D + K:
                assert len(A) == S + W + D + K, (S, W, D, K, t, len(A))
            assert set(range(min(S, t + 1))) <= set(A)
            recent = [j for j in A if j >= t - W - D + 1 and j >= S]
            assert recent == list(range(max(S, t - W - D + 1), t + 1))
            elig = list(range(S, max(S, t - W - D + 1)))
            assert set(T) <= set(elig) and len(T) == min(K, len(elig))
            # brute force over every subset size: T is the set of the K best keys
            if T:
                worst_kept = min(orc.rank_key(s[j], j) for j in T)
                for j in elig:
                    if j not in T:
                        assert orc.rank_key(s[j], j) < worst_kept
            assert not (set(T) & evicted), "evicted token came back"
            prev = res.topk_sets[i]
            evicted |= set(prev) - set(T)


def pin_softmax_rows_sum_to_one():
    k, v, q, s = _rand_unit(7, 50, 20, 3, 8)
    res = orc.run_unit(k, v, q, s, 2, 4, 0, 6, 30)
    np.testing.assert_allclose(res.weight_sums, 1.0, rtol=0, atol=1e-12)


def pin_delay_equivalence():
    """Stateless scorer: (W, D) behaves as (W + D, 0) with the same K; D = 0 is immediate."""
    S, W, D, K, P, n, G, d = 2, 4, 3, 5, 25, 25, 2, 8
    k, v, q, s = _rand_unit(11, P + n, n, G, d, tie_levels=2)
    a = orc.run_unit(k, v, q, s, S, W, D, K, P)
    b = orc.run_unit(k, v, q, s, S, W + D, 0, K, P)
    np.testing.assert_allclose(a.outputs, b.outputs, rtol=0, atol=1e-14)
    assert a.topk_sets == b.topk_sets


def pin_prefill_is_running_topk():
    """Prefill of P tokens equals prefill of P - m tokens followed by m decode steps."""
    S, W, D, K, G, d = 3, 4, 0, 6, 2, 8
    P, n, m = 30, 10, 7
    k, v, q, s = _rand_unit(5, P + n, n + m, G, d, tie_levels=3)
    a = orc.run_unit(k, v, q[m:], s, S, W, D, K, P)
    b = orc.run_unit(k, v, q, s, S, W, D, K, P - m)
    assert a.topk_sets == b.topk_sets[m:]
    np.testing.assert_allclose(a.outputs, b.outputs[m:], rtol=0, atol=1e-14)


def pin_attention_closed_forms():
    d = 4
    keys = np.array([[1.0, 0, 0, 0], [1.0, 0, 0, 0], [0, 1.0, 0, 0]])
    vals = np.array([[1.0, 2, 3, 4], [3.0, 2, 1, 0], [0, 0, 0, 8]])
    # equal logits on all keys -> mean of the values
    q = np.zeros((1, d))
    o, w = orc.attention(q, keys, vals)
    np.testing.assert_allclose(o[0], vals.mean(axis=0), atol=1e-15)
    # logits (q.k)/sqrt(d): q = [2 ln 3, 0, 0, 0] * sqrt(d)/2 -> keys 0,1 get ln 3, key 2 gets 0
    q = np.array([[math.log(3.0) * math.sqrt(d), 0, 0, 0]])
    o, w = orc.attention(q, keys, vals)
    np.testing.assert_allclose(w[0], [3 / 7, 3 / 7, 1 / 7], atol=1e-15)
    np.testing.assert_allclose(o[0], (3 * vals[0] + 3 * vals[1] + vals[2]) / 7, atol=1e-14)


def pin_decay_hand_example():
    """§B.3 decay, hand-derived: S=0, W=1, D=0, K=1, every score 0.  Token j
    becomes eligible at step j + 1 with priority (j + 1) / 8 for
    ln gamma = -1/8, so the newest eligible token always wins; without decay
    the scores tie and the oldest token stays.  Priorities of [1, .5, .5] at
    W=2, D=1, ln gamma = -1/4: 1 + 3/4, 1/2 + 4/4, 1/2 + 5/4."""
    pr = orc.decayed_priority([1.0, 0.5, 0.5], 2, 1, -0.25)
    assert list(pr) == [1.75, 1.5, 1.75], list(pr)
    n = 12
    zeros = [0.0] * n
    dec = orc.decayed_priority(zeros, 1, 0, -0.125)
    assert list(dec) == [(j + 1) / 8 for j in range(n)], list(dec)
    for q in range(1, n):
        assert orc.running_topk(dec, q, 0, 1, 0, 1) == [q - 1]
        assert orc.running_topk(zeros, q, 0, 1, 0, 1) == [0]
    # ln gamma = 0 leaves the scores as they are
    sc = orc.ranking_score(np.random.default_rng(3).standard_normal(50))
    assert np.array_equal(orc.decayed_priority(sc, 5, 2, 0.0), sc)


def pin_decay_static_priority_is_effective_score_topk():
    """The static priority ranks like the effective score at every step: the
    top-K of eff_q(j) = s_j + (q - e_j) ln gamma, computed exactly for each q
    by brute force, equals the top-K of the priorities, and the slot
    simulator (incremental argmin-replace) keeps that same set."""
    rng = np.random.default_rng(11)
    S, W, D, K, n = 2, 3, 1, 4, 60
    lg = float(np.float32(-0.07))
    sc = orc.ranking_score(rng.standard_normal(n))
    pr = orc.decayed_priority(sc, W, D, lg)
    st = orc.SlotState(S, W, D, K)
    st.append_chunk(S + W + D + 1, pr)   # holds tokens 0..q for q = S + W + D
    for q in range(S + W + D, n):
        if q > S + W + D:
            st.decode(pr)
        elig = list(orc.eligible_positions(q, S, W, D))
        brute = sorted(elig, key=lambda j: (orc.effective_score(sc[j], j, q, W, D, lg), -j), reverse=True)[:K]
        assert sorted(brute) == orc.running_topk(pr, q, S, W, D, K), q
        assert sorted(brute) == st.topk_positions(), q


def pin_float32_single_rounding():
    """Priorities are rounded once to float32 from the exact value: ties go
    to even, and a value just above a halfway point rounds up even where a
    detour through float64 would land on the tie and round down."""
    from fractions import Fraction
    rng = np.random.default_rng(5)
    for x in rng.standard_normal(500) * 1e3:
        assert orc.round_to_float32(float(x)) == float(np.float32(x))
    one = Fraction(1)
    assert orc.round_to_float32(one + Fraction(1, 2 ** 24)) == 1.0
    assert orc.round_to_float32(one + Fraction(3, 2 ** 24)) == 1.0 + 2.0 ** -22
    assert orc.round_to_float32(one + Fraction(1, 2 ** 24) + Fraction(1, 2 ** 80)) == 1.0 + 2.0 ** -23
    assert orc.round_to_float32(-(one + Fraction(1, 2 ** 24) + Fraction(1, 2 ** 80))) == -(1.0 + 2.0 ** -23)


def pin_linear_scorer():
    """§E.2 linear scorer: a hand example (x = [k; v] = [1, 2, -1, 0.5],
    w = [0.5, -0.25, 2, 4], b = 0.125: 0.5 - 0.5 - 2 + 2 + 0.125), and the
    identity relu(t) - relu(-t) = t: an MLP with hidden rows [w; -w],
    w2 = [1, -1], b1 = 0 is the linear scorer w . x + b2."""
    s = orc.linear_score(orc.head_input(np.array([1.0, 2.0]), np.array([-1.0, 0.5])),
                         np.array([0.5, -0.25, 2.0, 4.0]), 0.125)
    assert float(s) == 0.125, float(s)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((20, 8))
    w = rng.standard_normal(8)
    mlp = orc.mlp_score(x, np.stack([w, -w]), np.zeros(2), np.array([1.0, -1.0]), 0.3)
    assert np.allclose(mlp, orc.linear_score(x, w, 0.3), rtol=0, atol=1e-12)



# ---------------------------------------------------------------------------
# Parallel sparse prefill attention (§C.1 Mask Definition, §C.2 Fenwick-Tree
# Cutoff Computation)
# ---------------------------------------------------------------------------

def pin_prefill_mask_hand_example():
    """Hand-derived cutoffs and attended sets; with zero queries and one-hot
    values the prefill output of row q is the indicator of its attended set
    divided by its size, and the log-normaliser is log |A_q|."""
    g = _load("prefill_mask_s1_w1_d0_k1.json")
    S, W, D, K, s = g["S"], g["W"], g["D"], g["K"], g["scores"]
    n = len(s)
    assert orc.running_cutoffs(s, n, S, W, D, K) == g["cutoffs"]
    for q in range(n):
        T = orc.running_topk(s, q, S, W, D, K)
        assert orc.attended_positions(q, S, W, D, T) == g["attended"][q], q
    out, lse, counts = orc.prefill_attention(np.zeros((n, 1, n)), np.zeros((n, n)), np.eye(n), s, S, W, D, K)
    for q in range(n):
        A = g["attended"][q]
        expect = np.zeros(n)
        expect[A] = 1.0 / len(A)
        np.testing.assert_allclose(out[q, 0], expect, rtol=0, atol=1e-15)
        assert abs(lse[q, 0] - math.log(len(A))) < 1e-14
        assert counts[q] == len(A)


def _fenwick_cutoffs(scores, n, S, W, D, K):
    """The tree method of §C.2, written independently of the oracle: visit the
    eligible tokens best first (score, then older first; NaN lowest); before
    inserting token j, the K-th smallest position among the tokens already in
    a Fenwick tree over positions (those ranked above j) is the step at which
    j leaves the long-range set; fewer than K above it means it never leaves."""
    c = [-1] * n
    elig = list(range(S, n - W - D))
    tree = [0] * (n + 1)

    def add(i):
        i += 1
        while i <= n:
            tree[i] += 1
            i += i & -i

    def kth(k):
        pos, rem, step = 0, k, 1 << n.bit_length()
        while step:
            if pos + step <= n and tree[pos + step] < rem:
                pos += step
                rem -= tree[pos]
            step >>= 1
        return pos

    def key(j):
        x = float(scores[j])
        return (-math.inf if math.isnan(x) else x, -j)

    for r, j in enumerate(sorted(elig, key=key, reverse=True)):
        if r < K:
            c[j] = 2 ** 31 - 1
        else:
            c[j] = max(j, kth(K)) if K > 0 else j
        add(j)
    return c


def pin_running_cutoffs_match_fenwick():
    for i, (S, W, D, K, n, ties) in enumerate([(2, 3, 0, 4, 40, 3), (0, 1, 0, 1, 30, 2), (1, 2, 2, 5, 45, 0),
                                               (3, 4, 1, 0, 20, 2), (1, 1, 0, 50, 30, 0), (0, 2, 0, 3, 25, 1),
                                               (4, 2, 3, 6, 12, 0)]):
        _, _, _, s = _rand_unit(100 + i, n, 0, 1, 2, tie_levels=ties)
        assert orc.running_cutoffs(s, n, S, W, D, K) == _fenwick_cutoffs(s, n, S, W, D, K), (S, W, D, K)


def pin_running_cutoffs_are_intervals():
    """Token j is in the running top-k at newest-eligible position m exactly when
    j <= m < c_j (an evicted token never returns, §C.2)."""
    S, W, D, K, n = 2, 3, 1, 4, 36
    _, _, _, s = _rand_unit(21, n, 0, 1, 2, tie_levels=2)
    c = orc.running_cutoffs(s, n, S, W, D, K)
    for m in range(S, n - W - D):
        kept = set(orc.running_topk(s, m + W + D, S, W, D, K))
        for j in range(S, n - W - D):
            assert (j in kept) == (j <= m < c[j]), (m, j, c[j])


def pin_prefill_attention_dense_when_budget_covers_context():
    """K >= n: every row is causal dense attention (torch SDPA, float64) and its
    log-normaliser is torch.logsumexp of the causal logits."""
    S, W, D, K, n, G, d = 2, 3, 1, 64, 40, 2, 8
    rng = np.random.default_rng(3)
    k, v = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    q = rng.standard_normal((n, G, d))
    s = orc.ranking_score(rng.standard_normal(n))
    out, lse, _ = orc.prefill_attention(q, k, v, s, S, W, D, K)
    qt = torch.tensor(q).permute(1, 0, 2)  # [G][n][d]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, torch.tensor(k)[None], torch.tensor(v)[None],
                                                           is_causal=True)
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    logits = (qt @ torch.tensor(k).T) / math.sqrt(d)
    logits = logits.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(logits, -1).T.numpy(), rtol=1e-12, atol=1e-12)


def pin_prefill_attention_matches_slot_simulator():
    """Row q equals attention over the slot simulator's whole cache content after
    token q arrives one token at a time (sinks, window, staging, long-range slots),
    and it attends to min(q + 1, S + W + D + K) tokens."""
    for (S, W, D, K, n) in [(2, 4, 0, 5, 40), (1, 3, 2, 4, 36), (0, 2, 0, 3, 30)]:
        G, d = 2, 8
        k, v, qq, s = _rand_unit(S * 10 + W + D, n, n, G, d, tie_levels=3)
        out, lse, counts = orc.prefill_attention(qq, k, v, s, S, W, D, K)
        st = orc.SlotState(S, W, D, K)
        for q in range(n):
            st.decode(s)
            A = sorted(p for p in st.slot_pos if p >= 0)
            assert counts[q] == len(A) == min(q + 1, S + W + D + K), (q, counts[q], len(A))
            o, w = orc.attention(qq[q], k[A], v[A])
            np.testing.assert_allclose(out[q], o, rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# Stateful mLSTM scorer with delayed readout (§A, §E.3, §E.4)
# ---------------------------------------------------------------------------

def _mlstm_params(seed, d, p, dv, bi, bf):
    rng = np.random.default_rng(seed)
    return orc.MlstmParams(wq=rng.normal(size=(p, 2 * d)) * 0.7, wk=rng.normal(size=(p, 2 * d)) * 0.7,
                           wv=rng.normal(size=(dv, 2 * d)), wi=rng.normal(size=2 * d) * 0.3, bi=bi,
                           wf=rng.normal(size=2 * d) * 0.3, bf=bf, wo=rng.normal(size=dv), bo=0.1)


def pin_hedgehog_feature_map():
    """[softmax(z); softmax(-z)] as torch.softmax computes it; each half sums
    to 1; negating z swaps the halves."""
    z = np.random.default_rng(5).normal(size=(6, 7)) * 3.0
    phi = orc.hedgehog(z)
    zt = torch.tensor(z)
    ref = torch.cat([torch.softmax(zt, -1), torch.softmax(-zt, -1)], -1).numpy()
    np.testing.assert_allclose(phi, ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(phi[:, :7].sum(-1), 1.0, atol=1e-14)
    np.testing.assert_allclose(orc.hedgehog(-z), np.concatenate([phi[:, 7:], phi[:, :7]], -1), atol=1e-15)


def pin_mlstm_stabilised_equals_closed_form():
    """The stabilised recurrence reads out what the closed form of the gated
    outer-product sum gives (§A: recurrent and parallel forms agree): with
    g_t = exp(i~_t) * prod_{s=t+1..q} sigmoid(f~_s), C = sum_t g_t v_t phi_t^T,
    n = sum_t g_t phi_t and h = C r / max(|n . r|, 1).  A strongly negative
    input bias drives |n . r| below 1 so that the floor is exercised."""
    d, p, dv, n = 3, 4, 2, 18
    floor_used = False
    for seed, (bi, bf) in enumerate([(-4.0, 1.0), (0.5, -0.5), (3.0, 2.0)]):
        P = _mlstm_params(40 + seed, d, p, dv, bi, bf)
        x = np.random.default_rng(60 + seed).normal(size=(n, 2 * d))
        states = orc.mlstm_states(x, P)
        ig = [math.exp(float(P.wi @ xt) + P.bi) for xt in x]
        fg = [1.0 / (1.0 + math.exp(-(float(P.wf @ xt) + P.bf))) for xt in x]
        rr = np.random.default_rng(80 + seed).normal(size=(n, 2 * d))
        for q in range(n):
            C = np.zeros((dv, 2 * p))
            nn = np.zeros(2 * p)
            for t in range(q + 1):
                g = ig[t] * math.prod(fg[t + 1:q + 1])
                phi = orc.hedgehog(P.wk @ x[t])
                C += g * np.outer(P.wv @ x[t], phi)
                nn += g * phi
            r = orc.hedgehog(P.wq @ rr[q])
            den = abs(float(nn @ r))
            floor_used |= den < 1.0
            h_ref = (C @ r) / max(den, 1.0)
            np.testing.assert_allclose(orc.mlstm_readout(*states[q], r), h_ref, rtol=1e-10, atol=1e-12)
    assert floor_used


def pin_mlstm_delayed_readout_is_causal_and_forward_looking():
    """The score of token u (eligible at q = u + W + D) does not change when a
    later token changes, and does change when token q changes: the state it is
    read from has processed exactly the tokens through q (§E.4)."""
    S, W, D, d, n = 2, 4, 1, 3, 30
    P = _mlstm_params(7, d, 4, 2, 0.0, 1.0)
    rng = np.random.default_rng(9)
    k, v = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    s = orc.unit_scores_mlstm(k, v, P, S, W, D)
    assert np.isnan(s[:S]).all() and np.isnan(s[n - W - D:]).all() and np.isfinite(s[S:n - W - D]).all()
    u = 10
    q = u + W + D
    k2 = k.copy()
    k2[q + 1] += 5.0
    s2 = orc.unit_scores_mlstm(k2, v, P, S, W, D)
    np.testing.assert_array_equal(s2[:q + 1 - W - D], s[:q + 1 - W - D])
    k3 = k.copy()
    k3[q] += 5.0
    s3 = orc.unit_scores_mlstm(k3, v, P, S, W, D)
    assert s3[u] != s[u]
    np.testing.assert_array_equal(s3[:u], s[:u])


def pin_mlstm_scores_drive_the_running_topk():
    """Scores fixed at eligibility plug into the retention rule unchanged: the
    slot simulator holds the brute-force top-k at every decode step."""
    S, W, D, K, d, P_len, steps = 2, 4, 2, 5, 3, 20, 15
    P = _mlstm_params(11, d, 4, 2, 0.0, 1.0)
    rng = np.random.default_rng(12)
    n = P_len + steps
    k, v = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    q = rng.normal(size=(steps, 2, d))
    s = orc.unit_scores_mlstm(k, v, P, S, W, D)
    res = orc.run_unit(k, v, q, s, S, W, D, K, P_len)
    assert all(len(t) == min(K, max(0, P_len + i - W - D - S + 1)) for i, t in enumerate(res.topk_sets[1:]))


def pin_mlstm_readout_hand_example():
    """A hand-worked delayed readout (golden/mlstm_readout_hand_example.json):
    with one-dimensional Hedgehog projections every feature vector is [1, 1],
    so the readout h is a decayed average of the values and the score head
    w_o . SiLU(h) + b_o can be checked by eye (§E.4 Delayed Readout)."""
    g = _load("mlstm_readout_hand_example.json")
    P = orc.MlstmParams(wq=np.array(g["wq"]), wk=np.array(g["wk"]), wv=np.array(g["wv"]), wi=np.array(g["wi"]),
                        bi=g["bi"], wf=np.array(g["wf"]), bf=g["bf"], wo=np.array(g["wo"]), bo=g["bo"])
    k = np.array(g["k"])[:, None]
    v = np.array(g["v"])[:, None]
    x = orc.head_input(k, v)
    states = orc.mlstm_states(x, P)
    for u, h_ref in enumerate(g["h"]):
        q = u + g["W"] + g["D"]
        h = orc.mlstm_readout(*states[q], orc.hedgehog(P.wq @ x[u]))
        np.testing.assert_allclose(h, h_ref, rtol=0, atol=1e-12)
    s = orc.unit_scores_mlstm(k, v, P, g["S"], g["W"], g["D"])
    for u, ref in enumerate(g["scores"]):
        if ref is None:
            assert math.isnan(s[u]), (u, s[u])
        else:
            assert s[u] == float(np.float32(ref)), (u, s[u], ref)

ALL_PINS = [pin_mlp_hand_example, pin_retention_trace_d0, pin_retention_trace_d1,
            pin_prefill_chunk_placement, pin_dense_when_budget_covers_context,
            pin_budget_invariant_and_structure, pin_softmax_rows_sum_to_one,
            pin_delay_equivalence, pin_prefill_is_running_topk, pin_attention_closed_forms,
            pin_decay_hand_example, pin_decay_static_priority_is_effective_score_topk,
            pin_float32_single_rounding, pin_linear_scorer,
            pin_prefill_mask_hand_example, pin_running_cutoffs_match_fenwick,
            pin_running_cutoffs_are_intervals, pin_prefill_attention_dense_when_budget_covers_context,
            pin_prefill_attention_matches_slot_simulator, pin_hedgehog_feature_map,
            pin_mlstm_stabilised_equals_closed_form, pin_mlstm_delayed_readout_is_causal_and_forward_looking,
            pin_mlstm_scores_drive_the_running_topk, pin_mlstm_readout_hand_example]
