"""Planted mistakes in the CPU oracle must make at least one pin fail.

Each case monkeypatches one oracle function with a plausible slip (a dropped
term, a wrong sign or index, a swapped operand) and runs every pin; the case
passes only if some pin raises.  This is what makes the pins evidence.
"""
import math

import numpy as np
import pytest

import oracle_pins as pins
from oracle import kvpop_oracle as orc


def _ties_to_newer(score, pos):
    s = float(score)
    return (s, int(pos))


def _elig_off_by_one(q, S, W, D):
    return range(S, max(S, q - W - D + 2))


def _no_scale(q, keys, values):
    q = np.asarray(q, np.float64)
    logits = q @ np.asarray(keys, np.float64).T
    logits -= logits.max(axis=-1, keepdims=True)
    w = np.exp(logits)
    w /= w.sum(axis=-1, keepdims=True)
    return w @ np.asarray(values, np.float64), w


def _vk_order(k, v):
    return np.concatenate([np.asarray(v, np.float64), np.asarray(k, np.float64)], axis=-1)


def _drop_b1(x, w1, b1, w2, b2):
    h = np.maximum(np.asarray(x, np.float64) @ np.asarray(w1).T, 0.0)
    return h @ np.asarray(w2) + float(b2)


def _drop_b2(x, w1, b1, w2, b2):
    h = np.maximum(np.asarray(x, np.float64) @ np.asarray(w1).T + np.asarray(b1), 0.0)
    return h @ np.asarray(w2)


def _no_relu(x, w1, b1, w2, b2):
    h = np.asarray(x, np.float64) @ np.asarray(w1).T + np.asarray(b1)
    return h @ np.asarray(w2) + float(b2)


def _recent_without_current(q, S, W, D):
    return list(range(max(S, q - W - D + 1), q))


def _recent_ignores_staging(q, S, W, D):
    return list(range(max(S, q - W + 1), q + 1))


def _topk_keeps_lowest(scores, q, S, W, D, K):
    elig = list(orc.eligible_positions(q, S, W, D))
    ranked = sorted(elig, key=lambda j: orc.rank_key(scores[j], j))
    return sorted(ranked[:K])


def _topk_keeps_k_minus_1(scores, q, S, W, D, K):
    elig = list(orc.eligible_positions(q, S, W, D))
    ranked = sorted(elig, key=lambda j: orc.rank_key(scores[j], j), reverse=True)
    return sorted(ranked[:max(K - 1, 0)])


def _sinks_off_by_one(q, S):
    return list(range(0, min(S - 1, q + 1)))


def _softmax_without_max_shift_wrong_norm(q, keys, values):
    q = np.asarray(q, np.float64)
    logits = (q @ np.asarray(keys, np.float64).T) / math.sqrt(q.shape[-1])
    w = np.exp(logits)
    w /= w.shape[-1]
    return w @ np.asarray(values, np.float64), w


def _window_slot_wrong(self, t):
    return self.S + ((t + 1) % self.W)


def _decay_sign_flipped(scores, W, D, log_gamma):
    from fractions import Fraction
    lg = Fraction(float(np.float32(log_gamma)))
    return np.array([orc.round_to_float32(Fraction(float(s)) + (j + W + D) * lg) for j, s in enumerate(scores)])


def _decay_eligibility_off_by_one(scores, W, D, log_gamma):
    from fractions import Fraction
    lg = Fraction(float(np.float32(log_gamma)))
    return np.array([orc.round_to_float32(Fraction(float(s)) - (j + W + D - 1) * lg) for j, s in enumerate(scores)])


def _round_via_float64(x):
    return float(np.float32(float(x)))


def _linear_drops_bias(x, w, b):
    return np.asarray(x, np.float64) @ np.asarray(w, np.float64)


def _cutoff_last_kept(scores, n, S, W, D, K):
    c = _ORIG_CUTOFFS(scores, n, S, W, D, K)
    return [x - 1 if 0 <= x < 2 ** 31 - 1 else x for x in c]


def _prefill_stale_topk(q_all, k_all, v_all, scores, S, W, D, K):
    n = len(k_all)
    G, d = q_all.shape[1], q_all.shape[2]
    out, lse, counts = np.zeros((n, G, d)), np.zeros((n, G)), []
    for q in range(n):
        T = orc.running_topk(scores, max(q - 1, 0), S, W, D, K)
        A = orc.attended_positions(q, S, W, D, T)
        out[q] = orc.attention(q_all[q], k_all[A], v_all[A])[0]
        lse[q] = orc.attention_lse(q_all[q], k_all[A])
        counts.append(len(A))
    return out, lse, counts


def _lse_unscaled(q, keys):
    logits = np.asarray(q, np.float64) @ np.asarray(keys, np.float64).T
    mx = logits.max(axis=-1)
    return mx + np.log(np.exp(logits - mx[:, None]).sum(axis=-1))


_ORIG_CUTOFFS = orc.running_cutoffs


def _hedgehog_positive_only(z):
    z = np.asarray(z, np.float64)
    a = np.exp(z - z.max(axis=-1, keepdims=True))
    a = a / a.sum(axis=-1, keepdims=True)
    return np.concatenate([a, a], axis=-1)


def _mlstm_forget_not_log(x_all, P):
    x_all = np.asarray(x_all, np.float64)
    dv, f2 = P.wv.shape[0], 2 * P.wk.shape[0]
    C, nv, m = np.zeros((dv, f2)), np.zeros(f2), 0.0
    out = []
    for x in x_all:
        phi = orc.hedgehog(P.wk @ x)
        it = float(P.wi @ x) + P.bi
        f = 1.0 / (1.0 + math.exp(-(float(P.wf @ x) + P.bf)))
        m_new = max(f + m, it)
        ip, fp = math.exp(it - m_new), math.exp(f + m - m_new)
        C = fp * C + ip * np.outer(P.wv @ x, phi)
        nv = fp * nv + ip * phi
        m = m_new
        out.append((C.copy(), nv.copy(), m))
    return out


def _mlstm_readout_no_floor(C, nv, m, r):
    return (C @ r) / abs(float(nv @ r))


def _mlstm_not_delayed(k_all, v_all, P, S, W, D):
    x_all = orc.head_input(k_all, v_all)
    n = len(x_all)
    states = orc.mlstm_states(x_all, P)
    s = np.full(n, np.nan)
    for u in range(S, n):
        if u + W + D >= n:
            break
        C, nv, m = states[u]
        s[u] = float(P.wo @ orc.silu(orc.mlstm_readout(C, nv, m, orc.hedgehog(P.wq @ x_all[u])))) + P.bo
    return orc.ranking_score(s)


def _sigmoid_for_silu(x):
    x = np.asarray(x, np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def _identity_for_silu(x):
    return np.asarray(x, np.float64)


def _mlstm_score_drops_bias(k_all, v_all, P, S, W, D):
    import dataclasses
    return _ORIG_MLSTM_SCORES(k_all, v_all, dataclasses.replace(P, bo=0.0), S, W, D)


_ORIG_MLSTM_SCORES = orc.unit_scores_mlstm


MUTATIONS = {
    "tie_goes_to_newer": ("rank_key", _ties_to_newer),
    "eligible_off_by_one": ("eligible_positions", _elig_off_by_one),
    "attention_no_scale": ("attention", _no_scale),
    "scorer_input_v_then_k": ("head_input", _vk_order),
    "scorer_drops_b1": ("mlp_score", _drop_b1),
    "scorer_drops_b2": ("mlp_score", _drop_b2),
    "scorer_no_relu": ("mlp_score", _no_relu),
    "recent_excludes_current": ("recent_positions", _recent_without_current),
    "recent_ignores_staging": ("recent_positions", _recent_ignores_staging),
    "topk_keeps_lowest": ("running_topk", _topk_keeps_lowest),
    "topk_keeps_k_minus_1": ("running_topk", _topk_keeps_k_minus_1),
    "sinks_off_by_one": ("sink_positions", _sinks_off_by_one),
    "softmax_wrong_normaliser": ("attention", _softmax_without_max_shift_wrong_norm),
    "decay_sign_flipped": ("decayed_priority", _decay_sign_flipped),
    "decay_eligibility_off_by_one": ("decayed_priority", _decay_eligibility_off_by_one),
    "priority_double_rounding": ("round_to_float32", _round_via_float64),
    "linear_drops_bias": ("linear_score", _linear_drops_bias),
    "cutoff_records_last_kept_step": ("running_cutoffs", _cutoff_last_kept),
    "prefill_attends_before_update": ("prefill_attention", _prefill_stale_topk),
    "prefill_lse_unscaled": ("attention_lse", _lse_unscaled),
    "hedgehog_positive_only": ("hedgehog", _hedgehog_positive_only),
    "mlstm_forget_gate_not_in_log_space": ("mlstm_states", _mlstm_forget_not_log),
    "mlstm_normaliser_without_floor": ("mlstm_readout", _mlstm_readout_no_floor),
    "mlstm_readout_not_delayed": ("unit_scores_mlstm", _mlstm_not_delayed),
    "mlstm_score_head_sigmoid_for_silu": ("silu", _sigmoid_for_silu),
    "mlstm_score_head_identity_for_silu": ("silu", _identity_for_silu),
    "mlstm_score_head_drops_bias": ("unit_scores_mlstm", _mlstm_score_drops_bias),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(orc, attr, fn)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError, ZeroDivisionError):
            failed.append(pin.__name__)
    assert failed, f"mutation {name} passed every pin"


def test_slot_placement_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(orc.SlotState, "window_slot", _window_slot_wrong)
    with pytest.raises(AssertionError):
        pins.pin_retention_trace_d0()
