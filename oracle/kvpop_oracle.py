"""Plain CPU oracle for KVpop's decode-time hot path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module: it
is used by tests/, by __graft_entry__.smoke() and by the cpu_baseline leg of
bench.py.  It shares no code with the CUDA library (it does not import the
package, its kernels, or its binding).

Source: "KVpop -- Key-Value Cache Compression with Predictive Online Pruning"
(paperlayer.ai summary page of arXiv 2607.05061v2).  Each function names the
section it follows.  Everything is float64 numpy unless stated; ranking
decisions use float32 scores, because the page's §F (Experiment Details,
training setup) states that top-k ranking/selection runs in float32.

Readings of points the page leaves open (each one is also listed in the
design notes):

* Total order on tokens (tie rule): key(j) = (s_j, -j).  A higher score ranks
  higher; on equal scores the older token ranks higher.  A newcomer replaces
  the current minimum only if its key is strictly larger.  NaN scores rank as
  -inf; -0.0 equals +0.0.
* Window = the W most recent positions {q-W+1 .. q} (current token included),
  positions >= S only.  The token u = q - W leaves the window at q (§E.4
  Delayed Readout: "newly eligible token is u = q - w").
* Delay D > 0: a D-slot staging ring between window and the eligible region.
  Staged tokens stay in the cache and are attended (§E.1: keys and values
  remain cached until the eviction decision); they sit outside B = S+W+K.
  The eligible set at q is {S <= j <= q - W - D}.
* Update before attend: the query at position q attends to its own token and
  to the set decided at q (§C.1 Mask Definition / §I Pseudocode: past tokens
  that are sinks, recent, eligible and selected).
* Attention scale 1/sqrt(d).  Scorer input x = [k; v] (§E.1), MLP
  s = w2 . relu(W1 x + b1) + b2 (§E.2 stateless headwise MLP scorer).
* Slot placement (needed only to compare slot maps): a prefill chunk keeps the
  surviving long-range tokens in their slots and gives the admitted newcomers,
  in ascending position, the free-or-vacated top-k slots in ascending slot
  order; one decode step is the one-newcomer case (next free slot, else the
  slot of the evicted minimum).  Window slot of token t: S + (t mod W);
  staging slot: S + W + (t mod D); sink slot: t.
* Temporal decay (optional, §B.3): log-space, ranking by the static priority
  p_j = s_j - (j + W + D) ln gamma_h in float32 (see decayed_priority).
* Parallel prefill attention (§C.1, §C.2): every prompt position q attends to
  the set a decode step at q would attend to.  Running cutoff of token j: with
  m = q - W - D, j is kept exactly for m in [j, c_j) (see running_cutoffs).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np

NEG_INF = float("-inf")


# ---------------------------------------------------------------------------
# Scorer (§E.1 Headwise Inputs, §E.2 Stateless Linear and MLP Scorers)
# ---------------------------------------------------------------------------

def head_input(k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """x = [k; v]: the scorer sees only cached quantities of the KV head (§E.1)."""
    return np.concatenate([np.asarray(k, np.float64), np.asarray(v, np.float64)], axis=-1)


def mlp_score(x: np.ndarray, w1: np.ndarray, b1: np.ndarray, w2: np.ndarray, b2: float) -> np.ndarray:
    """Stateless headwise MLP score s = w2 . relu(W1 x + b1) + b2, float64 (§E.2).

    x: [..., 2d]; w1: [hidden, 2d]; b1: [hidden]; w2: [hidden]; b2: scalar.
    """
    x = np.asarray(x, np.float64)
    hidden = np.maximum(x @ np.asarray(w1, np.float64).T + np.asarray(b1, np.float64), 0.0)
    return hidden @ np.asarray(w2, np.float64) + float(b2)


def ranking_score(s) -> np.ndarray:
    """Round scores to float32, the precision of top-k ranking (§F)."""
    return np.asarray(s, np.float64).astype(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Temporal decay (§B.3 Temporal Decay and Static Priorities; teacher policy)
# ---------------------------------------------------------------------------
#
# The page gives shared per-head decay factors 0 < gamma_h < 1 on effective
# scores (a recency bias) and names the equivalent "static priorities", but no
# formula.  Reading: log-space decay.  Token j becomes eligible at step
# e_j = j + W + D; at step q >= e_j its effective score is
#     eff_q(j) = s_j + (q - e_j) * ln gamma_h,
# and since q * ln gamma_h is common to every token at step q, ranking by
# eff_q is ranking by the static priority
#     p_j = s_j - e_j * ln gamma_h,
# formed once, in float32 (§F), as one rounding of the exact value.

def round_to_float32(x) -> float:
    """Round an exact rational (Fraction) or float to the nearest float32,
    ties to even, in one step (no intermediate float64 rounding)."""
    from fractions import Fraction
    fr = Fraction(x)
    if fr == 0:
        return 0.0
    neg = fr < 0
    a = -fr if neg else fr
    e = a.numerator.bit_length() - a.denominator.bit_length()   # 2^e <= a < 2^(e+2)
    while a >= Fraction(2) ** (e + 1):
        e += 1
    while a < Fraction(2) ** e:
        e -= 1
    q = max(e, -126) - 23                  # weight of the last mantissa bit (subnormals below 2^-126)
    m = a / Fraction(2) ** q
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    val = float(n) * 2.0 ** q
    if val > float(np.finfo(np.float32).max):
        val = math.inf
    return -val if neg else val


def decayed_priority(scores: Sequence[float], W: int, D: int, log_gamma: float) -> np.ndarray:
    """Static priorities p_j = fl32(s_j - (j + W + D) * ln gamma) of tokens
    0..n-1 (scores already float32-valued), one rounding of the exact value."""
    from fractions import Fraction
    lg = Fraction(float(np.float32(log_gamma)))
    out = np.empty(len(scores), np.float64)
    for j, sj in enumerate(scores):
        sj = float(sj)
        if math.isnan(sj) or math.isinf(sj):
            out[j] = sj
            continue
        out[j] = round_to_float32(Fraction(sj) - (j + W + D) * lg)
    return out


def effective_score(s_j: float, j: int, q: int, W: int, D: int, log_gamma: float):
    """eff_q(j) = s_j + (q - e_j) * ln gamma, exactly (a Fraction), for q >= e_j."""
    from fractions import Fraction
    return Fraction(float(s_j)) + (q - (j + W + D)) * Fraction(float(np.float32(log_gamma)))


# ---------------------------------------------------------------------------
# Retention policy (§3 Fixed-budget pruning; §C.1 Mask Definition; §I)
# ---------------------------------------------------------------------------

def rank_key(score: float, pos: int):
    """Total order used for every retention decision: (score, -position)."""
    s = float(score)
    if math.isnan(s):
        s = NEG_INF
    return (s, -int(pos))


def eligible_positions(q: int, S: int, W: int, D: int) -> range:
    """Tokens that have left the protected window (and the staging ring) by query q."""
    return range(S, max(S, q - W - D + 1))


def running_topk(scores: Sequence[float], q: int, S: int, W: int, D: int, K: int) -> List[int]:
    """Brute-force running prefix top-k: the K best eligible tokens at q, by rank_key.

    Returned in ascending position order.  If at most K tokens are eligible all
    of them are kept (§C.1: the budget is enforced once the sequence is long
    enough).
    """
    elig = list(eligible_positions(q, S, W, D))
    ranked = sorted(elig, key=lambda j: rank_key(scores[j], j), reverse=True)
    return sorted(ranked[:K])


def sink_positions(q: int, S: int) -> List[int]:
    return list(range(0, min(S, q + 1)))


def recent_positions(q: int, S: int, W: int, D: int) -> List[int]:
    """Window {q-W+1..q} plus staging {q-W-D+1..q-W}, positions >= S only."""
    return list(range(max(S, q - W - D + 1), q + 1))


def attended_positions(q: int, S: int, W: int, D: int, topk: Sequence[int]) -> List[int]:
    """Sinks, recent and selected long-range tokens (§C.1, §I), ascending."""
    return sorted(set(sink_positions(q, S)) | set(recent_positions(q, S, W, D)) | set(topk))


# ---------------------------------------------------------------------------
# Attention over the retained set (§C.1: decoding attends directly over the
# retained cache entries)
# ---------------------------------------------------------------------------

def attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray):
    """Softmax attention of query heads q [G][d] over keys/values [n][d], float64.

    Returns (out [G][d], weights [G][n]).  Scale 1/sqrt(d).
    """
    q = np.asarray(q, np.float64)
    keys = np.asarray(keys, np.float64)
    values = np.asarray(values, np.float64)
    d = q.shape[-1]
    logits = (q @ keys.T) / math.sqrt(d)
    logits = logits - logits.max(axis=-1, keepdims=True)
    w = np.exp(logits)
    w = w / w.sum(axis=-1, keepdims=True)
    return w @ values, w


# ---------------------------------------------------------------------------
# Slot simulator: the incremental rule, slot by slot (for slot-map parity).
# ---------------------------------------------------------------------------

@dataclass
class SlotState:
    S: int
    W: int
    D: int
    K: int
    slot_pos: List[int] = field(default_factory=list)     # slot -> position (-1 = empty)
    slot_score: List[float] = field(default_factory=list)  # top-k slots' ranking scores
    n_seen: int = 0
    n_topk: int = 0

    def __post_init__(self):
        n = self.S + self.W + self.D + self.K
        self.slot_pos = [-1] * n
        self.slot_score = [NEG_INF] * n

    @property
    def topk_base(self) -> int:
        return self.S + self.W + self.D

    def window_slot(self, t: int) -> int:
        return self.S + (t % self.W)

    def staging_slot(self, t: int) -> int:
        return self.S + self.W + (t % self.D)

    def topk_positions(self) -> List[int]:
        b = self.topk_base
        return sorted(p for p in self.slot_pos[b:b + self.K] if p >= 0)

    def _admit(self, newcomers: Sequence[int], scores: Sequence[float]):
        """Merge newly eligible tokens into the long-range slots (see module notes)."""
        if not newcomers:
            return
        b = self.topk_base
        current = [(self.slot_pos[b + i], b + i) for i in range(self.n_topk)]
        pool = [(rank_key(scores[p], p), p) for p, _ in current] + \
               [(rank_key(scores[p], p), p) for p in newcomers]
        pool.sort(reverse=True)
        keep = {p for _, p in pool[:self.K]}
        vacated = [s for p, s in current if p not in keep]
        free = list(range(b + self.n_topk, b + self.K))
        targets = sorted(vacated + free)
        admitted = sorted(p for p in newcomers if p in keep)
        for slot in vacated:
            self.slot_pos[slot] = -1
            self.slot_score[slot] = NEG_INF
        for slot, p in zip(targets, admitted):
            self.slot_pos[slot] = p
            self.slot_score[slot] = float(scores[p])
        self.n_topk = min(self.K, self.n_topk + len(newcomers))

    def append_chunk(self, n_new: int, scores: Sequence[float]):
        """Prefill a chunk of n_new tokens (positions n_seen .. n_seen+n_new-1)."""
        S, W, D = self.S, self.W, self.D
        old, new = self.n_seen, self.n_seen + n_new
        # newly eligible: positions in [S, new-W-D) not eligible before
        lo = max(S, old - W - D)
        hi = max(S, new - W - D)
        newcomers = list(range(lo, hi))
        # staging / window / sink contents follow directly from n_seen
        self.n_seen = new
        self._admit(newcomers, scores)
        self._refresh_recent()

    def decode(self, scores: Sequence[float]):
        """One decode step: token p = n_seen arrives."""
        self.append_chunk(1, scores)

    def _refresh_recent(self):
        S, W, D, n = self.S, self.W, self.D, self.n_seen
        q = n - 1
        for t in range(0, min(S, n)):
            self.slot_pos[t] = t
        for i in range(W):
            self.slot_pos[S + i] = -1
        for i in range(D):
            self.slot_pos[S + W + i] = -1
        for t in range(max(S, q - W + 1), q + 1):
            self.slot_pos[self.window_slot(t)] = t
        for t in range(max(S, q - W - D + 1), max(S, q - W + 1)):
            self.slot_pos[self.staging_slot(t)] = t


# ---------------------------------------------------------------------------
# One (batch row, layer, KV head) unit, end to end.
# ---------------------------------------------------------------------------

@dataclass
class UnitResult:
    outputs: np.ndarray                 # [n_steps][G][d]
    slot_maps: List[List[int]]          # after prefill, then after each step
    topk_sets: List[List[int]]          # brute-force T_q after prefill and each step
    weight_sums: np.ndarray             # [n_steps][G] softmax row sums
    attended_counts: List[int]


class OracleUnit:
    """One (batch row, layer, KV head) unit stepped one decode token at a time.

    k_all, v_all: [n_tokens][d] keys/values of every token the unit will see
    (prompt, then decode tokens); scores: ranking score of every token.  The
    constructor prefills P tokens (in `prefill_chunks` if given); step(q)
    decodes the next token: slot-simulator update, brute-force running top-k
    at the new position, attention of q [G][d] over the attended set.
    """

    def __init__(self, k_all, v_all, scores, S, W, D, K, P, prefill_chunks=None, check_simulator=True):
        self.k_all, self.v_all, self.scores = k_all, v_all, scores
        self.S, self.W, self.D, self.K, self.P = S, W, D, K, P
        self.check = check_simulator
        self.state = SlotState(S, W, D, K)
        chunks = list(prefill_chunks) if prefill_chunks else ([P] if P > 0 else [])
        assert sum(chunks) == P
        for c in chunks:
            self.state.append_chunk(c, scores)
        self.topk = running_topk(scores, P - 1, S, W, D, K) if P > 0 else []
        if check_simulator and P > 0:
            assert self.state.topk_positions() == self.topk, "slot simulator disagrees with brute force"
        self.q = P  # position of the next decode token

    def step(self, qvec):
        q = self.q
        S, W, D, K = self.S, self.W, self.D, self.K
        self.state.decode(self.scores)
        T = running_topk(self.scores, q, S, W, D, K)
        if self.check:
            assert self.state.topk_positions() == T, f"slot simulator disagrees at q={q}"
        A = attended_positions(q, S, W, D, T)
        o, w = attention(qvec, self.k_all[A], self.v_all[A])
        self.topk = T
        self.q = q + 1
        return o, w, T, A


def run_unit(k_all: np.ndarray, v_all: np.ndarray, q_steps: np.ndarray, scores: Sequence[float],
             S: int, W: int, D: int, K: int, P: int,
             prefill_chunks: Optional[Sequence[int]] = None,
             check_simulator: bool = True) -> UnitResult:
    """Run prefill of P tokens, then len(q_steps) decode steps, for one unit.

    k_all, v_all: [P + n_steps][d] keys/values of every token (prompt then
    decode tokens); q_steps: [n_steps][G][d] queries of the decode steps;
    scores: ranking scores of every token (already in ranking precision).
    The attended set at every step is the brute-force definition; the slot
    simulator runs beside it and must hold the same long-range set.
    """
    n_steps = len(q_steps)
    unit = OracleUnit(k_all, v_all, scores, S, W, D, K, P, prefill_chunks, check_simulator)
    slot_maps = [list(unit.state.slot_pos)]
    topk_sets = [list(unit.topk)]
    outs, sums, counts = [], [], []
    for i in range(n_steps):
        o, w, T, A = unit.step(q_steps[i])
        outs.append(o)
        sums.append(w.sum(axis=-1))
        counts.append(len(A))
        slot_maps.append(list(unit.state.slot_pos))
        topk_sets.append(T)
    G = q_steps.shape[1] if n_steps else 0
    d = k_all.shape[-1]
    return UnitResult(outputs=np.array(outs).reshape(n_steps, G, d), slot_maps=slot_maps,
                      topk_sets=topk_sets, weight_sums=np.array(sums).reshape(n_steps, G),
                      attended_counts=counts)


def linear_score(x: np.ndarray, w: np.ndarray, b: float) -> np.ndarray:
    """Stateless headwise linear scorer s = w . x + b (§E.2), float64."""
    return np.asarray(x, np.float64) @ np.asarray(w, np.float64) + float(b)


def unit_scores_linear(k_all, v_all, w, b) -> np.ndarray:
    """Ranking scores of every token of a unit from the linear scorer (§E.2, §F)."""
    return ranking_score(linear_score(head_input(k_all, v_all), w, b))


def unit_scores_mlp(k_all, v_all, w1, b1, w2, b2) -> np.ndarray:
    """Ranking scores of every token of a unit from the MLP scorer (§E.2, §F)."""
    return ranking_score(mlp_score(head_input(k_all, v_all), w1, b1, w2, b2))


def dense_causal_attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray) -> np.ndarray:
    """Plain dense attention of one query [G][d] over all keys/values up to itself."""
    o, _ = attention(q, keys, values)
    return o


# ---------------------------------------------------------------------------
# Parallel sparse prefill attention (§C Efficient Running Top-k Sparse
# Attention: §C.1 Mask Definition, §C.2 Fenwick-Tree Cutoff Computation)
# ---------------------------------------------------------------------------
#
# Over a whole prompt of n tokens, query position q attends to exactly the
# set a decode step at q would attend to: sinks, the recent W + D positions
# and the running top-k of the eligible tokens at q (update before attend).
# The page computes, per head, one "running cutoff" per token and evaluates
# the mask from it on the fly.  Reading of the cutoff: with m = q - W - D the
# newest eligible position at query q, token j is in the long-range set at
# exactly the steps whose m lies in [j, c_j); the oracle computes c_j by its
# definition (the first m at which j is not kept), not by the tree.

INT32_MAX = 2 ** 31 - 1


def running_cutoffs(scores: Sequence[float], n: int, S: int, W: int, D: int, K: int) -> List[int]:
    """Running cutoff c_j of every token of a length-n prompt, by brute force.

    c_j (S <= j <= n-1-W-D) = the first newest-eligible position m >= j at
    which j is not in running_topk (c_j = j: never admitted), or INT32_MAX if
    j is still kept at the last position.  Tokens that never become eligible
    in the prompt (sinks, the last W + D positions) get -1.
    """
    c = [-1] * n
    m_last = n - 1 - W - D
    for j in range(S, m_last + 1):
        c[j] = INT32_MAX
    for m in range(S, m_last + 1):
        kept = set(running_topk(scores, m + W + D, S, W, D, K))
        for j in range(S, m + 1):
            if c[j] == INT32_MAX and j not in kept:
                c[j] = m
    return c


def attention_lse(q: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Log-normaliser log sum_j exp(q_g . k_j / sqrt(d)) of each query head, float64."""
    q = np.asarray(q, np.float64)
    logits = (q @ np.asarray(keys, np.float64).T) / math.sqrt(q.shape[-1])
    mx = logits.max(axis=-1)
    return mx + np.log(np.exp(logits - mx[:, None]).sum(axis=-1))


def prefill_attention(q_all: np.ndarray, k_all: np.ndarray, v_all: np.ndarray, scores: Sequence[float],
                      S: int, W: int, D: int, K: int):
    """Attention outputs of every prompt position under the fixed-budget mask.

    q_all: [n][G][d] queries; k_all, v_all: [n][d]; scores: ranking scores of
    the n tokens.  Position q attends to attended_positions(q, ...) with the
    brute-force running top-k at q (§C.1, §I).  Returns (out [n][G][d],
    lse [n][G] log-normalisers, counts [n] attended tokens per position).
    """
    n = len(k_all)
    G, d = q_all.shape[1], q_all.shape[2]
    out = np.zeros((n, G, d))
    lse = np.zeros((n, G))
    counts = []
    for q in range(n):
        T = running_topk(scores, q, S, W, D, K)
        A = attended_positions(q, S, W, D, T)
        o, _ = attention(q_all[q], k_all[A], v_all[A])
        out[q] = o
        lse[q] = attention_lse(q_all[q], k_all[A])
        counts.append(len(A))
    return out, lse, counts


# ---------------------------------------------------------------------------
# Stateful mLSTM scorer with delayed readout (§A Background: Linear Attention
# and mLSTM; §E.3 mLSTM Scorer; §E.4 Delayed Readout).  Oracle only.
# ---------------------------------------------------------------------------
#
# The pages name the parts but give no formulas; readings (each one also in
# the design notes):
# * Input x_t = [k_t; v_t] (§E.1).  Write features phi(W_k x_t), value
#   W_v x_t, read features phi(W_q x_u) of the token being scored.
# * Hedgehog feature map (§E.3): project to p dims, then [softmax(z); softmax(-z)]
#   (2p features: "halves the projected dimension before positive and negative
#   softmax features").
# * Scalar gates from headwise projections: input pre-activation
#   i~_t = w_i . x_t + b_i used as exp(i~_t); forget gate sigmoid(w_f . x_t + b_f)
#   (log-sigmoid in the stabilised form).  No output gate (§A: removed).
# * The numerically stabilised mLSTM recurrence (§E.3) with C_0 = 0, n_0 = 0,
#   m_0 = 0:  m_t = max(log f_t + m_{t-1}, i~_t),  i'_t = exp(i~_t - m_t),
#   f'_t = exp(log f_t + m_{t-1} - m_t),  C_t = f'_t C_{t-1} + i'_t v_t phi_t^T,
#   n_t = f'_t n_{t-1} + i'_t phi_t,  readout h = C r / max(|n . r|, exp(-m)).
# * Delayed readout (§E.4): the token u that becomes eligible at step
#   q = u + W + D is read with the state after token q; score =
#   w_o . SiLU(h) + b_o (the "SiLU-based transformation with a bias term"; the
#   optional normalisation is left out).  The score is fixed from then on, so
#   the running top-k rule above applies unchanged.

def hedgehog(z: np.ndarray) -> np.ndarray:
    """[softmax(z); softmax(-z)] along the last axis, float64 (§E.3)."""
    z = np.asarray(z, np.float64)
    a = np.exp(z - z.max(axis=-1, keepdims=True))
    b = np.exp(-z - (-z).max(axis=-1, keepdims=True))
    return np.concatenate([a / a.sum(axis=-1, keepdims=True), b / b.sum(axis=-1, keepdims=True)], axis=-1)


def log_sigmoid(x: float) -> float:
    x = float(x)
    return -math.log1p(math.exp(-x)) if x >= 0 else x - math.log1p(math.exp(x))


@dataclass
class MlstmParams:
    """Headwise mLSTM scorer weights: wq, wk [p][2d]; wv [dv][2d];
    wi, wf [2d]; bi, bf scalars; wo [dv]; bo scalar."""
    wq: np.ndarray
    wk: np.ndarray
    wv: np.ndarray
    wi: np.ndarray
    bi: float
    wf: np.ndarray
    bf: float
    wo: np.ndarray
    bo: float


def mlstm_states(x_all: np.ndarray, P: MlstmParams):
    """Stabilised recurrence over tokens 0..n-1; returns the list of
    (C_t, n_t, m_t) after each token t (§E.3)."""
    x_all = np.asarray(x_all, np.float64)
    dv, f2 = P.wv.shape[0], 2 * P.wk.shape[0]
    C, nv, m = np.zeros((dv, f2)), np.zeros(f2), 0.0
    out = []
    for x in x_all:
        phi = hedgehog(P.wk @ x)
        val = P.wv @ x
        it = float(P.wi @ x) + P.bi
        lf = log_sigmoid(float(P.wf @ x) + P.bf)
        m_new = max(lf + m, it)
        ip, fp = math.exp(it - m_new), math.exp(lf + m - m_new)
        C = fp * C + ip * np.outer(val, phi)
        nv = fp * nv + ip * phi
        m = m_new
        out.append((C.copy(), nv.copy(), m))
    return out


def mlstm_readout(C: np.ndarray, nv: np.ndarray, m: float, r: np.ndarray) -> np.ndarray:
    """h = C r / max(|n . r|, exp(-m)) (§A: normalised retrieval from the summary)."""
    return (C @ r) / max(abs(float(nv @ r)), math.exp(-m))


def silu(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, np.float64)
    return x / (1.0 + np.exp(-x))


def unit_scores_mlstm(k_all, v_all, P: MlstmParams, S: int, W: int, D: int) -> np.ndarray:
    """Delayed-readout score of every token u >= S whose eligibility step
    q = u + W + D lies inside the sequence, rounded to float32 (§E.4, §F);
    NaN for the others (sinks, and tokens not yet eligible at the end)."""
    x_all = head_input(k_all, v_all)
    n = len(x_all)
    states = mlstm_states(x_all, P)
    s = np.full(n, np.nan)
    for u in range(S, n):
        q = u + W + D
        if q >= n:
            break
        C, nv, m = states[q]
        h = mlstm_readout(C, nv, m, hedgehog(P.wq @ x_all[u]))
        s[u] = float(P.wo @ silu(h)) + P.bo
    return ranking_score(s)
