"""Seeded synthetic workloads for the KVpop decode path.

This module only draws random tensors with the shapes, value distributions and
structure of the workloads that the KVpop page ("KVpop -- Key-Value Cache
Compression with Predictive Online Pruning", §4 Experiments) evaluates on
Qwen3-4B / Qwen3-8B-shaped attention.  It holds none of the method's
arithmetic: both the CPU oracle and the CUDA path consume what it returns.

Readings of the workload recipe (stated once here, used everywhere):

* Q, K, V ~ N(0, 1), rounded to bf16 for the bf16 workloads (fp32 for the tiny
  workload).
* "2% of keys given a x3 heavy-hitter scale": an independent Bernoulli(0.02)
  draw per (batch, kv head, position); a selected key vector is multiplied by 3.
  Applies to prompt and decode keys alike.
* Tiny workload sink: one seeded unit direction u (shared by all heads); token
  0's key gets k0 <- k0 + 3 (u.k0) u, i.e. its component along u is scaled x4.
* Scorer MLP weights: W1 ~ N(0, 0.1^2) with layout [layer][kv_head][hidden][2d],
  w2 ~ N(0, 0.1^2) [layer][kv_head][hidden], biases zero.
* Seeds: one master seed; every tensor is drawn from its own sub-stream keyed by
  (workload, layer, kind, step), so any layer or step can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: str            # "f32" or "bf16"
    sinks: int
    window: int
    topk: int
    delay: int
    prefill: int          # prompt tokens per (batch row)
    decode: int           # decode steps in the workload's description
    scorer_hidden: int
    heavy_hitter_frac: float = 0.0
    heavy_hitter_scale: float = 3.0
    sink_direction: bool = False
    scorer_std: float = 0.1

    @property
    def budget(self) -> int:
        return self.sinks + self.window + self.topk

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def compression_ratio(self) -> float:
        # CR quoted against the prompt length: CR = 1 - B / P.
        return 1.0 - self.budget / self.prefill if self.prefill > 0 else 0.0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five workloads: a tiny CPU-checkable case, Qwen3-4B-shaped at 75% and
# 87.5% ("88%") compression, Qwen3-8B-shaped with a 32-step delayed scorer, and
# the bandwidth sweep on the Qwen3-8B shape.
TINY = Workload("tiny_b1_l1_hq4_hkv2_d64_f32_B64", batch=1, n_layers=1, n_q_heads=4,
                n_kv_heads=2, head_dim=64, dtype="f32", sinks=4, window=16, topk=44,
                delay=0, prefill=128, decode=128, scorer_hidden=32,
                sink_direction=True)
QWEN3_4B_CR75 = Workload("qwen3_4b_cr75_b16_B2048", batch=16, n_layers=36, n_q_heads=32,
                         n_kv_heads=8, head_dim=128, dtype="bf16", sinks=4, window=128,
                         topk=1916, delay=0, prefill=8192, decode=1024, scorer_hidden=64,
                         heavy_hitter_frac=0.02)
QWEN3_4B_CR88 = QWEN3_4B_CR75.replace(name="qwen3_4b_cr88_b64_B1024", batch=64, topk=892)
QWEN3_8B_D32 = Workload("qwen3_8b_cr88_d32_b32_B4096", batch=32, n_layers=36, n_q_heads=32,
                        n_kv_heads=8, head_dim=128, dtype="bf16", sinks=4, window=256,
                        topk=3836, delay=32, prefill=32768, decode=2048, scorer_hidden=64,
                        heavy_hitter_frac=0.02)


def sweep_point(budget: int, batch: int) -> Workload:
    """Bandwidth-sweep point on the Qwen3-8B shape (4 sinks, window 128)."""
    return Workload(f"qwen3_8b_sweep_b{batch}_B{budget}", batch=batch, n_layers=36,
                    n_q_heads=32, n_kv_heads=8, head_dim=128, dtype="bf16", sinks=4,
                    window=128, topk=budget - 132, delay=0, prefill=65536, decode=256,
                    scorer_hidden=64, heavy_hitter_frac=0.02)


SWEEP_BUDGETS = (512, 1024, 2048, 4096, 8192)
SWEEP_BATCHES = (1, 32, 256)

WORKLOADS = {w.name: w for w in (TINY, QWEN3_4B_CR75, QWEN3_4B_CR88, QWEN3_8B_D32)}


def _sub_seed(master: int, *key) -> int:
    h = hashlib.blake2b(repr((master,) + tuple(key)).encode(), digest_size=8)
    return int.from_bytes(h.digest(), "little") & ((1 << 63) - 1)


def _gen(device, master: int, *key) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_sub_seed(master, *key))
    return g


def _normal(shape, gen, device) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)


def _sink_direction(w: Workload, master: int) -> torch.Tensor:
    u = _normal((w.head_dim,), _gen("cpu", master, w.name, "sink_dir"), "cpu")
    return u / u.norm()


def _shape_keys(w: Workload, k: torch.Tensor, master: int, layer: int, tag, first_pos: int,
                device) -> torch.Tensor:
    """Apply the key structure (heavy hitters, token-0 sink) in place; k is [b][h][n][d]."""
    if w.heavy_hitter_frac > 0:
        g = _gen(device, master, w.name, layer, "hh", tag)
        hit = torch.rand(k.shape[:-1], generator=g, device=device) < w.heavy_hitter_frac
        k.mul_(torch.where(hit, w.heavy_hitter_scale, 1.0).unsqueeze(-1).to(k.dtype))
    if w.sink_direction and first_pos == 0 and k.shape[2] > 0:
        u = _sink_direction(w, master).to(device)
        k0 = k[:, :, 0, :]
        k0.add_(3.0 * (k0 @ u).unsqueeze(-1) * u)
    return k


def prompt_kv(w: Workload, layer: int, n_tokens: Optional[int] = None, master: int = 0,
              device="cpu", first_pos: int = 0):
    """Prompt keys/values for one layer: two tensors [batch][kv_heads][n][d] in w's dtype.

    `first_pos` > 0 draws a later chunk of the same prompt stream (a chunk is
    keyed by its first position, so chunked and whole-prompt draws differ; the
    tests that compare them draw once and slice).
    """
    n = w.prefill if n_tokens is None else n_tokens
    shape = (w.batch, w.n_kv_heads, n, w.head_dim)
    k = _normal(shape, _gen(device, master, w.name, layer, "pk", first_pos), device)
    v = _normal(shape, _gen(device, master, w.name, layer, "pv", first_pos), device)
    _shape_keys(w, k, master, layer, ("p", first_pos), first_pos, device)
    dt = w.torch_dtype()
    return k.to(dt), v.to(dt)


def prompt_queries(w: Workload, layer: int, n_tokens: Optional[int] = None, master: int = 0, device="cpu"):
    """Queries of every prompt position for one layer: [batch][q_heads][n][d] in w's dtype."""
    n = w.prefill if n_tokens is None else n_tokens
    q = _normal((w.batch, w.n_q_heads, n, w.head_dim), _gen(device, master, w.name, layer, "pq", n), device)
    return q.to(w.torch_dtype())


def decode_inputs(w: Workload, layer: int, step: int, master: int = 0, device="cpu"):
    """One decode step's inputs for one layer: q [b][Hq][d], k_new/v_new [b][Hkv][d]."""
    q = _normal((w.batch, w.n_q_heads, w.head_dim), _gen(device, master, w.name, layer, "q", step), device)
    k = _normal((w.batch, w.n_kv_heads, 1, w.head_dim),
                _gen(device, master, w.name, layer, "k", step), device)
    v = _normal((w.batch, w.n_kv_heads, w.head_dim), _gen(device, master, w.name, layer, "v", step), device)
    _shape_keys(w, k, master, layer, ("d", step), 1, device)
    dt = w.torch_dtype()
    return q.to(dt), k[:, :, 0, :].contiguous().to(dt), v.to(dt)


def decode_inputs_batched(w: Workload, layer: int, n_steps: int, master: int = 0, device="cpu",
                          first_step: int = 0):
    """n_steps decode steps at once: q [n][b][Hq][d], k/v [n][b][Hkv][d] (one draw per call)."""
    key = (w.name, layer, "steps", first_step, n_steps)
    q = _normal((n_steps, w.batch, w.n_q_heads, w.head_dim), _gen(device, master, *key, "q"), device)
    k = _normal((n_steps, w.batch, w.n_kv_heads, w.head_dim), _gen(device, master, *key, "k"), device)
    v = _normal((n_steps, w.batch, w.n_kv_heads, w.head_dim), _gen(device, master, *key, "v"), device)
    if w.heavy_hitter_frac > 0:
        g = _gen(device, master, *key, "hh")
        hit = torch.rand(k.shape[:-1], generator=g, device=device) < w.heavy_hitter_frac
        k.mul_(torch.where(hit, w.heavy_hitter_scale, 1.0).unsqueeze(-1))
    dt = w.torch_dtype()
    return q.to(dt), k.to(dt), v.to(dt)


def scorer_weights(w: Workload, master: int = 0, device="cpu"):
    """Per-(layer, kv head) MLP 2d -> hidden -> 1 weights: w1, b1, w2, b2 (fp32)."""
    L, H, hid, d2 = w.n_layers, w.n_kv_heads, w.scorer_hidden, 2 * w.head_dim
    w1 = _normal((L, H, hid, d2), _gen(device, master, w.name, "w1"), device) * w.scorer_std
    w2 = _normal((L, H, hid), _gen(device, master, w.name, "w2"), device) * w.scorer_std
    b1 = torch.zeros((L, H, hid), device=device)
    b2 = torch.zeros((L, H), device=device)
    return w1.contiguous(), b1, w2.contiguous(), b2


def mlstm_weights(w: Workload, p: int = 16, dv: int = 16, master: int = 0, device="cpu"):
    """Seeded weights of the stateful mLSTM scorer, packed per (layer, KV head)
    as the C ABI takes them: fp32 [L][Hkv][(2p + dv + 2) * 2d + pad] holding
    the rows W_q [p], W_k [p], W_v [dv], w_i, w_f (each 2d long), then w_o
    [dv], b_i, b_f, b_o and zero padding to a multiple of 4.

    Reading of the recipe (the pages give no trained weights): W_q, W_k, W_v
    and w_o ~ N(0, 0.1^2); w_i, w_f ~ N(0, 0.05^2); b_i = 0, b_f = 3 (a
    forget gate near sigmoid(3) = 0.95, the stable early memory the page's
    §E.5 initialisation aims at); b_o = 0."""
    L, H, d2 = w.n_layers, w.n_kv_heads, 2 * w.head_dim
    rows = 2 * p + dv + 2
    tail = ((dv + 3 + 3) // 4) * 4
    g = _gen(device, master, w.name, "mlstm", p, dv)
    mat = _normal((L, H, rows, d2), g, device)
    scale = torch.full((rows,), 0.1, device=device)
    scale[2 * p + dv:] = 0.05
    mat = mat * scale[:, None]
    t = torch.zeros((L, H, tail), device=device)
    t[..., :dv] = _normal((L, H, dv), g, device) * 0.1
    t[..., dv + 1] = 3.0
    return torch.cat([mat.reshape(L, H, rows * d2), t], dim=-1).contiguous()


def unpack_mlstm(packed_head, p: int, dv: int, d: int) -> dict:
    """One (layer, KV head) block of mlstm_weights as named float64 numpy
    arrays: wq, wk [p][2d], wv [dv][2d], wi, wf [2d], wo [dv]; bi, bf, bo."""
    x = packed_head.double().cpu().numpy()
    d2 = 2 * d
    rows = 2 * p + dv + 2
    m = x[:rows * d2].reshape(rows, d2)
    t = x[rows * d2:]
    return {"wq": m[:p], "wk": m[p:2 * p], "wv": m[2 * p:2 * p + dv], "wi": m[2 * p + dv], "wf": m[2 * p + dv + 1],
            "wo": t[:dv], "bi": float(t[dv]), "bf": float(t[dv + 1]), "bo": float(t[dv + 2])}


def external_scores(w: Workload, layer: int, n_tokens: int, master: int = 0, device="cpu",
                    tag: str = "ext", tie_levels: int = 0):
    """Caller-supplied per-token scores [b][Hkv][n] (fp32).

    tie_levels > 0 quantises the scores to that many distinct values so that
    equal scores occur often (exercises the tie rule).
    """
    g = _gen(device, master, w.name, layer, tag, n_tokens)
    s = _normal((w.batch, w.n_kv_heads, n_tokens), g, device)
    if tie_levels > 0:
        s = torch.floor(s * tie_levels / 4.0)
    return s
