"""Runs the CUDA path through the C ABI and the CPU oracle on the same seeded
inputs, and compares them.

GPU side: fixed_budget_kv_kvpop_b200 (libkvpop.so).  Oracle side:
oracle.kvpop_oracle.  The two only share the seeded inputs drawn from
kvpop_workloads.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import numpy as np
import torch

import kvpop_workloads as wl
from oracle import kvpop_oracle as orc

BF16_ATOL = 2e-2     # attention outputs, bf16 inputs/outputs, fp32 accumulation
F32_ATOL = 1e-4      # attention outputs, fp32 everywhere
SCORE_RTOL = 1e-4    # scorer outputs: |ds| <= 1e-4 * max(|s|, 1e-2 * rms)


@dataclasses.dataclass
class Run:
    w: wl.Workload
    layers: Sequence[int]
    prompt_k: dict          # layer -> tensor [b][Hkv][P][d] (device)
    prompt_v: dict
    dec_q: dict             # layer -> list of [b][Hq][d]
    dec_k: dict
    dec_v: dict
    outs: dict              # layer -> list of [b][Hq][d] (host, float64)
    slot_pos: dict          # layer -> list of [units][NS] int32 per inspected step (None = not inspected)
    slot_score: dict
    ext_prompt: Optional[dict] = None
    ext_dec: Optional[dict] = None
    weights: Optional[tuple] = None
    cache: object = None
    log_decay: Optional[np.ndarray] = None   # [L][Hkv] ln gamma, or None
    mlstm: Optional[tuple] = None            # (packed device weights, p, dv) of the mLSTM scorer, or None


def build_cache(w: wl.Workload, n_layers: int, external: bool, weights=None, max_chunk=None, debug=True,
                log_decay=None, mlstm=None, library=None):
    import fixed_budget_kv_kvpop_b200 as kp
    keep = ()
    kw = {}
    if mlstm is not None:
        packed, p, dv = mlstm
        kw = dict(scorer="mlstm", mlstm_p=p, mlstm_dv=dv, mlstm_w=packed)
        keep = (packed,)
    elif not external:
        w1, b1, w2, b2 = weights
        kw = dict(w1=w1, b1=b1, w2=w2, b2=b2)
        keep = weights
    cfg = kp.make_config(batch=w.batch, n_layers=n_layers, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                         head_dim=w.head_dim, sinks=w.sinks, window=w.window, topk=w.topk, delay=w.delay,
                         max_prefill_chunk=max_chunk if max_chunk is not None else max(w.prefill, 1),
                         dtype=w.dtype, scorer_hidden=w.scorer_hidden, external_scores=external,
                         debug_checks=debug, log_decay=log_decay, **kw)
    if log_decay is not None:
        keep = tuple(keep) + (log_decay,)
    return kp.KVPopCache(cfg, device="cuda", keepalive=keep, library=library)


def run_gpu(w: wl.Workload, n_layers: int, n_steps: int, *, external: bool = False, chunks=None,
            inspect_every: int = 1, layers_to_keep: Sequence[int] = (0,), tie_levels: int = 0,
            master: int = 0, gen_device: str = "cpu", debug=True, split: bool = False,
            log_decay: Optional[np.ndarray] = None, mlstm_dims: Optional[tuple] = None, library=None,
            step_hook=None) -> Run:
    """Prefill + n_steps decode steps of every layer on the GPU, through the C ABI.
    log_decay: optional float32 [n_layers][Hkv] ln gamma (temporal decay).
    mlstm_dims: (p, dv) to score with the stateful mLSTM scorer instead of the MLP.
    library: another build of libkvpop (load_library); step_hook(cache, i, when)
    is called with when = "before" / "after" around decode step i."""
    dev = "cuda"
    weights = None
    mlstm = None
    if mlstm_dims is not None:
        p_, dv_ = mlstm_dims
        mlstm = (wl.mlstm_weights(w.replace(n_layers=n_layers), p_, dv_, master=master).to(dev), p_, dv_)
    elif not external:
        # scorer_hidden 0 = linear scorer: one weight row per head (w1[..., 0, :]) and b2
        wshape = w.replace(n_layers=n_layers, scorer_hidden=max(w.scorer_hidden, 1))
        weights = tuple(t.to(dev) for t in wl.scorer_weights(wshape, master=master))
    chunks = list(chunks) if chunks else ([w.prefill] if w.prefill > 0 else [])
    dec_dev = None if log_decay is None else torch.tensor(np.asarray(log_decay, np.float32), device=dev)
    cache = build_cache(w, n_layers, external, weights, max_chunk=max(chunks) if chunks else 1, debug=debug,
                        log_decay=dec_dev, mlstm=mlstm, library=library)
    run = Run(w=w, layers=list(layers_to_keep), prompt_k={}, prompt_v={}, dec_q={}, dec_k={}, dec_v={},
              outs={}, slot_pos={}, slot_score={}, ext_prompt={} if external else None,
              ext_dec={} if external else None, weights=weights, cache=cache,
              log_decay=None if log_decay is None else np.asarray(log_decay, np.float32), mlstm=mlstm)
    for layer in range(n_layers):
        k, v = wl.prompt_kv(w, layer, master=master, device=gen_device)
        k, v = k.to(dev), v.to(dev)
        ext = None
        if external:
            ext = wl.external_scores(w, layer, w.prefill + n_steps, master=master, device=gen_device,
                                     tie_levels=tie_levels).to(dev)
        off = 0
        for c in chunks:
            cache.prefill(layer, k[:, :, off:off + c].contiguous(), v[:, :, off:off + c].contiguous(),
                          None if ext is None else ext[:, :, off:off + c].contiguous())
            off += c
        keep = layer in run.layers
        if keep:
            run.prompt_k[layer], run.prompt_v[layer] = k, v
            run.dec_q[layer], run.dec_k[layer], run.dec_v[layer], run.outs[layer] = [], [], [], []
            run.slot_pos[layer], run.slot_score[layer] = [], []
            if external:
                run.ext_prompt[layer] = ext[:, :, :w.prefill]
                run.ext_dec[layer] = []
            if inspect_every:
                p, s, _ = cache.inspect(layer)
                run.slot_pos[layer].append(p.copy())
                run.slot_score[layer].append(s.copy())
        else:
            del k, v
    for i in range(n_steps):
        if step_hook is not None:
            step_hook(cache, i, "before")
        for layer in range(n_layers):
            q, kn, vn = wl.decode_inputs(w, layer, i, master=master, device=gen_device)
            q, kn, vn = q.to(dev), kn.to(dev), vn.to(dev)
            es = None
            if external:
                es = wl.external_scores(w, layer, w.prefill + n_steps, master=master, device=gen_device,
                                        tie_levels=tie_levels)[:, :, w.prefill + i].contiguous().to(dev)
            out = torch.empty_like(q)
            if split:
                cache.decode_append(layer, kn, vn, es)
                cache.decode_attend(layer, q, out)
            else:
                cache.decode_step(layer, q, kn, vn, out, es)
            if layer in run.layers:
                run.dec_q[layer].append(q)
                run.dec_k[layer].append(kn)
                run.dec_v[layer].append(vn)
                run.outs[layer].append(out.double().cpu())
                if external:
                    run.ext_dec[layer].append(es)
                if inspect_every and ((i + 1) % inspect_every == 0 or i == n_steps - 1):
                    p, s, _ = cache.inspect(layer)
                    run.slot_pos[layer].append(p.copy())
                    run.slot_score[layer].append(s.copy())
                else:
                    run.slot_pos[layer].append(None)
                    run.slot_score[layer].append(None)
        if step_hook is not None:
            step_hook(cache, i, "after")
    torch.cuda.synchronize()
    st, bits = cache.get_error()
    assert st == 0, f"device error status {st} bits {bits}"
    return run


def unit_inputs(run: Run, layer: int, unit: int):
    """The oracle's view of one unit: k_all, v_all [P+n][d], q_steps [n][G][d] (float64)."""
    w = run.w
    b, h = divmod(unit, w.n_kv_heads)
    G = w.group
    kp_ = run.prompt_k[layer][b, h].double().cpu().numpy()
    vp_ = run.prompt_v[layer][b, h].double().cpu().numpy()
    kd = np.array([t[b, h].double().cpu().numpy() for t in run.dec_k[layer]]).reshape(-1, w.head_dim)
    vd = np.array([t[b, h].double().cpu().numpy() for t in run.dec_v[layer]]).reshape(-1, w.head_dim)
    qd = np.array([t[b, h * G:(h + 1) * G].double().cpu().numpy() for t in run.dec_q[layer]])
    qd = qd.reshape(len(run.dec_q[layer]), G, w.head_dim)
    return np.concatenate([kp_, kd]), np.concatenate([vp_, vd]), qd


def unit_scores(run: Run, layer: int, unit: int, k_all, v_all):
    """The oracle's ranking value of every token of a unit: its float32 score,
    or with temporal decay its static priority."""
    w = run.w
    b, h = divmod(unit, w.n_kv_heads)
    if run.ext_prompt is not None:
        pr = run.ext_prompt[layer][b, h].double().cpu().numpy()
        dc = np.array([t[b, h].item() for t in run.ext_dec[layer]], dtype=np.float64)
        s = orc.ranking_score(np.concatenate([pr, dc]))
    elif run.mlstm is not None:
        packed, p_, dv_ = run.mlstm
        P = orc.MlstmParams(**wl.unpack_mlstm(packed[layer, h], p_, dv_, w.head_dim))
        s = orc.unit_scores_mlstm(k_all, v_all, P, w.sinks, w.window, w.delay)
    else:
        w1, b1, w2, b2 = (t.double().cpu().numpy() for t in run.weights)
        if w.scorer_hidden == 0:
            s = orc.unit_scores_linear(k_all, v_all, w1[layer, h, 0], b2[layer, h])
        else:
            s = orc.unit_scores_mlp(k_all, v_all, w1[layer, h], b1[layer, h], w2[layer, h], b2[layer, h])
    if run.log_decay is not None:
        s = orc.decayed_priority(s, w.window, w.delay, float(run.log_decay[layer, h]))
    return s


def score_tol(s_ref: np.ndarray, all_scores: np.ndarray) -> np.ndarray:
    """|ds| allowed per token: 1e-4 of max(|s|, 1e-2 RMS of the unit's scores).
    Tokens without a score (NaN: not yet eligible under a delayed readout)
    are left out of the RMS."""
    fin = all_scores[np.isfinite(all_scores)]
    rms = float(np.sqrt(np.mean(np.square(fin)))) if fin.size else 0.0
    return SCORE_RTOL * np.maximum(np.abs(s_ref), 1e-2 * rms)


def sets_equivalent(gpu: Sequence[int], ref: Sequence[int], scores: np.ndarray, tol_all: np.ndarray) -> bool:
    """GPU and oracle long-range sets agree, or differ only on near-tied pairs."""
    a, b = set(gpu) - set(ref), set(ref) - set(gpu)
    if len(a) != len(b):
        return False
    xa = sorted(a, key=lambda j: scores[j])
    xb = sorted(b, key=lambda j: scores[j])
    return all(abs(scores[x] - scores[y]) <= max(tol_all[x], tol_all[y]) for x, y in zip(xa, xb))


def check_unit(run: Run, layer: int, unit: int, *, exact_slots: bool, atol: float, chunks=None,
               steps_to_check: Optional[Sequence[int]] = None):
    """Compare one unit against the oracle; raises AssertionError on a mismatch."""
    w = run.w
    k_all, v_all, qd = unit_inputs(run, layer, unit)
    scores = unit_scores(run, layer, unit, k_all, v_all)
    n = len(qd)
    res = orc.run_unit(k_all, v_all, qd, scores, w.sinks, w.window, w.delay, w.topk, w.prefill,
                       prefill_chunks=chunks)
    base = w.sinks + w.window + w.delay
    tol_all = score_tol(scores, scores)
    steps = range(n) if steps_to_check is None else steps_to_check
    for i in steps:
        gpu_out = run.outs[layer][i][unit // w.n_kv_heads,
                                     (unit % w.n_kv_heads) * w.group:(unit % w.n_kv_heads + 1) * w.group].numpy()
        pos = run.slot_pos[layer][i + 1]
        ref_out = res.outputs[i]
        if pos is not None:
            gp = pos[unit]
            gtop = sorted(int(x) for x in gp[base:] if x >= 0)
            if exact_slots:
                assert list(gp) == res.slot_maps[i + 1], (layer, unit, i, list(gp), res.slot_maps[i + 1])
            else:
                # GPU scores of the long-range tokens vs the oracle's
                gs = run.slot_score[layer][i + 1][unit]
                for sl in range(base, len(gp)):
                    if gp[sl] >= 0:
                        j = int(gp[sl])
                        assert abs(float(gs[sl]) - scores[j]) <= tol_all[j] * 1.0 + 1e-30, \
                            (layer, unit, i, j, float(gs[sl]), scores[j])
                assert sets_equivalent(gtop, res.topk_sets[i + 1], scores, tol_all), (layer, unit, i)
                if gtop != res.topk_sets[i + 1]:
                    q = w.prefill + i
                    A = orc.attended_positions(q, w.sinks, w.window, w.delay, gtop)
                    ref_out, _ = orc.attention(qd[i], k_all[A], v_all[A])
        np.testing.assert_allclose(gpu_out, ref_out, rtol=0, atol=atol,
                                   err_msg=f"layer {layer} unit {unit} step {i}")
    return res
