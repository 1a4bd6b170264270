"""Helpers shared by the GPU parity tests: oracle evaluation on the exact
stored inputs (regenerated on the CPU from the seeded generator) and the
comparison rules.

Tolerances (from the workload definitions):
  * selected-block sets identical, excluding blocks whose routing logit lies
    within 1e-4 of some head's threshold (on the (alpha-1) z scale);
  * entmax weights (per-head p and the group mean p_bar) within 1e-5;
  * outputs within 2e-2 max-abs for bf16/f16 inputs, 1e-4 for fp32.
"""

from __future__ import annotations

import numpy as np
import torch

from gen import kv_values, q_values
from oracle.dash_oracle import block_summaries, block_summaries_sdpa, candidate_blocks, forward_row

BAND = 1e-4
P_TOL = 1e-5
OUT_TOL = {"f32": 1e-4, "f16": 2e-2, "bf16": 2e-2}


def oracle_head(cfg, plan, b, g, rows, n_tokens=None, sigma=1.0, qbar=None):
    """Oracle records for query positions ``rows`` of (batch b, KV group g).

    sigma: prior strength; qbar: learned summary query of this KV head [d] (None: mean pooling).
    """
    G, d = cfg.group, cfg.head_dim
    n_tokens = cfg.seq if n_tokens is None else n_tokens
    k = kv_values(cfg, plan, "k", b, range(n_tokens), [g], as_float32=True)[:, 0].double().numpy()
    v = kv_values(cfg, plan, "v", b, range(n_tokens), [g], as_float32=True)[:, 0].double().numpy()
    q = q_values(cfg, plan, b, rows, range(g * G, (g + 1) * G), as_float32=True).double().numpy()
    w = plan.w_s.double().numpy()
    if qbar is None:
        summ = block_summaries(k, w, cfg.block, n_tokens)
    else:
        summ = block_summaries_sdpa(k, w, np.asarray(qbar, dtype=np.float64), cfg.block, n_tokens)
    recs = []
    for ri, pos in enumerate(rows):
        r = forward_row(q[ri], k, v, summ, pos, n_tokens, cfg.block, cfg.alpha, cfg.causal, sigma=sigma)
        recs.append(r)
    return recs, summ


def oracle_decode_pair(cfg, plan, b, g, sigma=1.0):
    G = cfg.group
    L = int(plan.seqlens[b])
    k = kv_values(cfg, plan, "k", b, range(L), [g], as_float32=True)[:, 0].double().numpy()
    v = kv_values(cfg, plan, "v", b, range(L), [g], as_float32=True)[:, 0].double().numpy()
    q = q_values(cfg, plan, b, [0], range(g * G, (g + 1) * G), as_float32=True)[0].double().numpy()
    n_complete = (L - 1) // cfg.block
    summ = block_summaries(k[: n_complete * cfg.block], plan.w_s.double().numpy(), cfg.block, n_complete * cfg.block)
    rec = forward_row(q, k, v, summ, L - 1, L, cfg.block, cfg.alpha, True, sigma=sigma)
    return rec, summ


def check_route_row(rec, gpu_idx, gpu_logp, gpu_cnt, where=""):
    """Selected sets (outside the tau band) and p_bar of one row."""
    cand = np.asarray(rec["cand"], dtype=np.int64)
    n = int(gpu_cnt)
    got = np.asarray(gpu_idx[:n], dtype=np.int64)
    assert np.all(np.diff(got) > 0), f"{where}: list not ascending: {got}"
    if len(cand) == 0:
        assert n == 0, f"{where}: blocks selected with no candidates"
        return 0
    margin = rec["x"] - rec["tau"][:, None]
    must_in = set(cand[(margin > BAND).any(axis=0)].tolist())
    must_out = set(cand[(margin < -BAND).all(axis=0)].tolist())
    gs = set(got.tolist())
    assert must_in <= gs, f"{where}: missing {sorted(must_in - gs)[:8]}"
    bad = must_out & gs
    assert not bad, f"{where}: extra {sorted(bad)[:8]}"
    # group-mean weights of blocks both sides selected
    pos_of = {c: i for i, c in enumerate(cand.tolist())}
    pg = np.exp(np.asarray(gpu_logp[:n], dtype=np.float64))
    po = np.array([rec["pbar"][pos_of[c]] for c in got.tolist()])
    err = np.abs(pg - po).max() if n else 0.0
    assert err <= P_TOL, f"{where}: p_bar error {err:.3g}"
    return err


def check_p_dense(rec, p_row_heads, tau_heads, where=""):
    """Per-head entmax weights [G, t_cap] and thresholds [G]."""
    cand = np.asarray(rec["cand"], dtype=np.int64)
    if len(cand) == 0:
        assert np.all(p_row_heads == 0)
        return 0.0
    got = p_row_heads[:, cand]
    err = np.abs(got - rec["p"]).max()
    assert err <= P_TOL, f"{where}: p error {err:.3g}"
    terr = np.abs(tau_heads - rec["tau"]).max()
    assert terr <= P_TOL, f"{where}: tau error {terr:.3g}"
    # non-candidates are zero
    mask = np.ones(p_row_heads.shape[1], bool)
    mask[cand] = False
    assert np.all(p_row_heads[:, mask] == 0)
    return err


def max_abs(a, b) -> float:
    return float(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64)).max())


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy() if t.dtype != torch.int32 else t.cpu().numpy()
