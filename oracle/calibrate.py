"""Measure routing sparsity of a synthetic workload with the oracle.

Used to choose the plant strengths recorded in ``gen/configs.py``.  Calls
only the oracle and the input generator.

    python -m oracle.calibrate prefill --strength 3 4 5
"""

from __future__ import annotations

import argparse

import numpy as np

from gen import get_config, kv_values, make_plan, q_values, sample_rows
from oracle.dash_oracle import block_summaries, candidate_blocks, route_row


def sparsity(cfg, kv_heads=None, row_stride=97, batches=None) -> dict:
    """Block-weighted sparsity 1 - sum|support| / sum N over sampled rows."""
    plan = make_plan(cfg)
    G = cfg.group
    kv_heads = range(cfg.kv_heads) if kv_heads is None else kv_heads
    batches = range(cfg.batch) if batches is None else batches
    sel = cand = 0
    per_head = {}
    for b in batches:
        for g in kv_heads:
            if cfg.mode == "decode":
                L = int(plan.seqlens[b])
                rows = [L - 1]
                n_tok = L
                qg = q_values(cfg, plan, b, [0], range(g * G, (g + 1) * G), as_float32=True).numpy()[None, 0]
            else:
                rows = sample_rows(cfg.seq, cfg.block, row_stride)
                n_tok = cfg.seq
                qg = q_values(cfg, plan, b, rows, range(g * G, (g + 1) * G), as_float32=True).numpy()
            k = kv_values(cfg, plan, "k", b, range(n_tok), [g], as_float32=True).numpy()[:, 0]
            summ = block_summaries(k, plan.w_s.numpy(), cfg.block, n_tok)
            hs = hc = 0
            for ri, pos in enumerate(rows):
                _, cands = candidate_blocks(pos, cfg.block, n_tok, cfg.causal)
                if not cands:
                    continue
                r = route_row(qg[ri], summ[cands], cfg.alpha)
                hs += len(r["idx"])
                hc += len(cands)
            per_head[(b, g)] = 1.0 - hs / max(hc, 1)
            sel += hs
            cand += hc
    return {"sparsity": 1.0 - sel / max(cand, 1), "per_head": per_head}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("config")
    ap.add_argument("--strength", type=float, nargs="*")
    ap.add_argument("--kv-heads", type=int, nargs="*")
    ap.add_argument("--batches", type=int, nargs="*")
    ap.add_argument("--stride", type=int, default=97)
    a = ap.parse_args()
    cfg = get_config(a.config)
    for s in a.strength or [cfg.key_strength]:
        r = sparsity(cfg.with_(key_strength=s), a.kv_heads, a.stride, a.batches)
        print(f"{a.config} key_strength={s}: sparsity {r['sparsity']:.4f}",
              {k: round(v, 3) for k, v in r["per_head"].items()})


if __name__ == "__main__":
    np.set_printoptions(precision=4)
    main()
