"""Plain fp64 CPU oracle of the DashAttention backward pass.

TEST INFRASTRUCTURE ONLY, like ``oracle.dash_oracle`` (whose forward it
differentiates): only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it.

Source.  The page "DashAttention: Differentiable and Adaptive Sparse
Hierarchical Attention" (gist.science explainer of arXiv 2605.18753),
sections "Stage 1: entmax chunk routing" (the router is differentiable, so
the loss reaches the summaries and the queries through the routing
probabilities) and "Stage 2: prior-induced sparse softmax" (the prior enters
the logits as log p_bar, so its gradient is the softmax gradient summed over
the tokens of the block).  The alpha-entmax Jacobian follows Peters, Niculae
& Martins (2019), "Sparse Sequence-to-Sequence Models", section 3: with
u_c = p_c^(2 - alpha) on the support (0 elsewhere),
dp/dz = diag(u) - u u^T / sum(u).

The loss is L = sum(dout * out) for the forward of ``oracle.dash_oracle``
(mean-pooled summaries, prior strength sigma); every gradient below is the
exact derivative of that forward, taken step by step in reverse order:

  stage 2   l_j = q . k_j / sqrt(d) + bias_j,  o = softmax(l) V
            dP_j = dout . v_j,  D = dout . o,  dS_j = P_j (dP_j - D)
            dq += dS K / sqrt(d),  dk_j += dS_j q / sqrt(d),  dv_j += P_j dout
            d log p_bar_c = sigma * sum_{j in c} dS_j   (summed over the heads)
  GQA mean  dp_{h,c} = d log p_bar_c / (G p_bar_c)
  entmax    dz_h = u_h * (dp_h - <u_h, dp_h> / sum(u_h))
  scores    z_{h,c} = gamma q_h . s_c:  dq_h += gamma dz_h S,  ds_c += gamma dz_{h,c} q_h
  stage 0   s_c = kbar_c W_s:  dkbar_c = ds_c W_s^T,  dW_s += kbar_c^T ds_c,
            dk_j += dkbar_c / |c|  for j in c

The diagonal block's bias sigma * log(1/N) is a constant and carries no
gradient.  Blocks outside the support carry none either: their probability is
exactly 0 on a neighbourhood of the input (the support is locally constant
away from ties at the threshold).
"""

from __future__ import annotations

import math

import numpy as np

from .dash_oracle import block_summaries, candidate_blocks, forward, forward_row, route_row


def entmax_vjp(p: np.ndarray, g: np.ndarray, alpha: float) -> np.ndarray:
    """dL/dz of p = alpha-entmax(z) given g = dL/dp (Peters et al. 2019, section 3).

    On the support u_c = p_c^(2 - alpha) (u_c = 1 for alpha = 2, sparsemax);
    off the support u_c = 0.  The Jacobian diag(u) - u u^T / sum(u) is
    symmetric, so the vector-Jacobian product is u * (g - <u, g> / sum(u)).
    """
    p = np.asarray(p, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    u = np.where(p > 0.0, np.power(np.where(p > 0.0, p, 1.0), 2.0 - alpha), 0.0)
    su = u.sum()
    if su == 0.0:
        return np.zeros_like(p)
    return u * (g - (u * g).sum() / su)


def _attended(r: dict, pos: int, n_tokens: int, block: int, causal: bool, sigma: float):
    """Token ids, biases and owning list entry (-1: diagonal) of one row, as in forward_row."""
    tok, bias, owner = [], [], []
    for e, (c, lp) in enumerate(zip(r["blocks"], r["logp"])):
        span = np.arange(c * block, min(n_tokens, (c + 1) * block))
        tok.append(span)
        bias.append(np.full(len(span), sigma * lp))
        owner.append(np.full(len(span), e))
    t = pos // block
    last = pos if causal else min(n_tokens, (t + 1) * block) - 1
    span = np.arange(t * block, last + 1)
    tok.append(span)
    bias.append(np.full(len(span), sigma * r["beta"]))
    owner.append(np.full(len(span), -1))
    return np.concatenate(tok), np.concatenate(bias), np.concatenate(owner)


def backward_row(q_group: np.ndarray, k: np.ndarray, v: np.ndarray, summaries: np.ndarray, dout_group: np.ndarray,
                 pos: int, n_tokens: int, block: int, alpha: float, causal: bool = True, sigma: float = 1.0,
                 out_group: np.ndarray | None = None, key_span: tuple[int, int] | None = None) -> dict:
    """The contribution of one query position of one KV group to the gradients.

    q_group, dout_group: [G, d]; k, v: [L, d] of the KV head; summaries: all
    block summaries of that head.  Returns dq [G, d] (complete: a row's query
    gradient has no other source), the attended token ids ``tok`` with their
    dk / dv contributions [len(tok), d], and the candidate ids ``cand`` with
    their summary gradients ds [len(cand), d].

    out_group: the forward output [G, d] as an attention backward consumes
    it, D = dout . out (the softmax-gradient shortcut for sum_j P_j dP_j).
    None takes the exact output, which makes every gradient the exact
    derivative; a given (e.g. rounded) output changes D and nothing else.

    key_span: (lo, hi) to return the dk / dv contributions (and their term
    sizes) of the attended tokens in [lo, hi) only; None returns all.  The
    softmax still runs over every attended token, so what is returned is the
    same as the matching rows of the full result.

    Also returns, for error bounds of reduced-precision implementations, the
    sizes of the terms the gradients are sums of (not derivatives): the
    sums of squares dq_ss [G, d], dk_ss_tok, dv_ss_tok of the products whose
    operand dS (dq, dk) or P (dv) a tensor-core implementation rounds, and
    the sums of absolute values dq_abs, dk_abs_tok, dv_abs_tok of all terms.
    """
    q_group = np.asarray(q_group, dtype=np.float64)
    dout_group = np.asarray(dout_group, dtype=np.float64)
    G, d = q_group.shape
    scale = 1.0 / math.sqrt(d)
    gamma = 1.0 / math.sqrt(d)
    r = forward_row(q_group, k, v, summaries, pos, n_tokens, block, alpha, causal, sigma)
    tok, bias, owner = _attended(r, pos, n_tokens, block, causal, sigma)
    kt = np.arange(len(tok)) if key_span is None else np.nonzero((tok >= key_span[0]) & (tok < key_span[1]))[0]
    dq = np.zeros((G, d))
    dk_tok = np.zeros((len(kt), d))
    dv_tok = np.zeros((len(kt), d))
    dq_abs = np.zeros((G, d))
    dk_abs = np.zeros((len(kt), d))
    dv_abs = np.zeros((len(kt), d))
    dq_ss = np.zeros((G, d))
    dk_ss = np.zeros((len(kt), d))
    dv_ss = np.zeros((len(kt), d))
    dlogp = np.zeros(len(r["blocks"]))
    dlogp_abs = np.zeros(len(r["blocks"]))
    k_t, v_t = k[tok], v[tok]  # the attended keys and values, gathered once
    k_abs, k_sq = np.abs(k_t), k_t * k_t
    for h in range(G):
        logits = k_t @ q_group[h] * scale + bias
        w = np.exp(logits - logits.max())
        P = w / w.sum()
        o = P @ v_t if out_group is None else np.asarray(out_group[h], dtype=np.float64)
        dP = v_t @ dout_group[h]
        dS = P * (dP - dout_group[h] @ o)
        dq[h] += scale * (dS @ k_t)
        dk_tok += scale * np.outer(dS[kt], q_group[h])
        dv_tok += np.outer(P[kt], dout_group[h])
        mag = np.abs(dS) + P * (np.abs(dout_group[h]) @ np.abs(o))
        dq_abs[h] += scale * (mag @ k_abs)
        dk_abs += scale * np.outer(mag[kt], np.abs(q_group[h]))
        dv_abs += np.outer(P[kt], np.abs(dout_group[h]))
        dq_ss[h] += scale * scale * ((dS * dS) @ k_sq)
        dk_ss += scale * scale * np.outer(dS[kt] * dS[kt], q_group[h] * q_group[h])
        dv_ss += np.outer(P[kt] * P[kt], dout_group[h] * dout_group[h])
        listed = owner >= 0  # per list entry: the sum over the tokens of its block
        dlogp += sigma * np.bincount(owner[listed], weights=dS[listed], minlength=len(dlogp))
        dlogp_abs += sigma * np.bincount(owner[listed], weights=mag[listed], minlength=len(dlogp))
    cand = np.asarray(r["cand"], dtype=np.int64)
    ds = np.zeros((len(cand), d))
    ds_abs = np.zeros((len(cand), d))
    if len(r["blocks"]):
        # through the GQA mean p_bar = mean_h p_h and the log
        gp = np.zeros(len(cand))
        gp[r["idx"]] = dlogp / (G * r["pbar"][r["idx"]])
        gp_abs = np.zeros(len(cand))
        gp_abs[r["idx"]] = dlogp_abs / (G * r["pbar"][r["idx"]])
        for h in range(G):
            dz = entmax_vjp(r["p"][h], gp, alpha)
            dq[h] += gamma * (dz @ summaries[cand])
            ds += gamma * np.outer(dz, q_group[h])
            # magnitudes through u * (g - <u, g> / sum(u))
            u = np.where(r["p"][h] > 0.0, np.power(np.where(r["p"][h] > 0.0, r["p"][h], 1.0), 2.0 - alpha), 0.0)
            dz_abs = u * (gp_abs + (u @ gp_abs) / max(u.sum(), 1e-300))
            dq_abs[h] += gamma * (dz_abs @ np.abs(summaries[cand]))
            ds_abs += gamma * np.outer(dz_abs, np.abs(q_group[h]))
    return {"dq": dq, "tok": tok[kt], "dk_tok": dk_tok, "dv_tok": dv_tok, "cand": cand, "ds": ds,
            "dq_abs": dq_abs, "dk_abs_tok": dk_abs, "dv_abs_tok": dv_abs, "ds_abs": ds_abs,
            "dq_ss": dq_ss, "dk_ss_tok": dk_ss, "dv_ss_tok": dv_ss}


def backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, w_s: np.ndarray, dout: np.ndarray, alpha: float,
             block: int, causal: bool = True, sigma: float = 1.0, out: np.ndarray | None = None) -> dict:
    """Gradients of L = sum(dout * out) for one batch element of the prefill forward.

    q, dout: [S, H, d]; k, v: [S, Hkv, d]; w_s: [d, d].  Inputs are promoted
    to fp64.  out: the forward output [S, H, d] the backward consumes for
    D = dout . out (None: the exact output; see backward_row).  Returns dq,
    dk, dv (shapes of q, k, v) and dw_s [d, d], plus the term sizes of
    backward_row summed over the rows (dq_abs, dk_abs, dv_abs and the root
    sums of squares dq_rss, dk_rss, dv_rss).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    w_s = np.asarray(w_s, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    out = None if out is None else np.asarray(out, dtype=np.float64)
    S, H, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dw_s = np.zeros_like(w_s)
    mags = {"dq_abs": np.zeros_like(q), "dk_abs": np.zeros_like(k), "dv_abs": np.zeros_like(v),
            "dq_rss": np.zeros_like(q), "dk_rss": np.zeros_like(k), "dv_rss": np.zeros_like(v)}
    n_blocks = -(-S // block)
    for g in range(Hkv):
        kg, vg = k[:, g], v[:, g]
        summ = block_summaries(kg, w_s, block, S)
        ds = np.zeros((n_blocks, d))
        ds_abs = np.zeros((n_blocks, d))
        for pos in range(S):
            hs = slice(g * G, (g + 1) * G)
            rb = backward_row(q[pos, hs], kg, vg, summ, dout[pos, hs], pos, S, block, alpha, causal, sigma,
                              None if out is None else out[pos, hs])
            dq[pos, hs] = rb["dq"]
            dk[rb["tok"], g] += rb["dk_tok"]
            dv[rb["tok"], g] += rb["dv_tok"]
            ds[rb["cand"]] += rb["ds"]
            ds_abs[rb["cand"]] += rb["ds_abs"]
            mags["dq_abs"][pos, hs] = rb["dq_abs"]
            mags["dk_abs"][rb["tok"], g] += rb["dk_abs_tok"]
            mags["dv_abs"][rb["tok"], g] += rb["dv_abs_tok"]
            mags["dq_rss"][pos, hs] = rb["dq_ss"]
            mags["dk_rss"][rb["tok"], g] += rb["dk_ss_tok"]
            mags["dv_rss"][rb["tok"], g] += rb["dv_ss_tok"]
        # stage 0: s_c = kbar_c W_s over the c's valid tokens
        for c in range(n_blocks):
            lo, hi = c * block, min(S, (c + 1) * block)
            kbar = kg[lo:hi].sum(axis=0) / (hi - lo)
            dw_s += np.outer(kbar, ds[c])
            dk[lo:hi, g] += (w_s @ ds[c]) / (hi - lo)
            mags["dk_abs"][lo:hi, g] += (np.abs(w_s) @ ds_abs[c]) / (hi - lo)
    for name in ("dq_rss", "dk_rss", "dv_rss"):
        mags[name] = np.sqrt(mags[name])
    return {"dq": dq, "dk": dk, "dv": dv, "dw_s": dw_s, **mags}


def key_block_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, w_s: np.ndarray, dout: np.ndarray,
                       out: np.ndarray | None, blocks, block: int, alpha: float, causal: bool = True,
                       sigma: float = 1.0, rows=None) -> dict:
    """dk and dv of the tokens of some key blocks of one KV group, from every row that reaches them.

    q, dout (and out, or None for the exact output): [S, G, d] of one KV
    group; k, v: [S, d].  A key of block c receives gradient from the rows
    that attend to it (c selected, i.e. p_bar_c > 0, or c the row's own
    block) and, through stage 0, from the rows whose routing weight of c is
    non-zero (the same rows: the entmax Jacobian vanishes off the support).
    Every other row contributes exactly zero, so this is the same sum as
    :func:`backward` restricted to those tokens.  Rows are routed with
    route_row first to find the ones that reach a block.

    rows: the query positions to take into account (default: all).  Every
    returned quantity is a sum over rows, so the results of disjoint row sets
    add up to the result over their union (callers may split the rows over
    processes).

    Returns {c: {"dk", "dv", "dk_abs", "dv_abs", "dk_ss", "dv_ss"}}, each
    [tokens of c, d] (the ``_ss`` entries are the sums of squares of the
    rounded terms, whose square roots are :func:`backward`'s ``_rss``), and
    "rows": the number of rows that reached each block.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    w_s = np.asarray(w_s, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    S, G, d = q.shape
    summ = block_summaries(k, w_s, block, S)
    res, reached = {}, {}
    for c in blocks:
        n = min(S, (c + 1) * block) - c * block
        res[c] = {name: np.zeros((n, d)) for name in ("dk", "dv", "dk_abs", "dv_abs", "dk_ss", "dv_ss")}
        res[c]["ds"] = np.zeros(d)
        res[c]["ds_abs"] = np.zeros(d)
        reached[c] = 0
    for pos in (range(S) if rows is None else rows):
        t, cand = candidate_blocks(pos, block, S, causal)
        reach = [c for c in blocks if c == t]
        if any(c in cand for c in blocks):
            r = route_row(q[pos], summ[cand], alpha)
            reach += [c for c in blocks if c in cand and r["pbar"][cand.index(c)] > 0.0]
        if not reach:
            continue
        lo, hi = min(reach) * block, min(S, (max(reach) + 1) * block)
        rb = backward_row(q[pos], k, v, summ, dout[pos], pos, S, block, alpha, causal, sigma,
                          None if out is None else out[pos], key_span=(lo, hi))
        for c in reach:
            reached[c] += 1
            sel = (rb["tok"] >= c * block) & (rb["tok"] < (c + 1) * block)
            off = rb["tok"][sel] - c * block
            rc = res[c]
            rc["dk"][off] += rb["dk_tok"][sel]
            rc["dv"][off] += rb["dv_tok"][sel]
            rc["dk_abs"][off] += rb["dk_abs_tok"][sel]
            rc["dv_abs"][off] += rb["dv_abs_tok"][sel]
            rc["dk_ss"][off] += rb["dk_ss_tok"][sel]
            rc["dv_ss"][off] += rb["dv_ss_tok"][sel]
            ci = np.nonzero(rb["cand"] == c)[0]
            if len(ci):
                rc["ds"] += rb["ds"][ci[0]]
                rc["ds_abs"] += rb["ds_abs"][ci[0]]
    for c in blocks:
        rc = res[c]
        lo, hi = c * block, min(S, (c + 1) * block)
        rc["dk"] += (w_s @ rc["ds"]) / (hi - lo)
        rc["dk_abs"] += (np.abs(w_s) @ rc["ds_abs"]) / (hi - lo)
    res["rows"] = reached
    return res


def loss(q, k, v, w_s, dout, alpha, block, causal=True, sigma=1.0) -> float:
    """L = sum(dout * out) of the forward oracle (the function the gradients differentiate)."""
    out = _forward_sigma(q, k, v, w_s, alpha, block, causal, sigma)
    return float((np.asarray(dout, dtype=np.float64) * out).sum())


def _forward_sigma(q, k, v, w_s, alpha, block, causal, sigma) -> np.ndarray:
    """Whole-sequence forward with prior strength sigma, [S, H, d]."""
    if sigma == 1.0:
        return forward(q, k, v, w_s, alpha, block, causal)["out"]
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    S, H, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    out = np.zeros((S, H, d))
    for g in range(Hkv):
        summ = block_summaries(k[:, g], w_s, block, S)
        for pos in range(S):
            r = forward_row(q[pos, g * G:(g + 1) * G], k[:, g], v[:, g], summ, pos, S, block, alpha, causal, sigma)
            out[pos, g * G:(g + 1) * G] = r["out"]
    return out
