"""Plain fp64 CPU oracle of the DashAttention forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  The product
path (the CUDA library and its Python binding) never does, and this module
imports nothing from it.

Source.  The page "DashAttention: Differentiable and Adaptive Sparse
Hierarchical Attention" (gist.science explainer of arXiv 2605.18753; the ja,
hi and ar editions carry the same technical summary).  Its sections are cited
below by heading: "Stage 0: local chunk summary", "Stage 1: entmax chunk
routing", "Stage 2: prior-induced sparse softmax".  The alpha-entmax
definition follows Peters, Niculae & Martins (2019), "Sparse
Sequence-to-Sequence Models"; sparsemax (alpha = 2) is Martins & Astudillo
(2016).

Everything is computed in fp64 from the stored input values, one query row
at a time, in the order the pages give the steps.  Readings of points that
the pages leave open (all fixed here and in the CUDA path alike):

* gamma, the routing temperature in "w = alpha-entmax(gamma z)", is
  1/sqrt(d).
* The summary of block c is the mean of its keys times W_s, taken as a row
  vector times the matrix: s_c = mean_j(k_j) @ W_s.  The learned-query form
  (block_summaries_sdpa) weights the keys by softmax(q_bar . k_j / sqrt(d))
  over the block, with one q_bar per KV head; q_bar = 0 is the mean.
* Causal: the candidates of a query at position pos are the complete blocks
  before its own block t = pos // B (N = t of them); the own block is the
  always-included "diagonal" block, masked to tokens <= pos.  Non-causal:
  every other block is a candidate (a trailing partial block is pooled over
  its valid tokens) and the own block is included whole.
* The diagonal block's prior is the uniform baseline, bias log(1/N) (0 when
  N = 0), so that selecting every block with a uniform prior reproduces full
  attention exactly.
* Under GQA each query head runs its own entmax; the mean over the heads of
  a KV group is the shared support and the shared prior.
* A block is selected iff its group-mean probability is > 0 (strictly).
* The prior strength sigma is 1.
"""

from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


# --------------------------------------------------------------------------
# Stage 0


def block_summaries(k: np.ndarray, w_s: np.ndarray, block: int, n_tokens: int) -> np.ndarray:
    """Stage 0 ("Stage 0: local chunk summary").

    The context is cut into contiguous chunks of ``block`` tokens.  The pages'
    summariser is a learned query attending to the chunk's keys; at its zero
    initialisation that is uniform mean pooling, which is what is computed
    here, followed by the fixed projection W_s:  s_c = (1/|c|) sum_{j in c} k_j @ W_s.

    k: [L, d] keys of one (batch, KV head); only tokens < n_tokens exist.
    Returns [ceil(n_tokens / block), d]; a trailing partial block is the mean
    over its valid tokens.
    """
    k = np.asarray(k, dtype=np.float64)
    w_s = np.asarray(w_s, dtype=np.float64)
    n_blocks = -(-n_tokens // block)
    out = np.zeros((n_blocks, k.shape[1]))
    for c in range(n_blocks):
        lo, hi = c * block, min(n_tokens, (c + 1) * block)
        mean = k[lo:hi].sum(axis=0) / (hi - lo)
        out[c] = mean @ w_s
    return out


def block_summaries_sdpa(k: np.ndarray, w_s: np.ndarray, qbar: np.ndarray, block: int, n_tokens: int) -> np.ndarray:
    """Stage 0 with the learned summary query ("Stage 0: local chunk summary").

    The pages' summariser: a learned query vector q_bar attends to the keys of
    each chunk through local scaled dot-product attention, and the keys are
    what it averages (the summary lives in key space, so stage 1 can score
    queries against it).  For block c with valid tokens j:

        a_j = q_bar . k_j / sqrt(d),   w = softmax(a) over the block,
        s_c = (sum_j w_j k_j) @ W_s.

    q_bar = 0 gives uniform weights, i.e. block_summaries (the pages' zero
    initialisation).  k: [L, d] keys of one (batch, KV head); qbar: [d], the
    query of that KV head.  Returns [ceil(n_tokens / block), d].
    """
    k = np.asarray(k, dtype=np.float64)
    w_s = np.asarray(w_s, dtype=np.float64)
    qbar = np.asarray(qbar, dtype=np.float64)
    d = k.shape[1]
    n_blocks = -(-n_tokens // block)
    out = np.zeros((n_blocks, d))
    for c in range(n_blocks):
        lo, hi = c * block, min(n_tokens, (c + 1) * block)
        a = k[lo:hi] @ qbar / math.sqrt(d)
        w = np.exp(a - a.max())
        w /= w.sum()
        out[c] = (w @ k[lo:hi]) @ w_s
    return out


# --------------------------------------------------------------------------
# alpha-entmax


def _support_tau(top: np.ndarray, alpha: float) -> float | None:
    """tau with sum_r (top_r - tau)^(1/(alpha-1)) = 1 and tau < min(top), or None.

    ``top`` are the k largest values of x = (alpha-1) z, descending.
    """
    k = len(top)
    if alpha == 2.0:
        tau = (top.sum() - 1.0) / k
    elif alpha == 1.5:
        mean = top.mean()
        ss = ((top - mean) ** 2).sum()  # k * variance
        if ss > 1.0:
            return None
        tau = mean - math.sqrt((1.0 - ss) / k)
    else:
        p = 1.0 / (alpha - 1.0)

        def f(t):
            return float((np.maximum(top - t, 0.0) ** p).sum()) - 1.0

        lo, hi = top[0] - 1.0, top[-1]
        if f(hi) >= 0.0:
            return None
        for _ in range(200):
            mid = 0.5 * (lo + hi)
            if f(mid) > 0.0:
                lo = mid
            else:
                hi = mid
        tau = 0.5 * (lo + hi)
    return tau if tau < top[-1] else None


def entmax_threshold(x: np.ndarray, alpha: float) -> float:
    """Exact threshold tau of alpha-entmax on x = (alpha - 1) * z.

    Sort x descending; for each support size k solve the normalisation on the
    top k and keep the k whose tau separates the support:
    x_(k) > tau >= x_(k+1).  For alpha = 2 (sparsemax) and alpha = 1.5 the
    per-k solve has a closed form in the running sums of x and x^2 and all k
    are evaluated at once; other alpha solve each k by fp64 bisection.
    """
    xs = np.sort(np.asarray(x, dtype=np.float64))[::-1]
    n = len(xs)
    nxt = np.append(xs[1:], NEG_INF)
    if alpha in (2.0, 1.5):
        k = np.arange(1, n + 1, dtype=np.float64)
        s1 = np.cumsum(xs)
        if alpha == 2.0:
            tau = (s1 - 1.0) / k
        else:
            mean = s1 / k
            ss = np.cumsum(xs * xs) - k * mean * mean  # k * variance of the top k
            with np.errstate(invalid="ignore"):
                tau = mean - np.sqrt((1.0 - ss) / k)
        ok = (xs > tau) & (tau >= nxt)
        if ok.any():
            return float(tau[np.argmax(ok)])
        raise ArithmeticError("no self-consistent entmax support")
    for k in range(1, n + 1):
        tau = _support_tau(xs[:k], alpha)
        if tau is not None and xs[k - 1] > tau >= nxt[k - 1]:
            return tau
    raise ArithmeticError("no self-consistent entmax support")


def entmax_threshold_bisect(x: np.ndarray, alpha: float, iters: int = 200) -> float:
    """Second, independent tau: bisection of sum_c [x_c - tau]_+^(1/(alpha-1)) = 1.

    The root lies in [max(x) - 1, max(x) - n^(1 - alpha)] (the two ends are the
    one-hot and the uniform solutions).
    """
    x = np.asarray(x, dtype=np.float64)
    p = 1.0 / (alpha - 1.0)
    n = len(x)
    lo, hi = x.max() - 1.0, x.max() - n ** (1.0 - alpha)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if (np.maximum(x - mid, 0.0) ** p).sum() > 1.0:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def entmax(z: np.ndarray, alpha: float) -> tuple[np.ndarray, float]:
    """alpha-entmax(z) ("Stage 1: entmax chunk routing"), 1 < alpha <= 2.

    The maximiser of <p, z> + H_alpha(p) over the simplex, with the Tsallis
    entropy H_alpha(p) = sum_j (p_j - p_j^alpha) / (alpha (alpha - 1)).  Its
    solution is p_j = [(alpha - 1) z_j - tau]_+^(1/(alpha-1)); the number of
    non-zeros depends on z.  Returns (p, tau) with tau on the x = (alpha-1) z
    scale.
    """
    if not 1.0 < alpha <= 2.0:
        raise ValueError("alpha must be in (1, 2]")
    x = (alpha - 1.0) * np.asarray(z, dtype=np.float64)
    tau = entmax_threshold(x, alpha)
    p = np.maximum(x - tau, 0.0) ** (1.0 / (alpha - 1.0))
    return p, tau


# --------------------------------------------------------------------------
# Stage 1 for one query row


def route_row(q_group: np.ndarray, summaries: np.ndarray, alpha: float) -> dict:
    """Stage 1 for one query position and one KV group.

    q_group: [G, d] the G query heads sharing the KV head; summaries: [N, d]
    the candidate block summaries.  Each head scores the candidates
    (z = gamma q . s_c, gamma = 1/sqrt(d)), runs alpha-entmax, and the heads'
    probabilities are averaged ("GQA handling" under "Stage 1") into p_bar,
    whose support is the selected block list (ascending) with log p_bar as
    the prior.
    """
    q_group = np.asarray(q_group, dtype=np.float64)
    G, d = q_group.shape
    n = len(summaries)
    gamma = 1.0 / math.sqrt(d)
    z = np.zeros((G, n))
    p = np.zeros((G, n))
    tau = np.zeros(G)
    for h in range(G):
        z[h] = gamma * (np.asarray(summaries, dtype=np.float64) @ q_group[h])
        if n > 0:
            p[h], tau[h] = entmax(z[h], alpha)
    pbar = p.mean(axis=0) if n > 0 else np.zeros(0)
    idx = np.array([c for c in range(n) if pbar[c] > 0.0], dtype=np.int64)
    return {
        "z": z, "x": (alpha - 1.0) * z, "tau": tau, "p": p, "pbar": pbar,
        "idx": idx, "logp": np.log(pbar[idx]) if len(idx) else np.zeros(0),
    }


# --------------------------------------------------------------------------
# Stage 2


def prior_softmax_attend(q: np.ndarray, keys: np.ndarray, values: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """Prior-induced softmax ("Stage 2: prior-induced sparse softmax").

    softmax maximises <p, l> - KL(p || u); with the reference u replaced by a
    prior g the maximiser is softmax(l + log g).  Here l_j = q . k_j / sqrt(d)
    and bias_j = log g_j (-inf where g_j = 0, i.e. a masked token).
    Returns sum_j softmax(l + bias)_j v_j, with max-subtraction, in fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    logits = np.asarray(keys, dtype=np.float64) @ q / math.sqrt(d) + np.asarray(bias, dtype=np.float64)
    m = logits.max()
    w = np.exp(logits - m)
    return (w[:, None] * np.asarray(values, dtype=np.float64)).sum(axis=0) / w.sum()


def diagonal_bias(n_candidates: int) -> float:
    """Prior of the always-included diagonal block: uniform baseline log(1/N), 0 if N = 0."""
    return math.log(1.0 / n_candidates) if n_candidates > 0 else 0.0


def candidate_blocks(pos: int, block: int, n_tokens: int, causal: bool) -> tuple[int, list[int]]:
    """(own block t, candidate block ids) for a query at ``pos``."""
    t = pos // block
    if causal:
        return t, list(range(t))
    n_blocks = -(-n_tokens // block)
    return t, [c for c in range(n_blocks) if c != t]


def forward_row(q_group: np.ndarray, k: np.ndarray, v: np.ndarray, summaries: np.ndarray,
                pos: int, n_tokens: int, block: int, alpha: float, causal: bool = True,
                sigma: float = 1.0) -> dict:
    """Stages 1 and 2 for one query position of one KV group.

    q_group: [G, d]; k, v: [L, d] of the KV head; summaries: all block
    summaries of that head (stage 0); n_tokens: valid context length.
    sigma: strength of the prior ("Stage 2: prior-induced sparse softmax"
    names a strength that balances the prior against the uniform baseline):
    the bias is sigma * log p_bar on the selected blocks and sigma * log(1/N)
    on the diagonal block, so a uniform prior still gives full attention for
    every sigma, and sigma = 0 is plain softmax over the selected tokens.
    Returns the route dict of :func:`route_row` (with ``idx`` as block ids)
    plus ``beta`` and ``out`` [G, d].
    """
    t, cand = candidate_blocks(pos, block, n_tokens, causal)
    r = route_row(q_group, summaries[cand] if cand else np.zeros((0, q_group.shape[1])), alpha)
    sel = [cand[i] for i in r["idx"]]
    beta = diagonal_bias(len(cand))
    tok, bias = [], []
    for c, lp in zip(sel, r["logp"]):
        span = np.arange(c * block, min(n_tokens, (c + 1) * block))
        tok.append(span)
        bias.append(np.full(len(span), sigma * lp))
    last = pos if causal else min(n_tokens, (t + 1) * block) - 1
    span = np.arange(t * block, last + 1)
    tok.append(span)
    bias.append(np.full(len(span), sigma * beta))
    tok = np.concatenate(tok)
    bias = np.concatenate(bias)
    k_t, v_t = k[tok], v[tok]  # the attended keys and values, gathered once for the G heads
    out = np.stack([prior_softmax_attend(q_group[h], k_t, v_t, bias) for h in range(len(q_group))])
    r.update({"blocks": np.array(sel, dtype=np.int64), "cand": cand, "beta": beta, "out": out})
    return r


def lists_to_mask(idx: np.ndarray, cnt: np.ndarray, n_words: int) -> np.ndarray:
    """Bit-packed active-block mask (the pages' kernel walks such a mask of the
    active chunks): word w of a row has bit b set iff block 32 w + b is among
    the row's cnt selected blocks.  idx [..., t_cap], cnt [...] -> [..., n_words] uint32."""
    idx = np.asarray(idx)
    cnt = np.asarray(cnt)
    out = np.zeros(cnt.shape + (n_words,), dtype=np.uint32)
    for pos in np.ndindex(cnt.shape):
        for c in idx[pos][: int(cnt[pos])]:
            out[pos + (int(c) // 32,)] |= np.uint32(1 << (int(c) % 32))
    return out


def forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, w_s: np.ndarray, alpha: float, block: int,
            causal: bool = True, rows=None) -> dict:
    """Whole prefill forward for one batch element.

    q: [S, H, d], k, v: [S, Hkv, d] (any float dtype; promoted to fp64).
    rows: query positions to evaluate (default: all).  Returns out
    [len(rows), H, d] and per (row, KV group) routing records.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    S, H, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    rows = list(range(S)) if rows is None else list(rows)
    out = np.zeros((len(rows), H, d))
    routes = {}
    for g in range(Hkv):
        summ = block_summaries(k[:, g], w_s, block, S)
        for ri, pos in enumerate(rows):
            r = forward_row(q[pos, g * G:(g + 1) * G], k[:, g], v[:, g], summ, pos, S, block, alpha, causal)
            out[ri, g * G:(g + 1) * G] = r.pop("out")
            routes[(pos, g)] = r
    return {"out": out, "routes": routes, "rows": rows}


def decode_pair(q_group: np.ndarray, k: np.ndarray, v: np.ndarray, w_s: np.ndarray, seqlen: int,
                block: int, alpha: float) -> dict:
    """One decode step for one (sequence, KV group): the query sits at pos = seqlen - 1.

    The candidates are the complete blocks before the query's block; their
    summaries are the cached stage-0 summaries (computed here from k).
    """
    pos = seqlen - 1
    n_complete = pos // block
    summ = block_summaries(k[: n_complete * block], w_s, block, n_complete * block)
    return forward_row(q_group, k, v, summ, pos, seqlen, block, alpha, causal=True)
