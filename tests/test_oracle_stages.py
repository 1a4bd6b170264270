"""Pins of the oracle's stage 0, GQA routing, stage 2 and the end-to-end forward.

Cited page: "DashAttention: Differentiable and Adaptive Sparse Hierarchical
Attention" (gist.science explainer), technical summary, sections "Stage 0:
local chunk summary", "Stage 1: entmax chunk routing" (GQA handling) and
"Stage 2: prior-induced sparse softmax".  The independent references here are
hand-computed values, library routines (numpy means, torch's
scaled_dot_product_attention in fp64, scipy's optimiser) and invariances.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.optimize import minimize

from scipy.special import expit

from oracle.dash_oracle import (
    block_summaries,
    block_summaries_sdpa,
    decode_pair,
    diagonal_bias,
    forward,
    forward_row,
    lists_to_mask,
    prior_softmax_attend,
    route_row,
)


# --------------------------------------------------------------------------
# Stage 0


def test_block_mean_hand_example():
    # two blocks of 2 tokens, d = 2, W_s = I: means by hand
    k = np.array([[1.0, 2.0], [3.0, 6.0], [-1.0, 0.0], [5.0, 4.0], [7.0, 7.0]])
    s = block_summaries(k, np.eye(2), block=2, n_tokens=5)
    np.testing.assert_array_equal(s, [[2.0, 4.0], [2.0, 2.0], [7.0, 7.0]])


def test_block_mean_matches_numpy_and_orientation():
    rng = np.random.default_rng(0)
    L, d, B = 640, 16, 64
    k = rng.normal(size=(L, d))
    s = block_summaries(k, np.eye(d), B, L)
    np.testing.assert_allclose(s, k.reshape(L // B, B, d).mean(axis=1), atol=1e-14)
    # row vector times matrix: a permutation W_s (W[i, pi(i)] = 1) moves
    # coordinate i of the mean to position pi(i); the transpose would not.
    perm = rng.permutation(d)
    w = np.zeros((d, d))
    w[np.arange(d), perm] = 1.0
    s2 = block_summaries(k, w, B, L)
    np.testing.assert_allclose(s2[:, perm], s, atol=1e-14)
    # a partial trailing block is averaged over its valid tokens only
    s3 = block_summaries(k, np.eye(d), B, 600)
    np.testing.assert_allclose(s3[-1], k[576:600].mean(axis=0), atol=1e-14)


def test_sdpa_summary_hand_example():
    # d = 2, W_s = I, one block of two orthogonal keys; q_bar chosen so the
    # scaled scores are (ln 3, 0): weights 3/4 and 1/4
    k = np.array([[1.0, 0.0], [0.0, 1.0]])
    qbar = np.array([math.sqrt(2.0) * math.log(3.0), 0.0])
    s = block_summaries_sdpa(k, np.eye(2), qbar, block=2, n_tokens=2)
    np.testing.assert_allclose(s, [[0.75, 0.25]], atol=1e-15)


def test_sdpa_summary_zero_query_is_mean_pooling():
    # the pages' zero initialisation behaves as uniform mean pooling
    rng = np.random.default_rng(3)
    L, d, B = 700, 32, 64
    k = rng.normal(size=(L, d))
    w = np.eye(d) + 0.1 * rng.normal(size=(d, d))
    np.testing.assert_allclose(block_summaries_sdpa(k, w, np.zeros(d), B, L), block_summaries(k, w, B, L),
                               atol=1e-13)


def test_sdpa_summary_two_token_logistic_form():
    # two tokens: s = sigmoid(a) k1 + sigmoid(-a) k2 with a = q_bar.(k1 - k2)/sqrt(d)
    rng = np.random.default_rng(4)
    d = 8
    for _ in range(20):
        k = rng.normal(size=(2, d))
        qbar = 3.0 * rng.normal(size=d)
        a = qbar @ (k[0] - k[1]) / math.sqrt(d)
        ref = expit(a) * k[0] + expit(-a) * k[1]
        np.testing.assert_allclose(block_summaries_sdpa(k, np.eye(d), qbar, 2, 2)[0], ref, atol=1e-13)


def test_sdpa_summary_invariances_and_limits():
    rng = np.random.default_rng(5)
    d, B = 16, 8
    w = rng.normal(size=(d, d))
    # identical keys: the summary is that key whatever the query
    k = np.tile(rng.normal(size=(1, d)), (B, 1))
    np.testing.assert_allclose(block_summaries_sdpa(k, w, 50.0 * rng.normal(size=d), B, B)[0], k[0] @ w,
                               atol=1e-12)
    # permuting the tokens of a block changes nothing
    k = rng.normal(size=(B, d))
    qbar = rng.normal(size=d)
    s = block_summaries_sdpa(k, w, qbar, B, B)
    np.testing.assert_allclose(block_summaries_sdpa(k[rng.permutation(B)], w, qbar, B, B), s, atol=1e-13)
    # a query aligned ever more strongly with one key selects that key
    m = 5
    far = block_summaries_sdpa(k, w, 1e4 * k[m], B, B)[0]
    np.testing.assert_allclose(far, k[m] @ w, atol=1e-9)
    # a partial trailing block weights only its valid tokens
    k = rng.normal(size=(3 * B, d))
    s = block_summaries_sdpa(k, np.eye(d), qbar, B, 2 * B + 3)
    np.testing.assert_allclose(s[-1], block_summaries_sdpa(k[2 * B:2 * B + 3], np.eye(d), qbar, B, 3)[0],
                               atol=1e-14)


# --------------------------------------------------------------------------
# Stage 1: GQA average


def test_gqa_average_hand_example():
    # d = 4, gamma = 1/2.  Head 0 is one-hot on block 0, head 1 on block 2.
    summaries = np.eye(4)[:3] * 10.0
    q = np.array([[1.0, 0, 0, 0], [0, 0, 1.0, 0]])
    r = route_row(q, summaries, alpha=1.5)
    np.testing.assert_allclose(r["p"], [[1, 0, 0], [0, 0, 1]], atol=0)
    np.testing.assert_allclose(r["pbar"], [0.5, 0.0, 0.5])
    np.testing.assert_array_equal(r["idx"], [0, 2])
    np.testing.assert_allclose(r["logp"], [math.log(0.5)] * 2)
    # z = gamma q.s with gamma = 1/sqrt(d)
    np.testing.assert_allclose(r["z"][0], [5.0, 0.0, 0.0])


# --------------------------------------------------------------------------
# Stage 2


def test_prior_softmax_is_the_variational_maximiser():
    """softmax(l + log g) maximises <p, l> - KL(p || g) (scipy cross-check)."""
    rng = np.random.default_rng(1)
    n, d = 6, 8
    q = rng.normal(size=d)
    keys = rng.normal(size=(n, d))
    g = rng.dirichlet(np.ones(n))
    logits = keys @ q / math.sqrt(d)
    # with values = identity rows the output is the attention distribution
    p = prior_softmax_attend(q, keys, np.eye(n), np.log(g))

    def obj(u):
        u = np.clip(u, 1e-300, None)
        return float(u @ logits - np.sum(u * np.log(u / g)))

    res = minimize(lambda u: -obj(u), np.full(n, 1.0 / n), method="SLSQP",
                   bounds=[(1e-12, 1.0)] * n,
                   constraints=[{"type": "eq", "fun": lambda u: u.sum() - 1.0}],
                   options={"ftol": 1e-15, "maxiter": 1000})
    np.testing.assert_allclose(p, res.x, atol=1e-5)
    assert obj(p) >= -res.fun - 1e-12


def test_bias_shift_and_masking():
    rng = np.random.default_rng(2)
    n, d = 40, 16
    q, keys, vals = rng.normal(size=d), rng.normal(size=(n, d)), rng.normal(size=(n, d))
    bias = rng.normal(size=n)
    o = prior_softmax_attend(q, keys, vals, bias)
    np.testing.assert_allclose(prior_softmax_attend(q, keys, vals, bias + 3.5), o, atol=1e-14)
    # a -inf prior (g = 0) removes the token exactly
    bias_m = bias.copy()
    bias_m[5:15] = -np.inf
    keep = np.r_[0:5, 15:n]
    np.testing.assert_allclose(prior_softmax_attend(q, keys, vals, bias_m),
                               prior_softmax_attend(q, keys[keep], vals[keep], bias[keep]), atol=1e-14)


def _sdpa(q, k, v, causal):
    """torch fp64 scaled_dot_product_attention; q [S,H,d], k/v [S,Hkv,d]."""
    S, H, d = q.shape
    G = H // k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)
    kt = torch.from_numpy(np.repeat(k, G, axis=1)).permute(1, 0, 2)
    vt = torch.from_numpy(np.repeat(v, G, axis=1)).permute(1, 0, 2)
    return F.scaled_dot_product_attention(qt, kt, vt, is_causal=causal).permute(1, 0, 2).numpy()


@pytest.mark.parametrize("causal", [True, False])
def test_zero_w_s_is_full_attention(causal):
    """W_s = 0 makes every score 0, entmax uniform over the N candidates, every
    prior log(1/N) equal to the diagonal prior: the forward is plain attention."""
    rng = np.random.default_rng(3)
    S, H, Hkv, d, B = 203, 4, 2, 16, 16  # ragged tail: 203 = 12 * 16 + 11
    q, k, v = rng.normal(size=(S, H, d)), rng.normal(size=(S, Hkv, d)), rng.normal(size=(S, Hkv, d))
    res = forward(q, k, v, np.zeros((d, d)), alpha=1.5, block=B, causal=causal)
    np.testing.assert_allclose(res["out"], _sdpa(q, k, v, causal), atol=1e-12)
    for (pos, g), r in res["routes"].items():
        assert len(r["blocks"]) == len(r["cand"])
        assert r["beta"] == diagonal_bias(len(r["cand"]))


@pytest.mark.parametrize("sigma", [0.0, 0.3, 2.5])
def test_uniform_prior_is_full_attention_for_any_sigma(sigma):
    """Tempering scales every bias by sigma; with a uniform prior all biases are
    equal, so the forward is plain causal attention whatever sigma is."""
    rng = np.random.default_rng(8)
    S, G, d, B = 150, 2, 16, 16
    q, k, v = rng.normal(size=(S, G, d)), rng.normal(size=(S, 1, d)), rng.normal(size=(S, 1, d))
    summ = np.zeros((-(-S // B), d))  # zero summaries: every candidate uniform
    ref = _sdpa(q, k, v, True)
    for pos in (0, 17, 64, 149):
        r = forward_row(q[pos], k[:, 0], v[:, 0], summ, pos, S, B, 1.5, True, sigma=sigma)
        np.testing.assert_allclose(r["out"], ref[pos], atol=1e-12)


def test_sigma_zero_is_softmax_over_the_selected_tokens():
    """sigma = 0 drops the prior: masked scaled dot-product attention (torch, fp64)
    over the tokens of the selected blocks and the causal diagonal block."""
    rng = np.random.default_rng(9)
    S, G, d, B = 300, 3, 16, 16
    q, k, v = rng.normal(size=(S, G, d)), rng.normal(size=(S, d)), rng.normal(size=(S, d))
    for b in range(4):  # plant a few strong blocks so the selection is sparse
        k[b * 3 * B:(b * 3 + 1) * B] += 3.0 * q[299, 0] / np.linalg.norm(q[299, 0])
    summ = block_summaries(k, np.eye(d), B, S)
    sparse = []
    for pos in (100, 255, 299):
        r = forward_row(q[pos], k, v, summ, pos, S, B, 1.5, True, sigma=0.0)
        t = pos // B
        allowed = np.zeros(S, dtype=bool)
        for c in r["blocks"]:
            allowed[c * B:(c + 1) * B] = True
        allowed[t * B:pos + 1] = True
        sparse.append(bool(allowed.sum() < pos + 1))
        qq = torch.from_numpy(q[pos])[:, None, :]
        kk = torch.from_numpy(k)[None].expand(G, S, d)
        vv = torch.from_numpy(v)[None].expand(G, S, d)
        ref = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=torch.from_numpy(allowed)[None, None, :])
        np.testing.assert_allclose(r["out"], ref[:, 0].numpy(), atol=1e-12)
    assert any(sparse)  # the selection skipped blocks for some row


def test_lists_to_mask():
    idx = np.array([[[0, 5, 31, 32, 70, -1], [3, -1, -1, -1, -1, -1]]])
    cnt = np.array([[5, 1]])
    m = lists_to_mask(idx, cnt, 3)
    assert m.shape == (1, 2, 3) and m.dtype == np.uint32
    assert m[0, 0].tolist() == [(1 << 0) | (1 << 5) | (1 << 31), 1 << 0, 1 << 6]
    assert m[0, 1].tolist() == [1 << 3, 0, 0]
    # round trip against the set of listed blocks
    rng = np.random.default_rng(2)
    idx = np.sort(rng.choice(100, size=(4, 40), replace=True), axis=1)
    idx = np.stack([np.unique(r)[:30] if len(np.unique(r)) >= 30 else np.pad(np.unique(r), (0, 30 - len(np.unique(r))))
                    for r in idx])
    cnt = np.array([len(set(r.tolist())) if len(set(r.tolist())) < 30 else 30 for r in idx])
    m = lists_to_mask(idx, cnt, 4)
    for r in range(4):
        bits = np.unpackbits(m[r].view(np.uint8), bitorder="little")
        assert set(np.nonzero(bits)[0].tolist()) == set(idx[r][: cnt[r]].tolist())


def test_first_block_rows_attend_within_the_block():
    rng = np.random.default_rng(4)
    S, d, B = 64, 8, 32
    q, k, v = rng.normal(size=(S, 1, d)), rng.normal(size=(S, 1, d)), rng.normal(size=(S, 1, d))
    w = rng.normal(size=(d, d))
    res = forward(q, k, v, w, alpha=1.5, block=B, rows=range(B))
    np.testing.assert_allclose(res["out"], _sdpa(q[:B], k[:B], v[:B], True), atol=1e-12)


def test_unselected_values_do_not_matter():
    """Perturbing V inside blocks with zero routing mass leaves the output unchanged."""
    rng = np.random.default_rng(5)
    S, d, B = 512, 16, 32
    q, k, v = rng.normal(size=(S, 1, d)), rng.normal(size=(S, 1, d)), rng.normal(size=(S, 1, d))
    e = np.eye(d)[3]
    k[64:96, 0] += 6.0 * e  # block 2 planted
    q[480:, 0] += 6.0 * e
    w = np.eye(d)
    pos = 500
    summ = block_summaries(k[:, 0], w, B, S)
    r = forward_row(q[pos], k[:, 0], v[:, 0], summ, pos, S, B, 1.5)
    assert 2 in r["blocks"] and len(r["blocks"]) < len(r["cand"])
    unsel = [c for c in r["cand"] if c not in set(r["blocks"].tolist())]
    v2 = v.copy()
    for c in unsel:
        v2[c * B:(c + 1) * B] += rng.normal(size=(B, 1, d)) * 100.0
    r2 = forward_row(q[pos], k[:, 0], v2[:, 0], summ, pos, S, B, 1.5)
    np.testing.assert_array_equal(r2["out"], r["out"])


def test_decode_pair_zero_w_s_is_attention_over_context():
    rng = np.random.default_rng(6)
    L, d, B, G = 300, 16, 32, 2
    q = rng.normal(size=(G, d))
    k, v = rng.normal(size=(L + 50, d)), rng.normal(size=(L + 50, d))
    r = decode_pair(q, k, v, np.zeros((d, d)), seqlen=L, block=B, alpha=2.0)
    logits = q @ k[:L].T / math.sqrt(d)
    w = np.exp(logits - logits.max(axis=1, keepdims=True))
    ref = (w / w.sum(axis=1, keepdims=True)) @ v[:L]
    np.testing.assert_allclose(r["out"], ref, atol=1e-12)
    assert len(r["cand"]) == (L - 1) // B


def _prior_mask_reference(q_group, k, v, summ, pos, n_tokens, block, alpha, causal, sigma, shift=0):
    """torch fp64 SDPA with an additive float mask that carries the prior token by token.

    p_bar comes from route_row (pinned on its own) over the candidates' summaries; entry i of
    that vector belongs to block cand[i].  ``shift`` = 1 instead attaches it to block i, the
    mistake this reference must catch (it differs from cand[i] once i passes the query's own
    block in non-causal mode)."""
    t = pos // block
    n_blocks = -(-n_tokens // block)
    cand = list(range(t)) if causal else [c for c in range(n_blocks) if c != t]
    r = route_row(q_group, summ[cand], alpha)
    mask = np.full(n_tokens, -np.inf)
    for i, c in enumerate(cand):
        owner = i if shift else c
        if r["pbar"][i] > 0.0:
            lo, hi = owner * block, min(n_tokens, (owner + 1) * block)
            mask[lo:hi] = sigma * math.log(r["pbar"][i])
    last = pos if causal else min(n_tokens, (t + 1) * block) - 1
    mask[t * block:last + 1] = sigma * (math.log(1.0 / len(cand)) if cand else 0.0)
    G, d = q_group.shape
    qq = torch.from_numpy(q_group)[:, None, :]
    kk = torch.from_numpy(k)[None].expand(G, n_tokens, d)
    vv = torch.from_numpy(v)[None].expand(G, n_tokens, d)
    am = torch.from_numpy(mask)[None, None, :].expand(G, 1, n_tokens)
    return F.scaled_dot_product_attention(qq, kk, vv, attn_mask=am)[:, 0].numpy(), r


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("sigma", [0.5, 1.0, 2.0])
def test_non_uniform_prior_lands_on_its_block(causal, sigma):
    """The prior of "Stage 2: prior-induced sparse softmax" with a sparse, non-uniform p_bar:
    every token of selected block c carries sigma * log p_bar_c, the diagonal block carries
    sigma * log(1/N), every other token is masked.  forward_row must equal fp64 SDPA with that
    additive mask, built here by block id from route_row's p_bar."""
    rng = np.random.default_rng(11)
    S, G, d, B = 610, 2, 16, 32  # 20 blocks, ragged tail of 2 tokens
    k, v = rng.normal(size=(S, d)), rng.normal(size=(S, d))
    dirs = np.linalg.qr(rng.normal(size=(d, 4)))[0].T
    # planted blocks of graded strength on both sides of the query blocks used below
    for c, (e, s) in {1: (0, 2.0), 4: (0, 3.0), 6: (1, 2.5), 11: (0, 2.2), 15: (1, 3.5), 17: (0, 2.8)}.items():
        k[c * B:(c + 1) * B] += s * dirs[e]
    w = np.eye(d) + 0.1 * rng.normal(size=(d, d))
    summ = block_summaries(k, w, B, S)
    q = rng.normal(size=(S, G, d))
    q[:, 0] += 4.0 * dirs[0]
    q[:, 1] += 4.0 * dirs[1]
    checked = 0
    for pos in (100, 300, 333, 420, 609):
        r = forward_row(q[pos], k, v, summ, pos, S, B, 1.5, causal, sigma=sigma)
        ref, rr = _prior_mask_reference(q[pos], k, v, summ, pos, S, B, 1.5, causal, sigma)
        np.testing.assert_allclose(r["out"], ref, atol=1e-12)
        sel = rr["pbar"][rr["pbar"] > 0]
        if len(sel) >= 2 and len(sel) < len(rr["pbar"]) and np.ptp(sel) > 1e-3:
            checked += 1  # a sparse and non-uniform prior
            if not causal and pos // B < int(np.nonzero(rr["pbar"])[0].max()) + 1:
                wrong, _ = _prior_mask_reference(q[pos], k, v, summ, pos, S, B, 1.5, causal, sigma, shift=1)
                assert np.abs(wrong - ref).max() > 1e-3  # the reference tells the two placements apart
    assert checked >= 3


def test_candidate_blocks_enumerated():
    """Candidates of "Stage 1": causal rows score the complete blocks before
    their own; non-causal rows every other block, the ragged last one included."""
    from oracle.dash_oracle import candidate_blocks

    assert candidate_blocks(0, 64, 1000, True) == (0, [])
    assert candidate_blocks(63, 64, 1000, True) == (0, [])
    assert candidate_blocks(64, 64, 1000, True) == (1, [0])
    assert candidate_blocks(130, 64, 200, True) == (2, [0, 1])
    # 200 tokens in blocks of 64: blocks 0, 1, 2 full, block 3 holds tokens 192..199
    assert candidate_blocks(130, 64, 200, False) == (2, [0, 1, 3])
    assert candidate_blocks(199, 64, 200, False) == (3, [0, 1, 2])
    assert candidate_blocks(5, 64, 200, False) == (0, [1, 2, 3])
    assert candidate_blocks(5, 64, 64, False) == (0, [])
    assert candidate_blocks(300, 128, 1024, True) == (2, [0, 1])
