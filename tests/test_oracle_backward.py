"""Pins of the oracle's backward pass.

Cited page: "DashAttention: Differentiable and Adaptive Sparse Hierarchical
Attention" (gist.science explainer), sections "Stage 1: entmax chunk routing"
and "Stage 2: prior-induced sparse softmax"; the entmax Jacobian is from
Peters, Niculae & Martins (2019), section 3, and the sparsemax Jacobian from
Martins & Astudillo (2016), section 2.5.  The independent references are
central finite differences of the (separately pinned) forward oracle in
fp64, the sparsemax closed form, torch autograd of
scaled_dot_product_attention in fp64, and invariances.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle.backward import backward, entmax_vjp, loss
from oracle.dash_oracle import entmax, forward


def _fd_entmax(z, g, alpha, eps=1e-6):
    out = np.zeros_like(z)
    for c in range(len(z)):
        zp, zm = z.copy(), z.copy()
        zp[c] += eps
        zm[c] -= eps
        out[c] = (g @ entmax(zp, alpha)[0] - g @ entmax(zm, alpha)[0]) / (2 * eps)
    return out


@pytest.mark.parametrize("alpha", [1.25, 1.5, 1.75, 2.0])
def test_entmax_vjp_matches_finite_differences(alpha):
    rng = np.random.default_rng(int(alpha * 100))
    partial = 0
    for _ in range(20):
        z = rng.normal(scale=3.0, size=10)
        g = rng.normal(size=10)
        p, _ = entmax(z, alpha)
        partial += 1 < (p > 0).sum() < len(z)
        np.testing.assert_allclose(entmax_vjp(p, g, alpha), _fd_entmax(z, g, alpha), atol=1e-7)
    assert partial >= 5  # the cases exercise supports strictly between one-hot and full


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_entmax_vjp_is_shift_invariant(alpha):
    # p(z + c 1) = p(z)  =>  the gradient with respect to z sums to zero
    rng = np.random.default_rng(7)
    for _ in range(10):
        z = rng.normal(scale=2.0, size=16)
        p, _ = entmax(z, alpha)
        dz = entmax_vjp(p, rng.normal(size=16), alpha)
        assert abs(dz.sum()) < 1e-12
        assert np.all(dz[p == 0] == 0.0)


def test_sparsemax_jacobian_closed_form():
    # alpha = 2: J = diag(s) - s s^T / |S| with s the support indicator
    rng = np.random.default_rng(3)
    for _ in range(10):
        z = rng.normal(scale=1.5, size=12)
        g = rng.normal(size=12)
        p, _ = entmax(z, 2.0)
        s = (p > 0).astype(np.float64)
        J = np.diag(s) - np.outer(s, s) / s.sum()
        np.testing.assert_allclose(entmax_vjp(p, g, 2.0), J @ g, atol=1e-14)


def _tiny(seed, S=40, H=2, Hkv=1, d=8, qs=2.0, ks=3.0):
    rng = np.random.default_rng(seed)
    q = rng.normal(scale=qs, size=(S, H, d))
    k = rng.normal(scale=ks, size=(S, Hkv, d))
    v = rng.normal(size=(S, Hkv, d))
    w_s = np.eye(d) + 0.3 * rng.normal(size=(d, d))
    dout = rng.normal(size=(S, H, d))
    return q, k, v, w_s, dout


@pytest.mark.parametrize("causal,alpha,sigma", [(True, 1.5, 0.7), (False, 1.5, 1.0), (True, 2.0, 1.0),
                                                (True, 1.25, 1.3)])
def test_backward_matches_finite_differences(causal, alpha, sigma):
    block = 8
    q, k, v, w_s, dout = _tiny(11)
    fw = forward(q, k, v, w_s, alpha, block, causal)
    sizes = [len(r["idx"]) for r in fw["routes"].values() if len(r["cand"]) > 1]
    assert any(1 < n for n in sizes) and any(n < len(r["cand"]) for n, r in
                                             zip(sizes, [r for r in fw["routes"].values() if len(r["cand"]) > 1]))
    grads = backward(q, k, v, w_s, dout, alpha, block, causal, sigma)
    rng = np.random.default_rng(5)
    eps = 1e-6
    for name, arr in (("q", q), ("k", k), ("v", v), ("w_s", w_s)):
        an = grads["d" + name]
        flat = rng.choice(arr.size, size=min(24, arr.size), replace=False)
        for f in flat:
            ix = np.unravel_index(f, arr.shape)
            args = {"q": q, "k": k, "v": v, "w_s": w_s}
            plus = {n: a.copy() for n, a in args.items()}
            minus = {n: a.copy() for n, a in args.items()}
            plus[name][ix] += eps
            minus[name][ix] -= eps
            fd = (loss(**plus, dout=dout, alpha=alpha, block=block, causal=causal, sigma=sigma)
                  - loss(**minus, dout=dout, alpha=alpha, block=block, causal=causal, sigma=sigma)) / (2 * eps)
            assert abs(fd - an[ix]) <= 1e-6 + 1e-6 * abs(fd), (name, ix, fd, an[ix])


def test_backward_ws_zero_is_causal_sdpa_gradient():
    # W_s = 0: every candidate gets p_bar = 1/N and the diagonal bias is
    # log(1/N), so the forward is causal attention; its input gradients are
    # those of torch's scaled_dot_product_attention (GQA by repeating K/V).
    S, H, Hkv, d, block = 48, 4, 2, 8, 8
    q, k, v, _, dout = _tiny(2, S=S, H=H, Hkv=Hkv, d=d)
    g = backward(q, k, v, np.zeros((d, d)), dout, 1.5, block, True)
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    rep = H // Hkv
    out = F.scaled_dot_product_attention(tq.transpose(0, 1), tk.repeat_interleave(rep, 1).transpose(0, 1),
                                         tv.repeat_interleave(rep, 1).transpose(0, 1), is_causal=True)
    out.transpose(0, 1).backward(torch.tensor(dout))
    np.testing.assert_allclose(g["dq"], tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(g["dk"], tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(g["dv"], tv.grad.numpy(), atol=1e-11)
    # the router still sees a gradient through W_s
    assert np.abs(g["dw_s"]).max() > 1e-3


def test_backward_sigma_zero_routes_no_gradient():
    # sigma = 0 removes the prior from the logits: the loss no longer depends
    # on the routing probabilities, so W_s gets exactly zero
    q, k, v, w_s, dout = _tiny(4)
    g = backward(q, k, v, w_s, dout, 1.5, 8, True, sigma=0.0)
    assert np.all(g["dw_s"] == 0.0)
    g1 = backward(q, k, v, w_s, dout, 1.5, 8, True, sigma=1.0)
    assert np.abs(g1["dw_s"]).max() > 1e-3


def test_backward_single_block_is_local_attention():
    # S <= block: one block, no candidates, plain causal attention in it
    q, k, v, w_s, dout = _tiny(9, S=8)
    g = backward(q, k, v, w_s, dout, 1.5, 8, True)
    assert np.all(g["dw_s"] == 0.0)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    out = F.scaled_dot_product_attention(tq.transpose(0, 1), tk.repeat_interleave(2, 1).transpose(0, 1),
                                         tv.repeat_interleave(2, 1).transpose(0, 1), is_causal=True)
    out.transpose(0, 1).backward(torch.tensor(dout))
    np.testing.assert_allclose(g["dq"], tq.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(g["dk"], tk.grad.numpy(), atol=1e-12)


@pytest.mark.parametrize("causal", [True, False])
def test_backward_shift_and_normalisation_identities(causal):
    # shifting every key of a KV head by one vector moves each row's logits
    # and each row's block scores by a constant, which neither softmax nor
    # entmax sees: sum_j dk_j = 0.  Each softmax row sums to one:
    # sum_j dv_j = sum over the rows and the group's heads of dout.
    S, H, Hkv, d = 40, 4, 2, 8
    q, k, v, w_s, dout = _tiny(21, S=S, H=H, Hkv=Hkv, d=d)
    g = backward(q, k, v, w_s, dout, 1.5, 8, causal, sigma=0.8)
    G = H // Hkv
    for kv in range(Hkv):
        np.testing.assert_allclose(g["dk"][:, kv].sum(axis=0), 0.0, atol=1e-11)
        np.testing.assert_allclose(g["dv"][:, kv].sum(axis=0), dout[:, kv * G:(kv + 1) * G].sum(axis=(0, 1)),
                                   atol=1e-11)


def test_backward_magnitudes_bound_the_gradients():
    # the magnitude sums returned for error bounds dominate the gradients
    # element by element (triangle inequality), and are zero only where the
    # gradient has no terms
    q, k, v, w_s, dout = _tiny(13, S=40, H=4, Hkv=2, d=8)
    g = backward(q, k, v, w_s, dout, 1.5, 8, True, sigma=0.9)
    for name in ("dq", "dk", "dv"):
        assert np.all(g[name + "_abs"] >= np.abs(g[name]) - 1e-12), name
        assert g[name + "_abs"].min() >= 0.0


def test_backward_given_exact_output_is_unchanged():
    # D = dout . out with the exact forward output is the softmax-gradient
    # identity sum_j P_j dP_j, so passing that output changes nothing; the
    # root sums of squares are below the absolute sums of the rounded terms
    q, k, v, w_s, dout = _tiny(17, S=40, H=4, Hkv=2, d=8)
    out = forward(q, k, v, w_s, 1.5, 8, True)["out"]
    g0 = backward(q, k, v, w_s, dout, 1.5, 8, True)
    g1 = backward(q, k, v, w_s, dout, 1.5, 8, True, out=out)
    for name in ("dq", "dk", "dv", "dw_s"):
        np.testing.assert_allclose(g1[name], g0[name], atol=1e-12)
    for name in ("dq", "dv"):
        assert np.all(g0[name + "_rss"] <= g0[name + "_abs"] + 1e-15)


def test_rounding_error_model_behind_the_gpu_tolerance():
    # The GPU backward rounds P (for dv) and dS (for dq, dk) to bf16 as
    # tensor-core operands.  Rounding those operands here, in the oracle's
    # own stage-2 sums, must stay inside the bound the GPU parity test uses:
    # 3.5 u times the root sum of squares of the rounded terms (u = 2^-8),
    # i.e. about six standard deviations of independent round-to-nearest errors.
    from oracle.backward import _attended
    from oracle.dash_oracle import block_summaries, forward_row

    def bf16(x):
        return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).double().numpy()

    rng = np.random.default_rng(8)
    S, H, Hkv, d, block = 96, 4, 2, 32, 16
    q = bf16(rng.normal(scale=0.5, size=(S, H, d)))
    k = bf16(rng.normal(scale=0.5, size=(S, Hkv, d)))
    v = bf16(rng.normal(size=(S, Hkv, d)))
    dout = bf16(rng.normal(size=(S, H, d)))
    w_s = np.eye(d) + 0.1 * rng.normal(size=(d, d))
    G, scale, u = H // Hkv, 1.0 / math.sqrt(d), 2.0 ** -8
    out = bf16(forward(q, k, v, w_s, 1.5, block, True)["out"])
    ref = backward(q, k, v, w_s, dout, 1.5, block, True, out=out)
    rounded = {n: np.zeros_like(a) for n, a in (("dq", q), ("dk", k), ("dv", v))}
    exact = {n: np.zeros_like(a) for n, a in (("dq", q), ("dk", k), ("dv", v))}
    for g in range(Hkv):
        summ = block_summaries(k[:, g], w_s, block, S)
        for pos in range(S):
            r = forward_row(q[pos, g * G:(g + 1) * G], k[:, g], v[:, g], summ, pos, S, block, 1.5, True)
            tok, bias, _ = _attended(r, pos, S, block, True, 1.0)
            for h in range(g * G, (g + 1) * G):
                lg = k[tok, g] @ q[pos, h] * scale + bias
                P = np.exp(lg - lg.max())
                P /= P.sum()
                dS = P * (v[tok, g] @ dout[pos, h] - dout[pos, h] @ out[pos, h])
                for acc, Pm, dSm in ((rounded, bf16(P), bf16(dS)), (exact, P, dS)):
                    acc["dq"][pos, h] += scale * dSm @ k[tok, g]
                    acc["dk"][tok, g] += scale * np.outer(dSm, q[pos, h])
                    acc["dv"][tok, g] += np.outer(Pm, dout[pos, h])
    for name in ("dq", "dk", "dv"):
        err = np.abs(rounded[name] - exact[name])
        assert err.max() > 0.0
        assert np.all(err <= 3.5 * u * ref[name + "_rss"] + 1e-12), name


@pytest.mark.parametrize("causal", [True, False])
def test_key_block_backward_is_the_whole_backward_restricted(causal):
    # the per-block form sums the same row contributions as backward(); rows
    # that do not reach a block add exactly nothing, so the two agree on the
    # block's tokens (dk with its stage-0 term, dv, and the term sizes)
    from oracle.backward import key_block_backward

    S, H, Hkv, d, block = 75, 4, 2, 8, 8  # ragged tail: 75 = 9 * 8 + 3
    q, k, v, w_s, dout = _tiny(31, S=S, H=H, Hkv=Hkv, d=d)
    full = backward(q, k, v, w_s, dout, 1.5, block, causal, sigma=1.2)
    G = H // Hkv
    for g in range(Hkv):
        hs = slice(g * G, (g + 1) * G)
        blocks = [0, 4, 9]
        kb = key_block_backward(q[:, hs], k[:, g], v[:, g], w_s, dout[:, hs], None, blocks, block, 1.5, causal,
                                sigma=1.2)
        for c in blocks:
            lo, hi = c * block, min(S, (c + 1) * block)
            for name in ("dk", "dv", "dk_abs", "dv_abs"):
                np.testing.assert_allclose(kb[c][name], full[name][lo:hi, g], atol=1e-12, err_msg=f"{name} c={c}")
            for name in ("dk", "dv"):
                np.testing.assert_allclose(np.sqrt(kb[c][name + "_ss"]), full[name + "_rss"][lo:hi, g], atol=1e-12)
        assert kb["rows"][0] >= block  # block 0 is reached by its own rows at least
        # disjoint row sets add up to the whole
        parts = [key_block_backward(q[:, hs], k[:, g], v[:, g], w_s, dout[:, hs], None, blocks, block, 1.5, causal,
                                    sigma=1.2, rows=range(r0, S, 3)) for r0 in range(3)]
        for c in blocks:
            for name in ("dk", "dv", "dk_ss", "dv_abs"):
                np.testing.assert_allclose(sum(p[c][name] for p in parts), kb[c][name], atol=1e-12)
