"""GPU parity of the backward pass (dash_attn_bwd) against the fp64 oracle.

Small cases run the whole oracle backward and compare every gradient; they
span several query and key blocks with a ragged tail, every group size, both
head dims and block sizes, the three alphas, sigma != 1, non-causal routing,
a batch of two and a single partial block.  At the full prefill size the
query gradients of sampled rows are compared with the oracle row by row, dk
and dv of the first, a middle and the last key block of one KV head element
by element (the oracle sums every row that reaches those blocks), and dk / dv
of every head with two identities that hold at any size: the loss does not change
when every key of a KV head moves by one vector (softmax and entmax are
shift invariant), so sum_j dk_j = 0; each softmax row sums to one, so
sum_j dv_j = sum of dout over the rows and the group's heads.

Tolerance, derived from the arithmetic.  Both sides read the same inputs,
the forward output included: the backward API takes the forward output as an
input (it enters D = dout . out), and the oracle is given the same one.  One
test gives both sides the oracle's own forward output, rounded to the input
type, so that no value from the GPU enters the oracle; the others give both
the kernel's forward output, as a user of the API does.  What remains is the kernel
rounding P (for dv) and dS (for dq, dk) once each to the input type as
tensor-core operands (unit roundoff u = 2^-8 for bf16, 2^-11 for f16), with
fp32 accumulation.  Round-to-nearest errors of different terms are
independent and unbiased, so an element's error has a standard deviation of
at most u / sqrt(3) times the root sum of squares of its rounded terms,
which the oracle returns (dq_rss, dk_rss, dv_rss).  The bound is 3.5 u times
that (six standard deviations), plus 2^-16 times the sum of the terms'
absolute values for fp32 accumulation and the fp32 routing gradient.  An
emulation of those roundings on the b64_g4 case stays within 3.2 standard
deviations over 4e5 elements.  dW_s comes out of the fp32 routing gradient
and is held to 2e-2 normwise.
"""

import numpy as np
import pytest
import torch

from gen import full_inputs, get_config
from oracle.backward import _forward_sigma, backward, backward_row
from oracle.dash_oracle import block_summaries

from tests._oracle_pool import key_block_backward_pooled

pytestmark = pytest.mark.gpu

NORM_TOL = 2e-2
UNIT_ROUNDOFF = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}

_BASE = get_config("prefill")
CASES = {
    "b64_g4": (_BASE.with_(name="b64_g4", heads=8, kv_heads=2, seq=700), 1.0),
    "b128_g8_d64_f16_noncausal": (_BASE.with_(name="b128_g8", heads=8, kv_heads=1, head_dim=64, dtype="f16",
                                              block=128, seq=420, causal=False), 0.7),
    "g1_alpha2": (_BASE.with_(name="g1_a2", heads=2, kv_heads=2, seq=333, alpha=2.0), 1.0),
    "g2_alpha125_b128": (_BASE.with_(name="g2_a125", heads=4, kv_heads=2, block=128, seq=600, alpha=1.25), 1.3),
    "batch2_f16_d64": (get_config("sweep").with_(name="sweep_b2", batch=2, heads=4, kv_heads=4, seq=300), 1.0),
    "single_partial_block": (_BASE.with_(name="tiny", heads=4, kv_heads=1, seq=40), 1.0),
    "full_heads_1k": (_BASE.with_(name="full_heads_1k", seq=1024), 1.0),
}


def _dout(q, seed=1234):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(q.shape, generator=g, dtype=torch.float32).to(q.dtype).to(q.device)


def _np(t):
    return t.detach().double().cpu().numpy()


def _close(name, got, ref):
    err = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    assert err <= NORM_TOL, f"{name}: normwise {err:.3g}"


def _within(name, got, ref, rss, absum, u):
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    bound = 3.5 * u * rss + 2.0 ** -16 * absum + 1e-7 * absum.max()
    excess = np.abs(got - ref) / bound
    worst = np.unravel_index(np.argmax(excess), excess.shape)
    assert excess.max() <= 1.0, (f"{name}: error {abs(got - ref)[worst]:.3g} at {worst} above the bound "
                                 f"{bound[worst]:.3g} (gradient {ref[worst]:.3g})")


@pytest.mark.parametrize("case", list(CASES))
def test_backward_matches_oracle(cuda_lib, case):
    dash = cuda_lib
    cfg, sigma = CASES[case]
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w_s = inp["q"], inp["k"], inp["v"], inp["w_s"]
    out = dash.fwd(q, k, v, w_s, cfg.alpha, cfg.block, cfg.causal, sigma=sigma)
    dout = _dout(q)
    g = dash.bwd(q, k, v, w_s, out, dout, cfg.alpha, cfg.block, cfg.causal, sigma=sigma)
    torch.cuda.synchronize()
    dw_ref = np.zeros((cfg.head_dim, cfg.head_dim))
    for b in range(cfg.batch):
        ref = backward(_np(q[b]), _np(k[b]), _np(v[b]), _np(w_s), _np(dout[b]), cfg.alpha, cfg.block, cfg.causal,
                       sigma, out=_np(out[b]))
        for name in ("dq", "dk", "dv"):
            _within(f"{case} b{b} {name}", _np(g[name][b]), ref[name], ref[name + "_rss"], ref[name + "_abs"],
                    UNIT_ROUNDOFF[q.dtype])
        dw_ref += ref["dw_s"]
    if cfg.seq > cfg.block:
        _close(f"{case} dw_s", _np(g["dw_s"]), dw_ref)
    else:
        assert torch.all(g["dw_s"] == 0)


@pytest.mark.parametrize("case", ["b64_g4", "b128_g8_d64_f16_noncausal"])
def test_backward_on_oracle_forward_output(cuda_lib, case):
    # the forward output both sides consume is the oracle's (fp64, rounded to
    # the input type), so nothing computed on the GPU enters the oracle
    dash = cuda_lib
    cfg, sigma = CASES[case]
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w_s = inp["q"], inp["k"], inp["v"], inp["w_s"]
    dout = _dout(q)
    for b in range(cfg.batch):
        ref_out = _forward_sigma(_np(q[b]), _np(k[b]), _np(v[b]), _np(w_s), cfg.alpha, cfg.block, cfg.causal, sigma)
        out_b = torch.from_numpy(ref_out).to(q.dtype)
        out = torch.zeros_like(q)
        out[b] = out_b.to(q.device)
        g = dash.bwd(q, k, v, w_s, out, dout, cfg.alpha, cfg.block, cfg.causal, sigma=sigma)
        torch.cuda.synchronize()
        ref = backward(_np(q[b]), _np(k[b]), _np(v[b]), _np(w_s), _np(dout[b]), cfg.alpha, cfg.block, cfg.causal,
                       sigma, out=out_b.double().numpy())
        for name in ("dq", "dk", "dv"):
            _within(f"{case} b{b} {name}", _np(g[name][b]), ref[name], ref[name + "_rss"], ref[name + "_abs"],
                    UNIT_ROUNDOFF[q.dtype])
        if cfg.batch == 1 and cfg.seq > cfg.block:
            _close(f"{case} dw_s", _np(g["dw_s"]), ref["dw_s"])


def test_backward_autograd_wrapper(cuda_lib):
    # torch.autograd through the library: the wrapper returns the same gradients
    dash = cuda_lib
    cfg = _BASE.with_(name="ag", heads=4, kv_heads=2, seq=200)
    inp = full_inputs(cfg, device="cuda")
    q, k, v = (inp[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    w_s = inp["w_s"].clone().requires_grad_(True)
    out = dash.attention(q, k, v, w_s, cfg.alpha, cfg.block, True)
    dout = _dout(out)
    out.backward(dout)
    g = dash.bwd(inp["q"], inp["k"], inp["v"], inp["w_s"], out.detach(), dout, cfg.alpha, cfg.block, True)
    torch.cuda.synchronize()
    assert torch.equal(q.grad, g["dq"].to(q.dtype))
    assert torch.equal(k.grad, g["dk"].to(k.dtype))
    assert torch.equal(v.grad, g["dv"].to(v.dtype))
    assert torch.equal(w_s.grad, g["dw_s"])


def test_backward_full_prefill(cuda_lib, tmp_path):
    # the full prefill workload: sampled rows' dq against the oracle, dk / dv
    # of three key blocks of KV head 0 element by element, and the two
    # identities for dk and dv over every KV head
    dash = cuda_lib
    cfg = get_config("prefill")
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w_s = inp["q"], inp["k"], inp["v"], inp["w_s"]
    out = dash.fwd(q, k, v, w_s, cfg.alpha, cfg.block, True)
    dout = _dout(q, seed=99)
    g = dash.bwd(q, k, v, w_s, out, dout, cfg.alpha, cfg.block, True)
    torch.cuda.synchronize()
    for name in ("dq", "dk", "dv", "dw_s"):
        assert torch.isfinite(g[name]).all(), name
    G = cfg.group
    for kv in range(cfg.kv_heads):
        dk = g["dk"][0, :, kv].double()
        assert (dk.sum(0).abs() <= 1e-3 * dk.abs().sum(0) + 1e-6).all(), f"sum dk, KV head {kv}"
        dv_sum = g["dv"][0, :, kv].double().sum(0)
        do = dout[0, :, kv * G:(kv + 1) * G].double()
        assert ((dv_sum - do.sum((0, 1))).abs() <= 1e-3 * do.abs().sum((0, 1))).all(), f"sum dv, KV head {kv}"
    w = _np(w_s)
    for kv in (0, cfg.kv_heads - 1):
        kg, vg = _np(k[0, :, kv]), _np(v[0, :, kv])
        summ = block_summaries(kg, w, cfg.block, cfg.seq)
        for pos in (0, 63, 64, 1000, 16385, cfg.seq - 1):
            hs = slice(kv * G, (kv + 1) * G)
            rb = backward_row(_np(q[0, pos, hs]), kg, vg, summ, _np(dout[0, pos, hs]), pos, cfg.seq, cfg.block,
                              cfg.alpha, True, out_group=_np(out[0, pos, hs]))
            _within(f"dq row {pos} KV head {kv}", _np(g["dq"][0, pos, hs]), rb["dq"], np.sqrt(rb["dq_ss"]),
                    rb["dq_abs"], UNIT_ROUNDOFF[q.dtype])
    # dk / dv of the first, a middle and the last key block of KV head 0, from
    # every row that reaches them (the same forward output on both sides)
    kv, hs = 0, slice(0, G)
    blocks = [0, cfg.n_blocks // 2, cfg.n_blocks - 1]
    arrays = {"q": _np(q[0, :, hs]).astype(np.float32), "k": _np(k[0, :, kv]).astype(np.float32),
              "v": _np(v[0, :, kv]).astype(np.float32), "w_s": _np(w_s), "dout": _np(dout[0, :, hs]).astype(np.float32),
              "out": _np(out[0, :, hs]).astype(np.float32)}
    kb = key_block_backward_pooled(tmp_path, arrays, blocks, cfg.block, cfg.alpha, True)
    assert kb["rows"][blocks[-1]] == cfg.block and kb["rows"][0] > cfg.block
    for c in blocks:
        lo, hi = c * cfg.block, (c + 1) * cfg.block
        for name in ("dk", "dv"):
            _within(f"{name} key block {c} KV head {kv}", _np(g[name][0, lo:hi, kv]), kb[c][name],
                    np.sqrt(kb[c][name + "_ss"]), kb[c][name + "_abs"], UNIT_ROUNDOFF[q.dtype])
