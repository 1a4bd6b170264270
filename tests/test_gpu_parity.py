"""GPU parity: every stage of the CUDA path against the fp64 oracle on the
same seeded inputs, at sizes the oracle finishes in seconds that still span
several tiles and a ragged tail, plus the edge cases (no candidates, a
single partial block, non-causal, every group size, both head dims, the
three alphas).  All calls go through the C ABI via the Python binding.
"""

import math

import numpy as np
import pytest
import torch

from gen import Config, full_inputs, get_config, kv_values, make_plan
from oracle.dash_oracle import block_summaries, block_summaries_sdpa, lists_to_mask
from tests._oracle_pool import oracle_heads_pooled
from tests._parity import (
    OUT_TOL,
    check_p_dense,
    check_route_row,
    max_abs,
    oracle_decode_pair,
    oracle_head,
    to_np,
)

pytestmark = pytest.mark.gpu

_BASE = get_config("prefill")
SMALL = {
    "pr1": get_config("pr1"),
    "prefill_small": _BASE.with_(name="prefill_small", seq=2000),
    "long_small": get_config("long_prefill").with_(name="long_small", seq=128 * 22 + 50),
    "g8_small": _BASE.with_(name="g8_small", heads=16, kv_heads=2, seq=1100),
    "g2_d64": _BASE.with_(name="g2_d64", heads=8, kv_heads=4, head_dim=64, seq=900, dtype="f16"),
    "g1_b128": _BASE.with_(name="g1_b128", heads=4, kv_heads=4, block=128, seq=1300, alpha=2.0),
    "noncausal": _BASE.with_(name="noncausal", seq=1000, causal=False),
    "tiny": _BASE.with_(name="tiny", seq=40),
    "f32_d128": _BASE.with_(name="f32_d128", heads=4, kv_heads=2, dtype="f32", seq=700, scaled=False,
                            query_strength=11.3, key_strength=3.0),
}
for a in (1.25, 1.5, 2.0):
    for s in (0.0, 4.0):
        n = f"sweep_a{a}_s{s:g}"
        SMALL[n] = get_config("sweep").with_(name=n, batch=2, seq=1500, alpha=a, key_strength=s)


def _kv_subset(cfg):
    return list(range(cfg.kv_heads))  # every KV group


@pytest.fixture(scope="module")
def dash(cuda_lib):
    return cuda_lib


def _run_all(dash, cfg):
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w = inp["q"], inp["k"], inp["v"], inp["w_s"]
    ws = torch.empty(dash.fwd_workspace_size(q, k, cfg.block), dtype=torch.uint8, device="cuda")
    out = dash.fwd(q, k, v, w, cfg.alpha, cfg.block, cfg.causal, workspace=ws)
    fl = dash.fwd_lists(ws, q, k, cfg.block)  # the lists the forward itself routed with
    summ = dash.summarize(k, w, cfg.block)
    rt = dash.route(q, summ, cfg.alpha, cfg.block, cfg.causal, want_tau=True, want_p=True)
    torch.cuda.synchronize()
    return inp, out, summ, rt, fl


def test_generator_identical_on_gpu(dash):
    for cfg in (SMALL["prefill_small"], SMALL["pr1"], SMALL["sweep_a1.5_s4"]):
        gpu = full_inputs(cfg, device="cuda")
        cpu = full_inputs(cfg, device="cpu")
        for key in ("q", "k", "v", "w_s"):
            assert torch.equal(gpu[key].cpu(), cpu[key]), (cfg.name, key)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_forward_parity_small(dash, name):
    cfg = SMALL[name]
    inp, out, summ, rt, fl = _run_all(dash, cfg)
    plan = inp["plan"]
    G = cfg.group
    tol = OUT_TOL[cfg.dtype]
    out_np = to_np(out)
    summ_np = summ.cpu().numpy()
    idx, logp, cnt = rt["idx"].cpu().numpy(), rt["logp"].cpu().numpy(), rt["cnt"].cpu().numpy()
    f_idx, f_logp, f_cnt = fl["idx"].cpu().numpy(), fl["logp"].cpu().numpy(), fl["cnt"].cpu().numpy()
    p_dense, tau = rt["p"].cpu().numpy(), rt["tau"].cpu().numpy()
    rows = list(range(cfg.seq))
    worst_out = worst_p = 0.0
    ref = oracle_heads_pooled(cfg, plan, [(b, g) for b in range(cfg.batch) for g in _kv_subset(cfg)], rows)
    for b in range(cfg.batch):
        for g in _kv_subset(cfg):
            recs, summ_o = ref[(b, g)]
            # stage 0
            serr = np.abs(summ_np[b, g, : len(summ_o)] - summ_o).max()
            assert serr <= 2e-5 * max(1.0, np.abs(summ_o).max()), f"{name}: summary error {serr:.3g}"
            for pos, rec in zip(rows, recs):
                where = f"{name} b{b} g{g} pos{pos}"
                check_route_row(rec, idx[b, g, pos], logp[b, g, pos], cnt[b, g, pos], where)
                check_route_row(rec, f_idx[b, g, pos], f_logp[b, g, pos], f_cnt[b, g, pos], where + " (fwd)")
                e = check_p_dense(rec, p_dense[b, g * G:(g + 1) * G, pos], tau[b, g * G:(g + 1) * G, pos], where)
                worst_p = max(worst_p, e)
                err = max_abs(out_np[b, pos, g * G:(g + 1) * G], rec["out"])
                worst_out = max(worst_out, err)
                assert err <= tol, f"{where}: output error {err:.3g} > {tol}"
    print(f"{name}: max |out err| {worst_out:.3g}, max |p err| {worst_p:.3g}")


def test_all_selected_uniform_prior_is_full_attention(dash):
    """Stage 2 with every candidate selected at log(1/N) equals plain causal attention."""
    cfg = SMALL["prefill_small"].with_(heads=8, kv_heads=2, seq=777)
    inp = full_inputs(cfg, device="cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    B, S, H, d = q.shape
    Hkv, T = k.shape[2], -(-S // cfg.block)
    pos = torch.arange(S)
    n_cand = (pos // cfg.block).int()
    idx = torch.arange(T, dtype=torch.int32).expand(B, Hkv, S, T).contiguous()
    logp = torch.where(n_cand > 0, torch.log(1.0 / n_cand.clamp(min=1).double()), torch.zeros(S, dtype=torch.float64))
    logp = logp.float()[None, None, :, None].expand(B, Hkv, S, T).contiguous()
    cnt = n_cand[None, None].expand(B, Hkv, S).contiguous()
    out = dash.sparse(q, k, v, idx.cuda(), logp.cuda(), cnt.cuda(), cfg.block, True)
    qq = q.double().cpu().permute(0, 2, 1, 3)
    kk = k.double().cpu().repeat_interleave(H // Hkv, dim=2).permute(0, 2, 1, 3)
    vv = v.double().cpu().repeat_interleave(H // Hkv, dim=2).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True).permute(0, 2, 1, 3)
    assert max_abs(out.double().cpu(), ref) <= 2e-2


def test_summarize_incremental_and_seqlens(dash):
    cfg = SMALL["prefill_small"].with_(seq=1000)
    inp = full_inputs(cfg, device="cuda")
    k, w = inp["k"], inp["w_s"]
    full = dash.summarize(k, w, cfg.block)
    # recompute from block 7 on into a buffer holding garbage before it
    part = torch.full_like(full, 123.0)
    dash.summarize(k, w, cfg.block, summaries=part, first_block=7)
    assert torch.equal(part[:, :, 7:], full[:, :, 7:])
    assert torch.all(part[:, :, :7] == 123.0)
    # seqlens: a shorter context pools a partial last block over its valid tokens
    sl = torch.tensor([333], dtype=torch.int32, device="cuda")
    s2 = dash.summarize(k, w, cfg.block, seqlens=sl)
    kk = kv_values(cfg, inp["plan"], "k", 0, range(333), [3], as_float32=True)[:, 0].double().numpy()
    ref = block_summaries(kk, inp["plan"].w_s.double().numpy(), cfg.block, 333)
    got = s2[0, 3, : len(ref)].cpu().numpy()
    assert np.abs(got - ref).max() <= 2e-5 * max(1.0, np.abs(ref).max())


@pytest.mark.parametrize("name,scale", [("prefill_small", 0.0), ("prefill_small", 3.0), ("prefill_small", 30.0),
                                        ("g2_d64", 3.0), ("g1_b128", 10.0), ("f32_d128", 3.0)])
def test_summarize_sdpa(dash, name, scale):
    """Stage 0 with learned summary queries against the oracle; a trailing partial block and seqlens."""
    cfg = SMALL[name]
    inp = full_inputs(cfg, device="cuda")
    k, w, plan = inp["k"], inp["w_s"], inp["plan"]
    d, Hkv = cfg.head_dim, cfg.kv_heads
    qbar = torch.from_numpy(np.random.default_rng(11).normal(size=(Hkv, d)) * scale).float()
    sl = torch.tensor([cfg.seq - 37] * cfg.batch, dtype=torch.int32, device="cuda")
    got = dash.summarize(k, w, cfg.block, qbar=qbar.cuda())
    got_sl = dash.summarize(k, w, cfg.block, seqlens=sl, qbar=qbar.cuda())
    torch.cuda.synchronize()
    if scale == 0.0:
        mean = dash.summarize(k, w, cfg.block)
        assert torch.allclose(got, mean, rtol=1e-6, atol=1e-6)
    for b in range(cfg.batch):
        for g in _kv_subset(cfg):
            kk = kv_values(cfg, plan, "k", b, range(cfg.seq), [g], as_float32=True)[:, 0].double().numpy()
            for n_tok, out in ((cfg.seq, got), (cfg.seq - 37, got_sl)):
                ref = block_summaries_sdpa(kk, plan.w_s.double().numpy(), qbar[g].double().numpy(), cfg.block, n_tok)
                err = np.abs(out[b, g, : len(ref)].cpu().numpy() - ref).max()
                assert err <= 2e-5 * max(1.0, np.abs(ref).max()), f"{name} scale {scale} b{b} g{g}: {err:.3g}"


@pytest.mark.parametrize("name,sigma,qscale", [("prefill_small", 0.0, None), ("prefill_small", 0.5, None),
                                               ("prefill_small", 2.0, 3.0), ("g1_b128", 0.5, 10.0),
                                               ("f32_d128", 0.5, 3.0)])
def test_forward_options(dash, name, sigma, qscale):
    """dash_attn_fwd_ex: prior strength sigma and learned summary queries, against the oracle."""
    cfg = SMALL[name]
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w, plan = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["plan"]
    qbar = None
    if qscale is not None:
        qbar = torch.from_numpy(np.random.default_rng(12).normal(size=(cfg.kv_heads, cfg.head_dim)) * qscale).float()
    out = dash.fwd(q, k, v, w, cfg.alpha, cfg.block, cfg.causal, sigma=sigma,
                   qbar=None if qbar is None else qbar.cuda())
    torch.cuda.synchronize()
    G, tol = cfg.group, OUT_TOL[cfg.dtype]
    out_np = to_np(out)
    rows = list(range(cfg.seq))
    ref = oracle_heads_pooled(cfg, plan, [(0, g) for g in _kv_subset(cfg)], rows, sigma=sigma,
                              qbar_of=None if qbar is None else {g: qbar[g].double().numpy()
                                                                 for g in _kv_subset(cfg)})
    for g in _kv_subset(cfg):
        recs, _ = ref[(0, g)]
        for pos, rec in zip(rows, recs):
            err = max_abs(out_np[0, pos, g * G:(g + 1) * G], rec["out"])
            assert err <= tol, f"{name} sigma {sigma} g{g} pos{pos}: output error {err:.3g}"


def test_decode_sigma(dash):
    cfg = get_config("decode").with_(name="decode_sigma", batch=3, seq=3000, seqlen_lo=200, seqlen_hi=3000)
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w, sl = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["seqlens"]
    summ = dash.summarize(k, w, cfg.block, seqlens=sl)
    out = dash.decode(q, k, v, sl, summ, cfg.alpha, cfg.block, sigma=0.5)
    torch.cuda.synchronize()
    G, out_np = cfg.group, to_np(out)
    for b in range(cfg.batch):
        for g in range(cfg.kv_heads):
            rec, _ = oracle_decode_pair(cfg, inp["plan"], b, g, sigma=0.5)
            err = max_abs(out_np[b, 0, g * G:(g + 1) * G], rec["out"])
            assert err <= OUT_TOL[cfg.dtype], f"b{b} g{g}: {err:.3g}"


def test_lists_to_mask_bit_exact(dash):
    cfg = SMALL["prefill_small"]
    inp = full_inputs(cfg, device="cuda")
    summ = dash.summarize(inp["k"], inp["w_s"], cfg.block)
    rt = dash.route(inp["q"], summ, cfg.alpha, cfg.block, True)
    for n_words in (None, 5):
        m = dash.lists_to_mask(rt["idx"], rt["cnt"], n_words)
        torch.cuda.synchronize()
        nw = m.shape[-1]
        ref = lists_to_mask(rt["idx"].cpu().numpy(), rt["cnt"].cpu().numpy(), nw)
        assert np.array_equal(m.cpu().numpy().view(np.uint32), ref)


DECODE_SMALL = {
    "decode_small": get_config("decode").with_(name="decode_small", batch=5, seq=4096, seqlen_lo=1, seqlen_hi=4096),
    "decode_g8_d64": get_config("decode").with_(name="decode_g8_d64", batch=3, heads=16, kv_heads=2, head_dim=64,
                                                 seq=3000, seqlen_lo=900, seqlen_hi=3000, dtype="f16", alpha=2.0),
    "decode_b128": get_config("decode").with_(name="decode_b128", batch=3, block=128, seq=5000, seqlen_lo=100,
                                              seqlen_hi=5000, alpha=1.25),
}


@pytest.mark.parametrize("name", sorted(DECODE_SMALL))
def test_decode_parity_small(dash, name):
    cfg = DECODE_SMALL[name]
    plan = make_plan(cfg)
    if name == "decode_small":  # cover a 1-token context and an exact block boundary
        plan.seqlens[0] = 1
        plan.seqlens[1] = 2 * cfg.block
        plan.seqlens[2] = 2 * cfg.block + 1
    inp = full_inputs(cfg, device="cuda", plan=plan)
    q, k, v, w, sl = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["seqlens"]
    summ = dash.summarize(k, w, cfg.block, seqlens=sl)
    out = dash.decode(q, k, v, sl, summ, cfg.alpha, cfg.block)
    rt = dash.route(q, summ, cfg.alpha, cfg.block, True, seqlens=sl, want_tau=True, want_p=True)
    torch.cuda.synchronize()
    G = cfg.group
    tol = OUT_TOL[cfg.dtype]
    out_np = to_np(out)
    idx, logp, cnt = rt["idx"].cpu().numpy(), rt["logp"].cpu().numpy(), rt["cnt"].cpu().numpy()
    for b in range(cfg.batch):
        for g in range(cfg.kv_heads):
            rec, _ = oracle_decode_pair(cfg, plan, b, g)
            where = f"{name} b{b} g{g} L{int(plan.seqlens[b])}"
            check_route_row(rec, idx[b, g, 0], logp[b, g, 0], cnt[b, g, 0], where)
            check_p_dense(rec, rt["p"][b, g * G:(g + 1) * G, 0].cpu().numpy(),
                          rt["tau"][b, g * G:(g + 1) * G, 0].cpu().numpy(), where)
            err = max_abs(out_np[b, 0, g * G:(g + 1) * G], rec["out"])
            assert err <= tol, f"{where}: output error {err:.3g}"


def test_forward_is_deterministic(dash):
    cfg = SMALL["prefill_small"]
    inp = full_inputs(cfg, device="cuda")
    a = dash.fwd(inp["q"], inp["k"], inp["v"], inp["w_s"], cfg.alpha, cfg.block)
    b = dash.fwd(inp["q"], inp["k"], inp["v"], inp["w_s"], cfg.alpha, cfg.block)
    assert torch.equal(a, b)


def test_device_status_and_bad_seqlens(dash):
    cfg = DECODE_SMALL["decode_small"]
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w, sl = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["seqlens"]
    summ = dash.summarize(k, w, cfg.block, seqlens=sl)
    ws = torch.empty(dash.decode_workspace_size(q, k, cfg.block, summ.shape[2]), dtype=torch.uint8, device="cuda")
    dash.decode(q, k, v, sl, summ, cfg.alpha, cfg.block, workspace=ws)
    assert dash.device_status(ws) == 0
    bad = sl.clone()
    bad[1] = cfg.seq + 5  # beyond the cache: clamped on the device and reported
    dash.decode(q, k, v, bad, summ, cfg.alpha, cfg.block, workspace=ws)
    assert dash.device_status(ws) == 1
    dash.decode(q, k, v, sl, summ, cfg.alpha, cfg.block, workspace=ws)
    assert dash.device_status(ws) == 0


# Tiles with more candidate blocks than TMEM holds logit columns (512) run the
# segmented routing kernel (logits through a scratch slot in global memory).
# Rows are sampled across the sequence, densely around the first such tile,
# and at the end.
WIDE = {
    "wide_g4": _BASE.with_(name="wide_g4", heads=8, kv_heads=2, seq=36000),
    "wide_g8_d64_f16": _BASE.with_(name="wide_g8_d64_f16", heads=16, kv_heads=2, head_dim=64, dtype="f16",
                                   seq=34000),
    "wide_g1_alpha2": _BASE.with_(name="wide_g1_alpha2", heads=2, kv_heads=2, seq=33500, alpha=2.0),
    "wide_noncausal": _BASE.with_(name="wide_noncausal", heads=8, kv_heads=2, seq=33000, causal=False),
    "wide_b128_g2_alpha125": _BASE.with_(name="wide_b128_g2_alpha125", heads=4, kv_heads=2, block=128, seq=70000,
                                         alpha=1.25),
}


def _wide_rows(cfg):
    P = 128 // cfg.group
    first_wide = ((512 + 1) * cfg.block) // P * P if cfg.causal else 0
    rows = set(range(0, cfg.seq, 211))
    rows.update(range(max(0, first_wide - 48), min(cfg.seq, first_wide + 48), 3))
    rows.update(range(cfg.seq - 70, cfg.seq))
    return sorted(rows)


@pytest.mark.parametrize("name", sorted(WIDE))
def test_wide_tile_routing_parity(dash, name):
    cfg = WIDE[name]
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w = inp["q"], inp["k"], inp["v"], inp["w_s"]
    ws = torch.empty(dash.fwd_workspace_size(q, k, cfg.block), dtype=torch.uint8, device="cuda")
    out = dash.fwd(q, k, v, w, cfg.alpha, cfg.block, cfg.causal, workspace=ws)
    fl = dash.fwd_lists(ws, q, k, cfg.block)
    summ = dash.summarize(k, w, cfg.block)
    rt = dash.route(q, summ, cfg.alpha, cfg.block, cfg.causal, want_tau=True, want_p=True)
    torch.cuda.synchronize()
    assert dash.device_status(ws) == 0
    assert -(-cfg.seq // cfg.block) > 512  # some tiles exceed TMEM's 512 columns
    rows = _wide_rows(cfg)
    rsel = torch.tensor(rows, device="cuda")
    G, tol = cfg.group, OUT_TOL[cfg.dtype]
    ref = oracle_heads_pooled(cfg, inp["plan"], [(0, g) for g in range(cfg.kv_heads)], rows)
    worst = 0.0
    for g in range(cfg.kv_heads):
        recs, summ_o = ref[(0, g)]
        serr = np.abs(fl["summaries"][0, g, : len(summ_o)].cpu().numpy() - summ_o).max()
        assert serr <= 2e-5 * max(1.0, np.abs(summ_o).max()), f"{name}: summary error {serr:.3g}"
        sel = {n: [t[0, g].index_select(0, rsel).cpu().numpy() for t in (src["idx"], src["logp"], src["cnt"])]
               for n, src in (("fwd", fl), ("route", rt))}
        p_rows = rt["p"][0, g * G:(g + 1) * G].index_select(1, rsel).cpu().numpy()
        tau_rows = rt["tau"][0, g * G:(g + 1) * G].index_select(1, rsel).cpu().numpy()
        o = out[0, :, g * G:(g + 1) * G].index_select(0, rsel).double().cpu().numpy()
        for i, (pos, rec) in enumerate(zip(rows, recs)):
            where = f"{name} g{g} pos{pos}"
            for n, (idx, logp, cnt) in sel.items():
                check_route_row(rec, idx[i], logp[i], cnt[i], f"{where} ({n})")
            check_p_dense(rec, p_rows[:, i], tau_rows[:, i], where)
            err = max_abs(o[i], rec["out"])
            worst = max(worst, err)
            assert err <= tol, f"{where}: output error {err:.3g} > {tol}"
    print(f"{name}: max |out err| {worst:.3g}")


def _dense_prior(idx, logp, cnt, fill=float("nan")):
    """[..., t_cap] log p_bar at column c from ascending lists; `fill` elsewhere (never read)."""
    T = idx.shape[-1]
    dense = torch.full(idx.shape, fill, dtype=torch.float32, device=idx.device)
    valid = torch.arange(T, device=idx.device) < cnt[..., None]
    cols = torch.where(valid, idx.long(), torch.full_like(idx.long(), T))
    padded = torch.cat([dense, torch.zeros(dense.shape[:-1] + (1,), device=idx.device)], dim=-1)
    padded.scatter_(-1, cols, torch.where(valid, logp, torch.zeros_like(logp)))
    return padded[..., :T].contiguous()


@pytest.mark.parametrize("name,sigma", [("prefill_small", 1.0), ("g8_small", 1.0), ("g2_d64", 0.5),
                                        ("g1_b128", 2.0), ("noncausal", 1.0), ("long_small", 1.0)])
def test_sparse_on_bit_packed_mask(dash, name, sigma):
    """dash_attn_sparse_mask (the pages' mask form) equals the list form bit for bit on the same
    routing, and the oracle within the output tolerance; the dense prior is NaN wherever the
    mask has no bit, so a read outside the selection would show."""
    cfg = SMALL[name]
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w = inp["q"], inp["k"], inp["v"], inp["w_s"]
    summ = dash.summarize(k, w, cfg.block)
    rt = dash.route(q, summ, cfg.alpha, cfg.block, cfg.causal)
    mask = dash.lists_to_mask(rt["idx"], rt["cnt"])
    dense = _dense_prior(rt["idx"], rt["logp"], rt["cnt"])
    ref = dash.sparse(q, k, v, rt["idx"], rt["logp"], rt["cnt"], cfg.block, cfg.causal, sigma=sigma)
    ws = torch.empty(dash.sparse_workspace_size(q, k, cfg.block, summ.shape[2]), dtype=torch.uint8, device="cuda")
    got = dash.sparse_mask(q, k, v, mask, dense, cfg.block, cfg.causal, workspace=ws, sigma=sigma)
    torch.cuda.synchronize()
    assert dash.device_status(ws) == 0
    assert torch.equal(got, ref)
    # against the oracle on every KV group, a spread of rows
    rows = sorted(set(range(0, cfg.seq, 7)) | {cfg.seq - 1})
    oref = oracle_heads_pooled(cfg, inp["plan"], [(0, g) for g in range(cfg.kv_heads)], rows, sigma=sigma)
    G, tol = cfg.group, OUT_TOL[cfg.dtype]
    o = to_np(got)
    for g in range(cfg.kv_heads):
        for pos, rec in zip(rows, oref[(0, g)][0]):
            err = max_abs(o[0, pos, g * G:(g + 1) * G], rec["out"])
            assert err <= tol, f"{name} g{g} pos{pos}: output error {err:.3g}"


def test_sparse_mask_ignores_and_reports_non_candidate_bits(dash):
    cfg = SMALL["prefill_small"]
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w = inp["q"], inp["k"], inp["v"], inp["w_s"]
    summ = dash.summarize(k, w, cfg.block)
    rt = dash.route(q, summ, cfg.alpha, cfg.block, True)
    mask = dash.lists_to_mask(rt["idx"], rt["cnt"])
    dense = _dense_prior(rt["idx"], rt["logp"], rt["cnt"])
    ref = dash.sparse(q, k, v, rt["idx"], rt["logp"], rt["cnt"], cfg.block, True)
    bad = mask.clone()
    pos = 700  # block 10: set the bit of its own block, not a candidate
    t = pos // cfg.block
    bad[0, 1, pos, t // 32] |= (1 << (t % 32)) if t % 32 < 31 else -(1 << 31)
    ws = torch.empty(dash.sparse_workspace_size(q, k, cfg.block, summ.shape[2]), dtype=torch.uint8, device="cuda")
    got = dash.sparse_mask(q, k, v, bad, dense, cfg.block, True, workspace=ws)
    assert dash.device_status(ws) == 1
    assert torch.equal(got, ref)


def test_bounded_wait_gives_up_and_reports(dash):
    """A stage-2 launch whose copies never come: every bounded wait runs out after 2^20
    cycles, the status word reads DASH_ERR_DEVICE_TIMEOUT (5) and the context stays usable;
    the next call on the same workspace reports 0 and matches a call that never stalled."""
    cfg = SMALL["prefill_small"]
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w = inp["q"], inp["k"], inp["v"], inp["w_s"]
    summ = dash.summarize(k, w, cfg.block)
    rt = dash.route(q, summ, cfg.alpha, cfg.block, True)
    ref = dash.sparse(q, k, v, rt["idx"], rt["logp"], rt["cnt"], cfg.block, True)
    ws = torch.empty(dash.sparse_workspace_size(q, k, cfg.block, summ.shape[2]), dtype=torch.uint8, device="cuda")
    junk = torch.zeros_like(q)
    dash.debug_sparse_stalled(q, k, v, rt["idx"], rt["logp"], rt["cnt"], cfg.block, True, junk, ws, 1 << 20)
    assert dash.device_status(ws) == 5
    out = dash.sparse(q, k, v, rt["idx"], rt["logp"], rt["cnt"], cfg.block, True, workspace=ws)
    assert dash.device_status(ws) == 0
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
