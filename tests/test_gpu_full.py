"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (one ``fwd`` / ``decode`` call over the whole batch with a
caller-owned workspace), checked on sampled rows that the fp64 oracle
computes one by one.  The summaries and routing lists checked are the ones
the timed call itself produced and left in its workspace (read at the
offsets the library reports), not those of a separate routing call:

  * prefill 32K (B=1, 32/8 heads, d=128, bf16, block 64): every 97th row,
    the first and last two blocks whole, the first and last row of every
    block, for the first and last KV group;
  * long prefill 128K (block 128, diffuse and needle KV heads): a sparser
    sample, one diffuse and one needle group;
  * decode (64 sequences, 64K..128K context): 40 (sequence, KV head) pairs
    spread over the batch and every KV head;
  * the alpha x plant-strength sweep (B=4, 16/16 heads, d=64, f16).

Same rules as the small-size tests: identical selected sets outside the
1e-4 band around tau, p_bar within 1e-5, outputs within 2e-2 (bf16/f16).
"""

import numpy as np
import pytest
import torch

from gen import full_inputs, get_config, sample_rows, sweep_configs
from tests._oracle_pool import oracle_decode_pooled, oracle_heads_pooled
from tests._parity import OUT_TOL, check_route_row, max_abs

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def dash(cuda_lib):
    return cuda_lib


def _bench_fwd(dash, cfg, inp):
    """The benchmark's launch: fwd over the whole batch with a preallocated workspace."""
    q, k, v, w = inp["q"], inp["k"], inp["v"], inp["w_s"]
    out = torch.empty_like(q)
    ws = torch.empty(dash.fwd_workspace_size(q, k, cfg.block), dtype=torch.uint8, device="cuda")
    dash.fwd(q, k, v, w, cfg.alpha, cfg.block, cfg.causal, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert dash.device_status(ws) == 0
    return out, ws


def _check_prefill(dash, cfg, batches, groups, rows):
    inp = full_inputs(cfg, device="cuda")
    out, ws = _bench_fwd(dash, cfg, inp)
    lists = dash.fwd_lists(ws, inp["q"], inp["k"], cfg.block)  # what the timed call routed with
    summ, idx_all, logp_all, cnt_all = lists["summaries"], lists["idx"], lists["logp"], lists["cnt"]
    rsel = torch.tensor(rows, device="cuda")
    G = cfg.group
    tol = OUT_TOL[cfg.dtype]
    worst = 0.0
    ref = oracle_heads_pooled(cfg, inp["plan"], [(b, g) for b in batches for g in groups], rows)
    for b in batches:
        for g in groups:
            recs, summ_o = ref[(b, g)]
            serr = np.abs(summ[b, g, : len(summ_o)].cpu().numpy() - summ_o).max()
            assert serr <= 2e-5 * max(1.0, np.abs(summ_o).max()), f"{cfg.name}: summary error {serr:.3g}"
            idx = idx_all[b, g].index_select(0, rsel).cpu().numpy()
            logp = logp_all[b, g].index_select(0, rsel).cpu().numpy()
            cnt = cnt_all[b, g].index_select(0, rsel).cpu().numpy()
            o = out[b, :, g * G:(g + 1) * G].index_select(0, rsel).double().cpu().numpy()
            for i, (pos, rec) in enumerate(zip(rows, recs)):
                where = f"{cfg.name} b{b} g{g} pos{pos}"
                check_route_row(rec, idx[i], logp[i], cnt[i], where)
                err = max_abs(o[i], rec["out"])
                worst = max(worst, err)
                assert err <= tol, f"{where}: output error {err:.3g} > {tol}"
    del inp, out, ws, lists, summ, idx_all, logp_all, cnt_all
    torch.cuda.empty_cache()
    return worst


def test_prefill_32k_sampled(dash):
    cfg = get_config("prefill")
    worst = _check_prefill(dash, cfg, [0], [0, cfg.kv_heads - 1], sample_rows(cfg.seq, cfg.block))
    print(f"prefill 32K: max |out err| {worst:.3g}")


def test_long_prefill_128k_sampled(dash):
    cfg = get_config("long_prefill")
    S, blk = cfg.seq, cfg.block
    rows = set(range(0, S, 1021))
    for c in (0, 1, S // blk - 2, S // blk - 1):
        rows.update({c * blk, c * blk + 1, c * blk + blk // 2, c * blk + blk - 1})
    # KV head 0 is diffuse (no plant), the last one carries needles
    worst = _check_prefill(dash, cfg, [0], [0, cfg.kv_heads - 1], sorted(rows))
    print(f"long prefill 128K: max |out err| {worst:.3g}")


@pytest.mark.parametrize("cfg", sweep_configs(), ids=lambda c: c.name)
def test_sweep_full_sampled(dash, cfg):
    S, blk = cfg.seq, cfg.block
    rows = set(range(0, S, 389))
    for c in (0, 1, S // blk - 2, S // blk - 1):
        rows.update(range(c * blk, (c + 1) * blk, 7))
    worst = _check_prefill(dash, cfg, [0, cfg.batch - 1], [0, cfg.kv_heads - 1], sorted(rows))
    print(f"{cfg.name}: max |out err| {worst:.3g}")


def test_decode_full_sampled(dash):
    cfg = get_config("decode")
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w, sl = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["seqlens"]
    T = -(-cfg.seq // cfg.block)
    summ = torch.zeros((cfg.batch, cfg.kv_heads, T, cfg.head_dim), dtype=torch.float32, device="cuda")
    dash.summarize(k, w, cfg.block, seqlens=sl, summaries=summ)
    out = torch.empty_like(q)
    ws = torch.empty(dash.decode_workspace_size(q, k, cfg.block, T), dtype=torch.uint8, device="cuda")
    dash.decode(q, k, v, sl, summ, cfg.alpha, cfg.block, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert dash.device_status(ws) == 0
    lists = dash.decode_lists(ws, q, k, cfg.block, T)  # the routing the timed step used
    G = cfg.group
    tol = OUT_TOL[cfg.dtype]
    worst = 0.0
    # 40 pairs: every KV head five times, sequences spread over the batch
    pairs = [((7 * i + 3 * (i // cfg.kv_heads)) % cfg.batch, i % cfg.kv_heads) for i in range(40)]
    assert len(set(pairs)) == 40
    ref = oracle_decode_pooled(cfg, inp["plan"], pairs)
    for b, g in pairs:
        rec, summ_o = ref[(b, g)]
        serr = np.abs(summ[b, g, : len(summ_o)].cpu().numpy() - summ_o).max()
        assert serr <= 2e-5 * max(1.0, np.abs(summ_o).max())
        where = f"decode b{b} g{g} L{int(inp['plan'].seqlens[b])}"
        check_route_row(rec, lists["idx"][b, g].cpu().numpy(), lists["logp"][b, g].cpu().numpy(),
                        lists["cnt"][b, g].cpu().numpy(), where)
        err = max_abs(out[b, 0, g * G:(g + 1) * G].double().cpu().numpy(), rec["out"])
        worst = max(worst, err)
        assert err <= tol, f"{where}: output error {err:.3g}"
    print(f"decode full: max |out err| {worst:.3g}")
