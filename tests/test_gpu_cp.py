"""Context-parallel decode on one GPU: R ranks emulated one after the other
(the score all-reduce is a sum of the ranks' buffers, the all-gather a stack
of their partials).  Checked against the whole-cache decode (identical
lists; outputs within the decode tolerance of each other) and the oracle;
both shard-attention paths (CUDA cores, and the split-KV tensor-core path
with a workspace) give the same partials."""

import pytest
import torch

from gen import full_inputs, get_config
from tests._parity import OUT_TOL, max_abs, oracle_decode_pair, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dash(cuda_lib):
    return cuda_lib


CASES = {
    "bf16_g4_r2": (get_config("decode").with_(name="cp_a", batch=3, seq=4096, seqlen_lo=200, seqlen_hi=4096), 2, 1.0),
    "bf16_g4_r4_sigma": (get_config("decode").with_(name="cp_b", batch=3, seq=4096, seqlen_lo=1, seqlen_hi=4096), 4,
                         0.5),
    "f16_g8_d64_b128_r2": (get_config("decode").with_(name="cp_c", batch=2, heads=16, kv_heads=2, head_dim=64,
                                                      dtype="f16", block=128, seq=3072, seqlen_lo=500,
                                                      seqlen_hi=3072), 2, 1.0),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_context_parallel_decode(dash, name):
    cfg, R, sigma = CASES[name]
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w, sl = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["seqlens"]
    B, lmax, Hkv, d = k.shape
    H, G, blk = q.shape[2], cfg.group, cfg.block
    t_cap = -(-lmax // blk)
    # whole cache
    summ = dash.summarize(k, w, blk, seqlens=sl)
    ref = dash.decode(q, k, v, sl, summ, cfg.alpha, blk, sigma=sigma)
    rt = dash.route(q, summ, cfg.alpha, blk, True, seqlens=sl)
    # shards: block-aligned token ranges
    bounds = [((lmax // blk) * r // R) * blk for r in range(R)] + [lmax]
    scores = torch.zeros((B, Hkv, G, t_cap), dtype=torch.float32, device="cuda")
    shards = []
    for r in range(R):
        lo, hi = bounds[r], bounds[r + 1]
        ks, vs = k[:, lo:hi].contiguous(), v[:, lo:hi].contiguous()
        sl_r = (sl - lo).clamp(0, hi - lo).to(torch.int32)
        summ_r = dash.summarize(ks, w, blk, seqlens=sl_r)
        part_scores = torch.zeros_like(scores)
        dash.cp_scores(q, summ_r, lo // blk, hi // blk, sl, lmax, cfg.alpha, blk, part_scores)
        scores += part_scores
        shards.append((lo, ks, vs))
    lists = dash.cp_lists(q, Hkv, scores, sl, lmax, cfg.alpha, blk)
    parts = torch.stack([dash.cp_attend(q, ks, vs, lo, sl, lmax, lists, blk, sigma=sigma) for lo, ks, vs in shards])
    out = dash.cp_merge(parts.contiguous(), torch.empty_like(q))
    # the same shards on the split-KV tensor-core path, one workspace reused
    ws = torch.empty(dash.cp_attend_workspace_size(B, H, Hkv, d, blk, t_cap), dtype=torch.uint8, device="cuda")
    parts_x = torch.stack([dash.cp_attend_ex(q, ks, vs, lo, sl, lmax, lists, blk, sigma=sigma, workspace=ws)
                           for lo, ks, vs in shards])
    out_x = dash.cp_merge(parts_x.contiguous(), torch.empty_like(q))
    torch.cuda.synchronize()
    # the routing is the whole cache's, bit for bit
    assert torch.equal(lists["cnt"], rt["cnt"][:, :, 0])
    for b in range(B):
        for g in range(Hkv):
            n = int(lists["cnt"][b, g])
            assert torch.equal(lists["idx"][b, g, :n], rt["idx"][b, g, 0, :n])
            assert torch.equal(lists["logp"][b, g, :n], rt["logp"][b, g, 0, :n])
    tol = OUT_TOL[cfg.dtype]
    assert max_abs(to_np(out), to_np(ref)) <= tol
    assert max_abs(to_np(out_x), to_np(ref)) <= tol
    # per shard and head: the two paths find the same mass (l = 0 exactly
    # where the shard holds none of the head's blocks) and the same
    # normalised partial output
    l, lx = parts[..., d + 1], parts_x[..., d + 1]
    assert torch.equal(l == 0, lx == 0)
    held = l > 0
    o_n = parts[..., :d] / l.clamp_min(1e-30)[..., None]
    ox_n = parts_x[..., :d] / lx.clamp_min(1e-30)[..., None]
    assert (o_n - ox_n)[held].abs().max().item() <= tol
    # l relative to each path's own reference max m: l * 2^m agrees
    lm = torch.log2(l[held]) + parts[..., d][held]
    lmx = torch.log2(lx[held]) + parts_x[..., d][held]
    assert (lm - lmx).abs().max().item() <= 1e-2
    for b in range(B):
        for g in sorted({0, Hkv - 1}):
            rec, _ = oracle_decode_pair(cfg, inp["plan"], b, g, sigma=sigma)
            for o_, tag in ((out, "cuda cores"), (out_x, "split-KV")):
                err = max_abs(to_np(o_)[b, 0, g * G:(g + 1) * G], rec["out"])
                assert err <= tol, f"{name} {tag} b{b} g{g}: {err:.3g}"


@pytest.mark.parametrize("block,dtype,qscale", [(64, "bf16", None), (128, "f16", 3.0)])
def test_paged_cache_matches_dense(dash, block, dtype, qscale):
    """A paged cache (pages of one block, shuffled, through a block table) gives the
    dense cache's summaries and decode output bit for bit."""
    cfg = get_config("decode").with_(name="paged", batch=3, seq=4096, seqlen_lo=100, seqlen_hi=4096, block=block,
                                     dtype=dtype)
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w, sl = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["seqlens"]
    B, lmax, Hkv, d = k.shape
    nb = lmax // block
    qbar = None
    if qscale is not None:
        qbar = (torch.randn((Hkv, d), generator=torch.Generator().manual_seed(5)) * qscale).float().cuda()
    # pages: every (sequence, block) in a shuffled pool, plus unused pages
    perm = torch.randperm(B * nb + 7, generator=torch.Generator().manual_seed(3))
    table = perm[: B * nb].view(B, nb).to(torch.int32).cuda()
    kp = torch.zeros((B * nb + 7, block, Hkv, d), dtype=k.dtype, device="cuda")
    vp = torch.zeros_like(kp)
    kp[table.view(-1).long()] = k.view(B, nb, block, Hkv, d).reshape(B * nb, block, Hkv, d)
    vp[table.view(-1).long()] = v.view(B, nb, block, Hkv, d).reshape(B * nb, block, Hkv, d)
    summ = dash.summarize(k, w, block, seqlens=sl, qbar=qbar)
    summ_p = dash.summarize_paged(kp, table, sl, w, block, qbar=qbar)
    ref = dash.decode(q, k, v, sl, summ, cfg.alpha, block)
    out = dash.decode_paged(q, kp, vp, table, sl, summ_p, cfg.alpha, block)
    torch.cuda.synchronize()
    assert torch.equal(summ_p, summ)
    assert torch.equal(out, ref)
