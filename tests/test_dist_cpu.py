"""The multi-rank path of the benchmark on CPU: two gloo ranks run the same
setup, barrier and max-over-ranks timing as the NCCL ranks on GPUs, and each
rank draws its own independent sequence (weak scaling, no data-path
collective)."""

import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from gen import full_inputs, get_config

    w, r, _ = bench.dist_setup(world, backend="gloo")
    assert (w, r) == (world, rank)
    # the slowest rank sets the time
    t = bench.max_over_ranks(10.0 + rank, w)
    # independent inputs per rank: a small instance drawn with the rank's seed
    cfg = get_config("prefill").with_(seq=256, heads=4, kv_heads=1)
    q = full_inputs(cfg, device="cpu", seed=bench.rank_seed(cfg, r))["q"].float()
    sums = [torch.zeros(1, dtype=torch.float64) for _ in range(w)]
    dist.all_gather(sums, q.double().sum().reshape(1))
    bench.barrier(w)
    res = {"rank": r, "t": t, "sums": [float(x) for x in sums],
           "value": bench.job_throughput(cfg.seq, w, t)}
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump(res, f)
    bench.finish(w)


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["t"] == 10.0 + (world - 1)  # max over ranks, on every rank
        assert r["value"] == pytest.approx(256 * world / (r["t"] * 1e-3))
    # both ranks saw the same gathered checksums, and the ranks' inputs differ
    assert res[0]["sums"] == res[1]["sums"]
    assert res[0]["sums"][0] != res[0]["sums"][1]


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""


# --------------------------------------------------------------------------
# context-parallel decode: the orchestration (shard ranges, the score
# all-reduce, the partial all-gather, the merge) with fp64 compute steps
# built from the oracle, on two gloo ranks


class _OracleOps:
    """The four compute steps of a context-parallel decode step in fp64 (test only)."""

    @staticmethod
    def zeros(shape, like):
        return torch.zeros(shape, dtype=torch.float64)

    @staticmethod
    def scores(q, summ, block_lo, block_hi, seqlens, lmax, alpha, block, scores):
        B, _, H, d = q.shape
        Hkv, G = summ.shape[1], H // summ.shape[1]
        for b in range(B):
            N = (int(seqlens[b]) - 1) // block
            for c in range(block_lo, min(block_hi, N)):
                for g in range(Hkv):
                    for h in range(G):
                        z = float(q[b, 0, g * G + h].double() @ summ[b, g, c - block_lo].double())
                        scores[b, g, h, c] = (alpha - 1.0) * z / np.sqrt(d)
        return scores

    @staticmethod
    def lists(q, kv_heads, scores, seqlens, lmax, alpha, block):
        from oracle.dash_oracle import entmax_threshold

        B, Hkv, G, t_cap = scores.shape
        out = {"idx": [[None] * Hkv for _ in range(B)], "logp": [[None] * Hkv for _ in range(B)]}
        for b in range(B):
            N = (int(seqlens[b]) - 1) // block
            for g in range(Hkv):
                pb = np.zeros(N)
                for h in range(G):
                    x = scores[b, g, h, :N].numpy()
                    if N:
                        tau = entmax_threshold(x, alpha)
                        pb += np.maximum(x - tau, 0.0) ** (1.0 / (alpha - 1.0))
                pb /= G
                sel = np.nonzero(pb > 0)[0]
                out["idx"][b][g] = sel
                out["logp"][b][g] = np.log(pb[sel])
        return out

    @staticmethod
    def attend(q, kshard, vshard, tok_lo, seqlens, lmax, lists, block, sigma):
        B, _, H, d = q.shape
        n, Hkv = kshard.shape[1], kshard.shape[2]
        G = H // Hkv
        part = torch.zeros((B, H, d + 2), dtype=torch.float64)
        part[:, :, d] = -np.inf
        for b in range(B):
            pos = int(seqlens[b]) - 1
            t = pos // block
            beta = np.log(1.0 / t) if t > 0 else 0.0
            for g in range(Hkv):
                toks, bias = [], []
                for c, lp in zip(lists["idx"][b][g], lists["logp"][b][g]):
                    if tok_lo <= c * block < tok_lo + n:
                        toks += list(range(c * block, (c + 1) * block))
                        bias += [sigma * lp] * block
                if tok_lo <= t * block < tok_lo + n:
                    toks += list(range(t * block, pos + 1))
                    bias += [sigma * beta] * (pos + 1 - t * block)
                if not toks:
                    continue
                loc = np.array(toks) - tok_lo
                kk = kshard[b, loc, g].double().numpy()
                vv = vshard[b, loc, g].double().numpy()
                for h in range(G):
                    qq = q[b, 0, g * G + h].double().numpy()
                    l2 = (kk @ qq / np.sqrt(d) + np.array(bias)) / np.log(2.0)
                    m = l2.max()
                    w = np.exp2(l2 - m)
                    part[b, g * G + h, :d] = torch.from_numpy(w @ vv)
                    part[b, g * G + h, d] = m
                    part[b, g * G + h, d + 1] = w.sum()
        return part

    @staticmethod
    def merge(parts, q):
        d = parts.shape[-1] - 2
        M = parts[..., d].max(dim=0).values
        f = torch.exp2(parts[..., d] - M)
        o = (f[..., None] * parts[..., :d]).sum(0) / (f * parts[..., d + 1]).sum(0)[..., None]
        return o[:, None]


def _cp_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch.distributed as dist

    from gen import full_inputs, get_config
    from oracle.dash_oracle import block_summaries
    from sparse_hierarchical_attention_mean_b200.cp import decode_step

    dist.init_process_group("gloo")
    cfg = get_config("decode").with_(name="cp_cpu", batch=2, heads=4, kv_heads=2, head_dim=16, seq=512,
                                     seqlen_lo=100, seqlen_hi=512, block=64)
    inp = full_inputs(cfg, device="cpu")
    q, k, v, sl = inp["q"], inp["k"], inp["v"], inp["seqlens"]
    lmax, blk = cfg.seq, cfg.block
    lo, hi = rank * lmax // world, (rank + 1) * lmax // world
    ks, vs = k[:, lo:hi], v[:, lo:hi]
    # this rank's summaries (fp64 oracle pooling of its complete blocks)
    nb = (hi - lo) // blk
    summ = torch.zeros((cfg.batch, cfg.kv_heads, nb, cfg.head_dim), dtype=torch.float64)
    w = inp["w_s"].double().numpy()
    for b in range(cfg.batch):
        n_tok = max(0, min(int(sl[b]) - lo, hi - lo))
        for g in range(cfg.kv_heads):
            s = block_summaries(ks[b, :, g].double().numpy(), w, blk, n_tok)
            summ[b, g, : len(s)] = torch.from_numpy(s)
    out = decode_step(q, ks, vs, summ, lo, sl, lmax, lmax // blk, cfg.alpha, blk, sigma=0.7, ops=_OracleOps)
    torch.save(out, os.path.join(out_dir, f"cp{rank}.pt"))
    dist.destroy_process_group()


def test_context_parallel_decode_two_gloo_ranks(tmp_path):
    from gen import full_inputs, get_config
    from oracle.dash_oracle import block_summaries, forward_row

    world = 2
    mp.start_processes(_cp_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    outs = [torch.load(tmp_path / f"cp{r}.pt") for r in range(world)]
    assert torch.equal(outs[0], outs[1])
    cfg = get_config("decode").with_(name="cp_cpu", batch=2, heads=4, kv_heads=2, head_dim=16, seq=512,
                                     seqlen_lo=100, seqlen_hi=512, block=64)
    inp = full_inputs(cfg, device="cpu")
    q, k, v, sl = inp["q"], inp["k"], inp["v"], inp["seqlens"]
    G = cfg.group
    for b in range(cfg.batch):
        for g in range(cfg.kv_heads):
            L = int(sl[b])
            kk = k[b, :L, g].double().numpy()
            vv = v[b, :L, g].double().numpy()
            n_complete = (L - 1) // cfg.block
            summ = block_summaries(kk[: n_complete * cfg.block], inp["w_s"].double().numpy(), cfg.block,
                                   n_complete * cfg.block)
            rec = forward_row(q[b, 0, g * G:(g + 1) * G].double().numpy(), kk, vv, summ, L - 1, L, cfg.block,
                              cfg.alpha, True, sigma=0.7)
            np.testing.assert_allclose(outs[0][b, 0, g * G:(g + 1) * G].numpy(), rec["out"], atol=1e-10)
