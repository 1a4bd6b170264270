"""Runs oracle row sums in worker processes (spawned, so they never inherit a CUDA context).

Test infrastructure: the workers read the stored inputs from .npy files
(memory-mapped) and call the oracle on a subset of the query rows; the oracle
functions used here return sums over rows, which the caller adds up.
"""

from __future__ import annotations

import atexit
import multiprocessing as mp
import os

import numpy as np

_POOL = None
_LIMIT = None


def _pool_size(n_tasks: int = 1 << 30) -> int:
    return max(1, min(n_tasks, 24, (os.cpu_count() or 2) - 1))


def _one_thread():
    """Worker start-up: one BLAS / OpenMP thread per process (the pool supplies the parallelism).

    The limits are set before torch (whose CPU ops generate the inputs) starts its thread pool,
    and applied again to every numerical library loaded by then."""
    os.environ["OMP_NUM_THREADS"] = "1"
    os.environ["MKL_NUM_THREADS"] = "1"
    import torch

    torch.set_num_threads(1)
    torch.set_num_interop_threads(1)
    from threadpoolctl import threadpool_limits

    global _LIMIT
    _LIMIT = threadpool_limits(1)


def _spawn_pool(n: int):
    return mp.get_context("spawn").Pool(n, initializer=_one_thread)


def shared_pool():
    """One spawned worker pool for the whole test session (started on first use)."""
    global _POOL
    if _POOL is None:
        _POOL = _spawn_pool(_pool_size())
        atexit.register(_close_pool)
    return _POOL


def _close_pool():
    global _POOL
    if _POOL is not None:
        _POOL.terminate()
        _POOL = None


def _key_block_part(args):
    from oracle.backward import key_block_backward

    paths, blocks, block, alpha, causal, sigma, rows = args
    arr = {name: np.load(path, mmap_mode="r") for name, path in paths.items()}
    return key_block_backward(arr["q"], arr["k"], arr["v"], arr["w_s"], arr["dout"], arr.get("out"), blocks, block,
                              alpha, causal, sigma, rows=rows)


def key_block_backward_pooled(tmpdir, arrays: dict, blocks, block, alpha, causal=True, sigma=1.0, workers=None):
    """oracle.backward.key_block_backward over all rows, the rows split over spawned processes.

    arrays: q, k, v, w_s, dout and optionally out (numpy, one KV group, see the oracle).
    Returns the same dict as the oracle, summed over the workers' row sets.
    """
    paths = {}
    for name, a in arrays.items():
        paths[name] = os.path.join(str(tmpdir), f"{name}.npy")
        np.save(paths[name], np.ascontiguousarray(a))
    S = arrays["q"].shape[0]
    n = workers or _pool_size()
    n_chunks = 4 * n  # interleaved row sets, so late (long) rows spread evenly
    chunks = [range(r0, S, n_chunks) for r0 in range(n_chunks)]
    tasks = [(paths, list(blocks), block, alpha, causal, sigma, ch) for ch in chunks]
    if workers:
        with _spawn_pool(n) as pool:
            parts = pool.map(_key_block_part, tasks, chunksize=1)
    else:
        parts = shared_pool().map(_key_block_part, tasks, chunksize=1)
    total = parts[0]
    for p in parts[1:]:
        for c in blocks:
            for name, val in p[c].items():
                total[c][name] = total[c][name] + val
            total["rows"][c] += p["rows"][c]
    return total


def _oracle_head_part(args):
    from tests._parity import oracle_head

    cfg, plan, b, g, rows, kw = args
    return (b, g), oracle_head(cfg, plan, b, g, rows, **kw)


def _oracle_decode_part(args):
    from tests._parity import oracle_decode_pair

    cfg, plan, b, g, kw = args
    return (b, g), oracle_decode_pair(cfg, plan, b, g, **kw)


def oracle_heads_pooled(cfg, plan, pairs, rows, qbar_of=None, **kw) -> dict:
    """tests._parity.oracle_head for every (batch, KV group) in ``pairs``, the rows of each pair
    split into interleaved parts so that every worker is busy, in spawned processes.
    qbar_of: optional {g: learned summary query of KV head g}.
    Returns {(b, g): (records in the order of ``rows``, summaries)}."""
    rows = list(rows)
    n_parts = max(1, min(len(rows), -(-2 * _pool_size() // max(1, len(pairs)))))
    tasks = []
    for b, g in pairs:
        kwg = dict(kw, **({"qbar": qbar_of[g]} if qbar_of else {}))
        for r0 in range(n_parts):
            tasks.append((cfg, plan, b, g, rows[r0::n_parts], kwg))
    if len(tasks) == 1:
        parts = [_oracle_head_part(tasks[0])]
    else:
        parts = shared_pool().map(_oracle_head_part, tasks, chunksize=1)
    out = {}
    for (b, g) in pairs:
        recs = [None] * len(rows)
        summ = None
        for i, ((pb, pg), (r, sm)) in enumerate(parts):
            if (pb, pg) != (b, g):
                continue
            r0 = i % n_parts
            recs[r0::n_parts] = r
            summ = sm
        out[(b, g)] = (recs, summ)
    return out


def oracle_decode_pooled(cfg, plan, pairs, **kw) -> dict:
    """tests._parity.oracle_decode_pair for every (sequence, KV group) in ``pairs``, in spawned
    processes.  Returns {(b, g): (record, summaries)}."""
    tasks = [(cfg, plan, b, g, kw) for b, g in pairs]
    return dict(shared_pool().map(_oracle_decode_part, tasks, chunksize=1))
