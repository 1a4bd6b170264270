"""Counter-based seeded generator and topic planting.

Value generator
---------------
Every entry of q, k, v and W_s is a function of (tensor key, flat element
index) alone::

    h     = mix(mix(lo32(index) ^ key) ^ ((hi32(index) + key2) mod 2^32))
    value = NORMAL_TABLE[h >> 16]

``mix`` is the 32-bit "lowbias32" integer finaliser from Chris Wellons'
hash-prospector (xor-shift 16, multiply 0x7feb352d, xor-shift 15, multiply
0x846ca68b, xor-shift 16).  ``NORMAL_TABLE[i]`` is the standard normal
quantile at (i + 0.5) / 65536, rounded to fp32: a 65536-level
discretisation of N(0, 1) with support about +-4.32.

Everything is integer arithmetic, one table gather and single IEEE fp32
multiplies and adds, so the CPU and the CUDA builds of torch produce
bit-identical tensors, and any slice (one sequence, one KV head, a few query
rows) can be regenerated alone from its indices.  The oracle tests use that
to rebuild exactly the inputs that the GPU saw.

Planting
--------
Routing only becomes sparse when some key blocks are aligned with a query.
Per (batch, KV head) a small table of planted vectors is added to keys
(per key block) and to queries (per query block, all heads of the group);
see :func:`make_plan`.  The random choices (directions, topics, lengths) are
drawn on the CPU with numpy's PCG64 and are small.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from statistics import NormalDist

import numpy as np
import torch

from .configs import Config

_M32 = 0xFFFFFFFF
_TID = {"q": 1, "k": 2, "v": 3, "w_s": 4}
_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _DTYPES[name]


def _build_table() -> np.ndarray:
    nd = NormalDist()
    return np.array([nd.inv_cdf((i + 0.5) / 65536.0) for i in range(65536)], dtype=np.float32)


_TABLE_NP = _build_table()
_TABLES: dict[str, torch.Tensor] = {}


def _table(device) -> torch.Tensor:
    key = str(device)
    t = _TABLES.get(key)
    if t is None:
        t = torch.from_numpy(_TABLE_NP).to(device)
        _TABLES[key] = t
    return t


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for x < 2^32 held in int64, without int64 overflow."""
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & _M32


def _mix32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    return x ^ (x >> 16)


def _mix32_int(x: int) -> int:
    x &= _M32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & _M32
    x ^= x >> 15
    x = (x * 0x846CA68B) & _M32
    return x ^ (x >> 16)


def stream_key(seed: int, tensor: str) -> tuple[int, int]:
    k0 = _mix32_int(_mix32_int(seed * 0x9E3779B1 + 0x632BE5AB) ^ _TID[tensor])
    k1 = _mix32_int(k0 ^ 0x5BD1E995)
    return k0, k1


def draw(key: tuple[int, int], index: torch.Tensor) -> torch.Tensor:
    """fp32 N(0,1) quantile draws at the int64 flat indices ``index``."""
    k0, k1 = key
    h = _mix32((index & _M32) ^ k0)
    h = _mix32(h ^ (((index >> 32) + k1) & _M32))
    return _table(index.device)[h >> 16]


# --------------------------------------------------------------------------
# Planting plan


@dataclass
class Plan:
    """Small CPU-side description of one seeded instance of a config.

    k_tab[b, g, m]  fp32 vector added to every key of a block whose
                    k_sel[b, g, c] == m (the last row of k_tab is zero).
    q_tab[b, g, m]  fp32 vector added to every query (all heads of group g)
                    of query block t with q_sel[b, g, t] == m; in decode mode
                    q_sel[b, g, 0] applies to the single query token.
    seqlens[b]      decode context lengths (None for prefill).
    """

    k_tab: torch.Tensor
    k_sel: torch.Tensor
    q_tab: torch.Tensor
    q_sel: torch.Tensor
    seqlens: torch.Tensor | None
    w_s: torch.Tensor


def _rng(seed: int, tag: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag])))


def _orthonormal(rng: np.random.Generator, d: int, r: int) -> np.ndarray:
    q, _ = np.linalg.qr(rng.standard_normal((d, r)))
    return q.T.copy()  # [r, d], rows orthonormal


def w_s_matrix(cfg: Config, seed: int | None = None) -> torch.Tensor:
    """W_s = I + ws_noise * N(0,1), fp32 [d, d] row-major (CPU)."""
    seed = cfg.seed if seed is None else seed
    d = cfg.head_dim
    idx = torch.arange(d * d, dtype=torch.int64)
    n = draw(stream_key(seed, "w_s"), idx).reshape(d, d)
    return torch.eye(d, dtype=torch.float32) + torch.tensor(cfg.ws_noise, dtype=torch.float32) * n


def make_plan(cfg: Config, seed: int | None = None) -> Plan:
    seed = cfg.seed if seed is None else seed
    B, Hkv, d, T = cfg.batch, cfg.kv_heads, cfg.head_dim, cfg.n_blocks
    tq = 1 if cfg.mode == "decode" else T
    seqlens = None
    if cfg.mode == "decode":
        seqlens = torch.from_numpy(
            _rng(seed, 7).integers(cfg.seqlen_lo, cfg.seqlen_hi + 1, size=B).astype(np.int32)
        )

    if cfg.plant == "none" or (cfg.plant == "topics" and cfg.key_strength == 0.0 and cfg.query_strength == 0.0):
        k_tab = np.zeros((B, Hkv, 1, d), np.float32)
        q_tab = np.zeros((B, Hkv, 1, d), np.float32)
        k_sel = np.zeros((B, Hkv, T), np.int64)
        q_sel = np.zeros((B, Hkv, tq), np.int64)
    elif cfg.plant == "pr1":
        # One direction per query block t >= 1; min(3, t) distinct earlier key
        # blocks get key_strength * e_t added (a block may carry several); the
        # rows of block t get query_strength * e_t.
        rng = _rng(seed, 11)
        k_tab = np.zeros((B, Hkv, T + 1, d), np.float32)
        q_tab = np.zeros((B, Hkv, T + 1, d), np.float32)
        k_sel = np.tile(np.arange(T, dtype=np.int64), (B, Hkv, 1))
        q_sel = np.tile(np.arange(T, dtype=np.int64), (B, Hkv, 1))
        for b in range(B):
            for g in range(Hkv):
                e = _orthonormal(rng, d, max(T - 1, 1))
                acc = np.zeros((T, d), np.float64)
                for t in range(1, T):
                    chosen = rng.choice(t, size=min(3, t), replace=False)
                    for c in chosen:
                        acc[c] += cfg.key_strength * e[t - 1]
                    q_tab[b, g, t] = (cfg.query_strength * e[t - 1]).astype(np.float32)
                k_tab[b, g, :T] = acc.astype(np.float32)
        q_sel[:, :, 0] = T  # block 0 has no earlier block: no plant
    elif cfg.plant == "topics":
        # R orthonormal topic directions per (b, g); every key block and every
        # query block (or the decode query) draws a topic uniformly.
        R = cfg.n_topics
        rng = _rng(seed, 13)
        k_tab = np.zeros((B, Hkv, R + 1, d), np.float32)
        q_tab = np.zeros((B, Hkv, R + 1, d), np.float32)
        for b in range(B):
            for g in range(Hkv):
                e = _orthonormal(rng, d, R)
                k_tab[b, g, :R] = (np.float32(cfg.key_strength) * e.astype(np.float32))
                q_tab[b, g, :R] = (np.float32(cfg.query_strength) * e.astype(np.float32))
        k_sel = rng.integers(0, R, size=(B, Hkv, T)).astype(np.int64)
        q_sel = rng.integers(0, R, size=(B, Hkv, tq)).astype(np.int64)
    elif cfg.plant == "needles":
        # KV heads [0, Hkv/2) are diffuse (nothing planted).  For the others:
        # R topics, topic r owns m_r ~ U{1..16} disjoint random key blocks;
        # every query block takes a random topic.
        R = cfg.n_topics
        rng = _rng(seed, 17)
        k_tab = np.zeros((B, Hkv, R + 1, d), np.float32)
        q_tab = np.zeros((B, Hkv, R + 1, d), np.float32)
        k_sel = np.full((B, Hkv, T), R, np.int64)
        q_sel = np.full((B, Hkv, tq), R, np.int64)
        for b in range(B):
            for g in range(Hkv // 2, Hkv):
                e = _orthonormal(rng, d, R)
                k_tab[b, g, :R] = np.float32(cfg.key_strength) * e.astype(np.float32)
                q_tab[b, g, :R] = np.float32(cfg.query_strength) * e.astype(np.float32)
                m = rng.integers(1, 17, size=R)
                perm = rng.permutation(T)
                pos = 0
                for r in range(R):
                    k_sel[b, g, perm[pos:pos + m[r]]] = r
                    pos += m[r]
                q_sel[b, g] = rng.integers(0, R, size=tq)
    else:
        raise ValueError(f"unknown plant scheme {cfg.plant!r}")

    return Plan(
        k_tab=torch.from_numpy(k_tab), k_sel=torch.from_numpy(k_sel),
        q_tab=torch.from_numpy(q_tab), q_sel=torch.from_numpy(q_sel),
        seqlens=seqlens, w_s=w_s_matrix(cfg, seed),
    )


# --------------------------------------------------------------------------
# Tensor values


def _as_index(x, device) -> torch.Tensor:
    if isinstance(x, range):
        return torch.arange(x.start, x.stop, x.step, dtype=torch.int64, device=device)
    return torch.as_tensor(x, dtype=torch.int64).to(device)


def _base(cfg: Config, seed: int, tensor: str, b: int, s_idx, h_idx, s_total: int, h_total: int, device):
    d = cfg.head_dim
    s = _as_index(s_idx, device)
    h = _as_index(h_idx, device)
    e = torch.arange(d, dtype=torch.int64, device=device)
    flat = ((b * s_total + s[:, None, None]) * h_total + h[None, :, None]) * d + e[None, None, :]
    x = draw(stream_key(seed, tensor), flat)
    if cfg.scaled:
        x = x * torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32, device=device)
    return x, s, h


def q_values(cfg: Config, plan: Plan, b: int, s_idx, h_idx, device="cpu", seed=None,
             as_float32: bool = False) -> torch.Tensor:
    """Query values q[b, s, h, :] for the given positions and heads.

    Prefill: positions index the sequence.  Decode: the only position is 0
    (the query token sits at context position seqlens[b] - 1).
    Returns [len(s), len(h), d] in the config dtype (fp32 if as_float32,
    holding exactly the stored values).
    """
    seed = cfg.seed if seed is None else seed
    s_total = 1 if cfg.mode == "decode" else cfg.seq
    x, s, h = _base(cfg, seed, "q", b, s_idx, h_idx, s_total, cfg.heads, device)
    g = h // cfg.group
    if cfg.mode == "decode":
        m = plan.q_sel[b].to(device)[g, 0][None, :].expand(len(s), -1)
    else:
        m = plan.q_sel[b].to(device)[g[None, :], (s // cfg.block)[:, None]]
    x = x + plan.q_tab[b].to(device)[g[None, :].expand_as(m), m]
    x = x.to(torch_dtype(cfg.dtype))
    return x.float() if as_float32 else x


def kv_values(cfg: Config, plan: Plan, which: str, b: int, s_idx, g_idx, device="cpu", seed=None,
              as_float32: bool = False) -> torch.Tensor:
    """Key or value rows k[b, s, g, :] / v[b, s, g, :] -> [len(s), len(g), d]."""
    seed = cfg.seed if seed is None else seed
    x, s, g = _base(cfg, seed, which, b, s_idx, g_idx, cfg.seq, cfg.kv_heads, device)
    if which == "k":
        m = plan.k_sel[b].to(device)[g[None, :], (s // cfg.block)[:, None]]
        x = x + plan.k_tab[b].to(device)[g[None, :].expand_as(m), m]
    x = x.to(torch_dtype(cfg.dtype))
    return x.float() if as_float32 else x


def full_inputs(cfg: Config, device="cpu", seed=None, plan: Plan | None = None,
                chunk_elems: int = 1 << 25) -> dict:
    """All tensors of one instance, built chunk by chunk on ``device``.

    Returns q [B, Sq, H, d], k and v [B, S, Hkv, d] in the config dtype, W_s
    [d, d] fp32, seqlens [B] int32 (decode) or None, and the plan.
    """
    seed = cfg.seed if seed is None else seed
    plan = make_plan(cfg, seed) if plan is None else plan
    B, S, H, Hkv, d = cfg.batch, cfg.seq, cfg.heads, cfg.kv_heads, cfg.head_dim
    dt = torch_dtype(cfg.dtype)
    sq = 1 if cfg.mode == "decode" else S
    q = torch.empty((B, sq, H, d), dtype=dt, device=device)
    k = torch.empty((B, S, Hkv, d), dtype=dt, device=device)
    v = torch.empty((B, S, Hkv, d), dtype=dt, device=device)
    rows_q = max(1, chunk_elems // (H * d))
    rows_kv = max(1, chunk_elems // (Hkv * d))
    for b in range(B):
        for s0 in range(0, sq, rows_q):
            s1 = min(sq, s0 + rows_q)
            q[b, s0:s1] = q_values(cfg, plan, b, range(s0, s1), range(H), device, seed)
        for s0 in range(0, S, rows_kv):
            s1 = min(S, s0 + rows_kv)
            k[b, s0:s1] = kv_values(cfg, plan, "k", b, range(s0, s1), range(Hkv), device, seed)
            v[b, s0:s1] = kv_values(cfg, plan, "v", b, range(s0, s1), range(Hkv), device, seed)
    seqlens = None if plan.seqlens is None else plan.seqlens.to(device)
    return {"q": q, "k": k, "v": v, "w_s": plan.w_s.to(device), "seqlens": seqlens, "plan": plan}


def sample_rows(seq: int, block: int, stride: int = 97) -> list[int]:
    """Deterministic row subsample used for parity and CPU timing at full size.

    Every ``stride``-th row, all rows of the first two and last two blocks,
    and the first and last row of every block.
    """
    rows = set(range(0, seq, stride))
    nb = -(-seq // block)
    for c in (0, 1, nb - 2, nb - 1):
        if 0 <= c < nb:
            rows.update(range(c * block, min(seq, (c + 1) * block)))
    for c in range(nb):
        rows.add(c * block)
        rows.add(min(seq, (c + 1) * block) - 1)
    return sorted(r for r in rows if 0 <= r < seq)
