"""The synthetic workloads.

The pages measure DashAttention on MiniCPM-4 models over long-context
benchmarks (RULER, HELMET); neither the weights nor the datasets exist here.
These seeded configurations stand in for them: shapes, dtypes, block sizes
and alpha as the workloads name them, and "topic planting" (see
:mod:`gen.synth`) so that alpha-entmax routing becomes sparse at the target
rate the way trained attention would (about 75% of candidate blocks get zero
routing mass).

``key_strength`` values marked "calibrated" were chosen with
``oracle/calibrate.py``, which calls only the oracle and this package.
"""

from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Config:
    name: str
    mode: str  # "prefill" or "decode"
    batch: int
    heads: int
    kv_heads: int
    head_dim: int
    seq: int  # prefill: sequence length; decode: KV-cache capacity per sequence
    dtype: str  # "f32" | "f16" | "bf16"
    block: int
    alpha: float
    causal: bool = True
    scaled: bool = False  # entries N(0,1)/sqrt(d) instead of N(0,1)
    ws_noise: float = 0.0  # W_s = I + ws_noise * N(0,1)
    plant: str = "none"  # "none" | "pr1" | "topics" | "needles"
    n_topics: int = 0
    key_strength: float = 0.0
    query_strength: float = 0.0
    seqlen_lo: int = 0  # decode: context lengths drawn uniformly from [lo, hi]
    seqlen_hi: int = 0
    seed: int = 0

    @property
    def group(self) -> int:
        return self.heads // self.kv_heads

    @property
    def n_blocks(self) -> int:
        return -(-self.seq // self.block)

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


# Plant strengths (calibrated with oracle/calibrate.py on a row subsample).
# prefill: 4 -> 67.2%, 6 -> 73.1%, 8 -> 74.2% block-weighted sparsity; the
# ceiling is 75% (one topic in four), approached as N grows.
# long prefill needle heads: 6 -> 3.7%, 24 -> 94.5%, 32 -> 96.7% (the
# diffuse heads stay at 0%).
_PREFILL_KEY_STRENGTH = 8.0
_NEEDLE_KEY_STRENGTH = 24.0

CONFIGS: dict[str, Config] = {
    # 1K-token single-head fp32 case that the oracle runs in full.
    "pr1": Config(
        name="pr1", mode="prefill", batch=1, heads=1, kv_heads=1, head_dim=64,
        seq=1024, dtype="f32", block=64, alpha=1.5, scaled=False, ws_noise=0.1,
        plant="pr1", key_strength=2.0, query_strength=8.0, seed=0,
    ),
    # 32K GQA bf16 prefill: the headline throughput workload.
    "prefill": Config(
        name="prefill", mode="prefill", batch=1, heads=32, kv_heads=8, head_dim=128,
        seq=32768, dtype="bf16", block=64, alpha=1.5, scaled=True, ws_noise=0.05,
        plant="topics", n_topics=4, key_strength=_PREFILL_KEY_STRENGTH,
        query_strength=1.0, seed=0,
    ),
    # 64 sequences decoding one token against 64K..128K of cached context.
    "decode": Config(
        name="decode", mode="decode", batch=64, heads=32, kv_heads=8, head_dim=128,
        seq=131072, dtype="bf16", block=64, alpha=1.5, scaled=True, ws_noise=0.05,
        plant="topics", n_topics=4, key_strength=_PREFILL_KEY_STRENGTH,
        query_strength=1.0, seqlen_lo=65536, seqlen_hi=131072, seed=0,
    ),
    # 128K prefill with block 128; KV heads 0-3 diffuse, 4-7 needle heads.
    "long_prefill": Config(
        name="long_prefill", mode="prefill", batch=1, heads=32, kv_heads=8, head_dim=128,
        seq=131072, dtype="bf16", block=128, alpha=1.5, scaled=True, ws_noise=0.05,
        plant="needles", n_topics=64, key_strength=_NEEDLE_KEY_STRENGTH,
        query_strength=1.0, seed=0,
    ),
    # alpha / sparsity sweep base point (alpha and key_strength vary).
    "sweep": Config(
        name="sweep", mode="prefill", batch=4, heads=16, kv_heads=16, head_dim=64,
        seq=16384, dtype="f16", block=64, alpha=1.5, scaled=False, ws_noise=0.05,
        plant="topics", n_topics=16, key_strength=2.0, query_strength=8.0, seed=0,
    ),
}

SWEEP_ALPHAS = (1.25, 1.5, 2.0)
SWEEP_STRENGTHS = (0.0, 1.0, 2.0, 4.0)


def get_config(name: str) -> Config:
    return CONFIGS[name]


def sweep_configs() -> list[Config]:
    base = CONFIGS["sweep"]
    return [
        base.with_(name=f"sweep_a{a}_s{s:g}", alpha=a, key_strength=s)
        for a in SWEEP_ALPHAS
        for s in SWEEP_STRENGTHS
    ]
