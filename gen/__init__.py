"""Seeded synthetic inputs for the DashAttention forward.

This package is shared by the fp64 oracle tests and by the CUDA path.  It
holds no arithmetic of the attention method: only value generation, topic
planting and row sampling.  See :mod:`gen.synth` for the generator and
:mod:`gen.configs` for the workloads.
"""

from .configs import CONFIGS, Config, get_config, sweep_configs  # noqa: F401
from .synth import (  # noqa: F401
    Plan,
    draw,
    full_inputs,
    kv_values,
    make_plan,
    q_values,
    sample_rows,
    w_s_matrix,
)
