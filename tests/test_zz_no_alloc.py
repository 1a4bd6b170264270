"""The decode step without a workspace (dash_attn_decode_noalloc).

Some callers may not allocate device memory while they run: code inside
another engine's execution hook (a serving runtime or graph-executor plugin),
where allocation is forbidden or would stall the device, and programs that
fix their device-memory budget at start-up.  They call the decode entry
point that keeps its scratch in a fixed library-owned array; it must give
the same results as the regular entry point with a caller workspace, call
after call.  This file is collected last so that a failure here never hides
another test's result.
"""

import pytest
import torch

from gen import full_inputs, get_config
from tests._parity import OUT_TOL, max_abs

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode(cuda_lib):
    dash = cuda_lib
    cfg = get_config("decode").with_(batch=5, seq=4096, seqlen_lo=1, seqlen_hi=4096)
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w, sl = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["seqlens"]
    summ = dash.summarize(k, w, cfg.block, seqlens=sl)
    ref = dash.decode(q, k, v, sl, summ, cfg.alpha, cfg.block)
    torch.cuda.synchronize()
    for _ in range(2):  # two calls in a row share the scratch array
        got = dash.decode_noalloc(q, k, v, sl, summ, cfg.alpha, cfg.block)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        assert max_abs(got.float().cpu(), ref.float().cpu()) <= OUT_TOL[cfg.dtype]


def test_noalloc_decode_refuses_problems_beyond_its_scratch(cuda_lib):
    dash = cuda_lib
    # 64 sequences x 8 KV heads x 2048 blocks: far more than 16 MiB of scratch.
    # Expanded views keep the device memory of this check small.
    q = torch.zeros(64, 1, 32, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(1, 131072, 8, 128, dtype=torch.bfloat16, device="cuda").expand(64, -1, -1, -1)
    summ = torch.zeros(1, 8, 2048, 128, dtype=torch.float32, device="cuda").expand(64, -1, -1, -1)
    sl = torch.full((64,), 1000, dtype=torch.int32, device="cuda")
    with pytest.raises(dash.DashError) as e:
        dash.decode_noalloc(q, kc, kc, sl, summ, 1.5, 64)
    assert e.value.status == 2
    assert "scratch" in str(e.value)


def test_noalloc_decode_reports_bad_seqlens_through_its_status(cuda_lib):
    # the status word lives in the library-owned array; the accessor reads it
    # without allocating: an out-of-range context length is clamped on the
    # device and reported, and the next valid call reports success again
    dash = cuda_lib
    cfg = get_config("decode").with_(batch=3, seq=2048, seqlen_lo=100, seqlen_hi=2048)
    inp = full_inputs(cfg, device="cuda")
    q, k, v, w, sl = inp["q"], inp["k"], inp["v"], inp["w_s"], inp["seqlens"]
    summ = dash.summarize(k, w, cfg.block, seqlens=sl)
    bad = sl.clone()
    bad[1] = cfg.seq + 5
    dash.decode_noalloc(q, k, v, bad, summ, cfg.alpha, cfg.block)
    assert dash.decode_noalloc_status() == 1
    dash.decode_noalloc(q, k, v, sl, summ, cfg.alpha, cfg.block)
    assert dash.decode_noalloc_status() == 0
