"""The seeded input generator: determinism, slicing and distribution."""

import numpy as np
import torch

from gen import draw, full_inputs, get_config, kv_values, make_plan, q_values, sample_rows
from gen.synth import stream_key


def test_draw_is_deterministic_and_normal():
    idx = torch.arange(1 << 20, dtype=torch.int64)
    a = draw(stream_key(0, "k"), idx)
    b = draw(stream_key(0, "k"), idx)
    assert torch.equal(a, b)
    assert abs(a.mean().item()) < 5e-3
    assert abs(a.std().item() - 1.0) < 5e-3
    # different streams and seeds differ
    assert not torch.equal(a, draw(stream_key(0, "v"), idx))
    assert not torch.equal(a, draw(stream_key(1, "k"), idx))
    # a slice is the same values as the full draw
    sub = torch.tensor([5, 77, 1 << 19, (1 << 20) - 1])
    assert torch.equal(draw(stream_key(0, "k"), sub), a[sub])
    # indices above 2^32 are distinct streams of values
    hi = draw(stream_key(0, "k"), idx + (1 << 33))
    assert not torch.equal(a, hi)


def test_slices_match_full_tensors():
    cfg = get_config("prefill").with_(seq=640)
    inp = full_inputs(cfg)
    plan = inp["plan"]
    rows = [0, 63, 64, 639]
    assert torch.equal(q_values(cfg, plan, 0, rows, [0, 5, 31]), inp["q"][0, rows][:, [0, 5, 31]])
    assert torch.equal(kv_values(cfg, plan, "k", 0, rows, [2, 7]), inp["k"][0, rows][:, [2, 7]])
    assert torch.equal(kv_values(cfg, plan, "v", 0, rows, [3]), inp["v"][0, rows][:, [3]])
    assert inp["q"].dtype == torch.bfloat16


def test_decode_plan_and_plants():
    cfg = get_config("decode").with_(batch=3, seq=2048, seqlen_lo=700, seqlen_hi=2048)
    plan = make_plan(cfg)
    assert plan.seqlens.dtype == torch.int32
    assert int(plan.seqlens.min()) >= 700 and int(plan.seqlens.max()) <= 2048
    # planted key blocks of the query's topic carry the query direction
    b, g = 1, 2
    k = kv_values(cfg, plan, "k", b, range(2048), [g], as_float32=True)[:, 0]
    e = plan.q_tab[b, g, plan.q_sel[b, g, 0]]
    e = e / e.norm()
    proj = (k.reshape(-1, cfg.block, cfg.head_dim).mean(1) @ e).numpy()
    match = (plan.k_sel[b, g] == plan.q_sel[b, g, 0]).numpy()
    assert proj[match].min() > proj[~match].max()


def test_pr1_plan():
    cfg = get_config("pr1")
    plan = make_plan(cfg)
    # block 0 queries carry no plant; later blocks carry sqrt(d) along e_t
    assert float(plan.q_tab[0, 0, plan.q_sel[0, 0, 0]].abs().max()) == 0.0
    norms = plan.q_tab[0, 0, 1:cfg.n_blocks].norm(dim=-1)
    np.testing.assert_allclose(norms.numpy(), 8.0, rtol=1e-6)


def test_sample_rows():
    rows = sample_rows(32768, 64)
    assert rows == sorted(set(rows))
    assert set(range(0, 128)) <= set(rows) and set(range(32768 - 128, 32768)) <= set(rows)
    assert {64 * 100, 64 * 100 + 63} <= set(rows)
    assert all(0 <= r < 32768 for r in rows)
