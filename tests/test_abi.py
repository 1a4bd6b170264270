"""The C-ABI library: it loads, exports every symbol include/dashattn.h
declares, and rejects bad arguments on the host before touching the GPU.

These run without a GPU: the argument checks return before any CUDA call,
and the pointers handed in are never dereferenced.
"""

import ctypes
import os
import re
import subprocess

import pytest

import sparse_hierarchical_attention_mean_b200 as dash
from sparse_hierarchical_attention_mean_b200 import DashTensor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dashattn.h")

FAKE = 0x100000  # 256-byte aligned, never dereferenced


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(dash_attn_\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    lib = dash.load()
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(dash.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", dash.library_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (dash_attn_\w+)", out))
    assert set(names) <= exported
    assert dash.version() == 100


def tensor(b, s, h, d, dtype=2, data=FAKE, strides=None):
    sb, ss, sh = strides or (s * h * d, h * d, d)
    return DashTensor(data, dtype, 0, b, s, h, d, sb, ss, sh)


def call_fwd(q, k, v, out, alpha=1.5, block=64, ws_bytes=1 << 40, ws=FAKE):
    lib = dash.load()
    st = lib.dash_attn_fwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), FAKE, alpha, block, 1,
                           ctypes.byref(out), ws, ws_bytes, None)
    return st, lib.dash_attn_last_error().decode()


def good():
    return tensor(1, 256, 8, 128), tensor(1, 256, 2, 128), tensor(1, 256, 2, 128), tensor(1, 256, 8, 128)


@pytest.mark.parametrize(
    "mutate, status, text",
    [
        (lambda q, k, v, o: setattr(q, "d", 96), 2, "head dim"),
        (lambda q, k, v, o: setattr(k, "dtype", 1), 1, "dtype"),
        (lambda q, k, v, o: setattr(q, "dtype", 7), 1, "dtype"),
        (lambda q, k, v, o: (setattr(k, "h", 3), setattr(v, "h", 3)), 1, "multiple"),
        (lambda q, k, v, o: (setattr(q, "h", 48), setattr(o, "h", 48), setattr(k, "h", 3), setattr(v, "h", 3)), 2,
         "group size"),
        (lambda q, k, v, o: setattr(q, "data", FAKE + 8), 1, "aligned"),
        (lambda q, k, v, o: setattr(q, "data", 0), 1, "null"),
        (lambda q, k, v, o: setattr(q, "stride_s", 8 * 128 + 4), 1, "16 bytes"),
        (lambda q, k, v, o: setattr(k, "s", 255), 1, "equal length"),
        (lambda q, k, v, o: setattr(o, "s", 100), 1, "shape"),
        (lambda q, k, v, o: setattr(v, "b", 2), 1, "batch"),
    ],
)
def test_fwd_rejects_bad_arguments(mutate, status, text):
    q, k, v, o = good()
    mutate(q, k, v, o)
    st, msg = call_fwd(q, k, v, o)
    assert st == status, msg
    assert text in msg


@pytest.mark.parametrize("alpha, block, status", [(1.0, 64, 1), (2.5, 64, 1), (float("nan"), 64, 1), (1.5, 32, 2)])
def test_fwd_rejects_alpha_and_block(alpha, block, status):
    st, msg = call_fwd(*good(), alpha=alpha, block=block)
    assert st == status, msg


def test_workspace_size_and_too_small():
    q, k, v, o = good()
    lib = dash.load()
    need = lib.dash_attn_fwd_workspace_size(ctypes.byref(q), ctypes.byref(k), 64)
    T = 4
    # summaries + lists + counts + union lists, each 256-aligned
    assert need >= 2 * 256 * T * 4 * 2 + 2 * T * 128 * 4
    st, msg = call_fwd(q, k, v, o, ws_bytes=need - 1)
    assert st == 3 and "workspace" in msg
    st, msg = call_fwd(q, k, v, o, ws=FAKE + 16)
    assert st == 1 and "256-byte" in msg
    bad = tensor(1, 256, 8, 96)
    assert lib.dash_attn_fwd_workspace_size(ctypes.byref(bad), ctypes.byref(k), 64) == 0


def test_decode_and_route_reject_bad_arguments():
    lib = dash.load()
    q = tensor(4, 1, 8, 128)
    kc = tensor(4, 4096, 2, 128)
    o = tensor(4, 1, 8, 128)
    ws = lib.dash_attn_decode_workspace_size(ctypes.byref(q), ctypes.byref(kc), 64, 64)
    assert ws > 0
    st = lib.dash_attn_decode(ctypes.byref(q), ctypes.byref(kc), ctypes.byref(kc), FAKE, FAKE, 32, 1.5, 64,
                              ctypes.byref(o), FAKE, ws, None)
    assert st == 1 and "t_cap" in lib.dash_attn_last_error().decode()
    q2 = tensor(4, 2, 8, 128)
    st = lib.dash_attn_decode(ctypes.byref(q2), ctypes.byref(kc), ctypes.byref(kc), FAKE, FAKE, 64, 1.5, 64,
                              ctypes.byref(o), FAKE, ws, None)
    assert st == 1
    qf = tensor(4, 1, 8, 128, dtype=0)
    of = tensor(4, 1, 8, 128, dtype=0)
    kf = tensor(4, 4096, 2, 128, dtype=0)
    st = lib.dash_attn_decode(ctypes.byref(qf), ctypes.byref(kf), ctypes.byref(kf), FAKE, FAKE, 64, 1.5, 64,
                              ctypes.byref(of), FAKE, ws, None)
    assert st == 2
    st = lib.dash_attn_decode(ctypes.byref(q), ctypes.byref(kc), ctypes.byref(kc), FAKE, FAKE, 64, 1.5, 64,
                              ctypes.byref(o), FAKE, ws - 1, None)
    assert st == 3
    # route: decode mode needs a workspace
    st = lib.dash_attn_route(ctypes.byref(q), FAKE, 2, 64, FAKE, 1.5, 64, 1, FAKE, FAKE, FAKE, None, None, None, 0,
                             None)
    assert st == 1
    st = lib.dash_attn_route(ctypes.byref(q), FAKE, 3, 64, None, 1.5, 64, 1, FAKE, FAKE, FAKE, None, None, None, 0,
                             None)
    assert st == 1
    st = lib.dash_attn_summarize(ctypes.byref(kc), None, FAKE, 64, FAKE, 10, 0, None)
    assert st == 1 and "t_cap" in lib.dash_attn_last_error().decode()
    # learned summary queries: misaligned qbar, and the same checks as summarize
    st = lib.dash_attn_summarize_sdpa(ctypes.byref(kc), None, FAKE, FAKE + 4, 64, FAKE, 64, 0, None)
    assert st == 1 and "aligned" in lib.dash_attn_last_error().decode()
    st = lib.dash_attn_summarize_sdpa(ctypes.byref(kc), None, FAKE, FAKE, 96, FAKE, 64, 0, None)
    assert st == 2
    # options: negative sigma; a learned query where no summaries are computed
    bad = dash.DashOptions(-1.0, None)
    st = lib.dash_attn_decode_ex(ctypes.byref(q), ctypes.byref(kc), ctypes.byref(kc), FAKE, FAKE, 64, 1.5, 64,
                                 ctypes.byref(o), FAKE, ws, ctypes.byref(bad), None)
    assert st == 1 and "sigma" in lib.dash_attn_last_error().decode()
    withq = dash.DashOptions(1.0, FAKE)
    st = lib.dash_attn_decode_ex(ctypes.byref(q), ctypes.byref(kc), ctypes.byref(kc), FAKE, FAKE, 64, 1.5, 64,
                                 ctypes.byref(o), FAKE, ws, ctypes.byref(withq), None)
    assert st == 1 and "qbar" in lib.dash_attn_last_error().decode()
    # masks: too few words for the list capacity
    st = lib.dash_attn_lists_to_mask(FAKE, FAKE, 10, 100, FAKE, 3, None)
    assert st == 1 and "n_words" in lib.dash_attn_last_error().decode()


def test_paged_and_context_parallel_reject_bad_arguments():
    lib = dash.load()
    q = tensor(4, 1, 8, 128)
    o = tensor(4, 1, 8, 128)
    pages = tensor(100, 64, 2, 128)
    # page size must equal the block; a block table is required
    st = lib.dash_attn_decode_paged(ctypes.byref(q), ctypes.byref(pages), ctypes.byref(pages), FAKE, 16, FAKE, FAKE, 64,
                                    1.5, 128, ctypes.byref(o), FAKE, 1 << 30, None, None)
    assert st == 1 and "page size" in lib.dash_attn_last_error().decode()
    st = lib.dash_attn_decode_paged(ctypes.byref(q), ctypes.byref(pages), ctypes.byref(pages), None, 16, FAKE, FAKE, 64,
                                    1.5, 64, ctypes.byref(o), FAKE, 1 << 30, None, None)
    assert st == 1 and "block table" in lib.dash_attn_last_error().decode()
    st = lib.dash_attn_decode_paged(ctypes.byref(q), ctypes.byref(pages), ctypes.byref(pages), FAKE, 16, FAKE, FAKE, 8,
                                    1.5, 64, ctypes.byref(o), FAKE, 1 << 30, None, None)
    assert st == 1 and "t_cap" in lib.dash_attn_last_error().decode()
    st = lib.dash_attn_summarize_paged(ctypes.byref(pages), FAKE, 16, 4, FAKE, FAKE, None, 64, FAKE, 8, 0, None)
    assert st == 1 and "t_cap" in lib.dash_attn_last_error().decode()
    # context parallelism: shard ranges must be block-aligned, the block range must fit
    shard = tensor(4, 100, 2, 128)
    st = lib.dash_attn_cp_attend(ctypes.byref(q), ctypes.byref(shard), ctypes.byref(shard), 64, FAKE, 4096, FAKE, FAKE,
                                 FAKE, 64, 64, None, FAKE, None)
    assert st == 1 and "multiples of the block" in lib.dash_attn_last_error().decode()
    st = lib.dash_attn_cp_scores(ctypes.byref(q), 2, FAKE, 8, 10, 30, FAKE, 4096, 1.5, 64, FAKE, 64, None)
    assert st == 1 and "block range" in lib.dash_attn_last_error().decode()
    qf = tensor(4, 1, 8, 128, dtype=0)
    st = lib.dash_attn_cp_lists(ctypes.byref(qf), 2, FAKE, FAKE, 4096, 1.5, 64, FAKE, FAKE, FAKE, 64, None)
    assert st == 2


def test_context_parallel_split_kv_workspace_checks():
    """dash_attn_cp_attend_ex: its workspace size, and the host checks of the shard and the workspace."""
    lib = dash.load()
    B, H, Hkv, d, blk, t_cap = 4, 8, 2, 128, 64, 64
    n = lib.dash_attn_cp_attend_workspace_size(B, H, Hkv, d, blk, t_cap)
    # shard ranges [4 ints], work items of 16 blocks (block 64) with G heads' partials each
    items = B * Hkv * (-(-(t_cap + 1) // 16))
    assert n >= B * Hkv * 16 + items * 8 + B * Hkv * 4 + items * (H // Hkv) * (d + 2) * 4
    assert n % 256 == 0
    assert lib.dash_attn_cp_attend_workspace_size(B, H, Hkv, d, 128, t_cap) > n  # 8-block items: more of them
    assert lib.dash_attn_cp_attend_workspace_size(B, H, 3, d, blk, t_cap) == 0  # H not a multiple of Hkv
    assert lib.dash_attn_cp_attend_workspace_size(0, H, Hkv, d, blk, t_cap) == 0
    q = tensor(B, 1, H, d)
    shard = tensor(B, 1024, Hkv, d)

    def call(shard_t=shard, tok_lo=1024, ws=FAKE, ws_bytes=n):
        st = lib.dash_attn_cp_attend_ex(ctypes.byref(q), ctypes.byref(shard_t), ctypes.byref(shard_t), tok_lo, FAKE,
                                        4096, FAKE, FAKE, FAKE, t_cap, blk, None, FAKE, ws, ws_bytes, None)
        return st, lib.dash_attn_last_error().decode()

    st, msg = call(tok_lo=1000)
    assert st == 1 and "multiples of the block" in msg
    st, msg = call(shard_t=tensor(B, 1000, Hkv, d))
    assert st == 1 and "multiples of the block" in msg
    st, msg = call(ws=None)
    assert st == 1 and "256-byte aligned" in msg
    st, msg = call(ws=FAKE + 128)
    assert st == 1 and "256-byte aligned" in msg
    st, msg = call(ws_bytes=n - 1)
    assert st == 3 and "workspace" in msg
    st, msg = call(shard_t=tensor(B, 1024, Hkv, d, dtype=1))
    assert st == 1 and "dtype" in msg


def test_binding_refuses_host_tensors():
    import torch

    x = torch.zeros(1, 64, 1, 64)
    with pytest.raises(ValueError):
        dash.fwd(x, x, x, torch.zeros(64, 64), 1.5, 64)


def call_bwd(q, k, v, o, do, dq, dk, dv, ws_bytes=1 << 42, opts=None, dw_s=FAKE):
    lib = dash.load()
    st = lib.dash_attn_bwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), FAKE, ctypes.byref(o), ctypes.byref(do),
                           1.5, 64, 1, opts, ctypes.byref(dq), ctypes.byref(dk), ctypes.byref(dv), dw_s, FAKE,
                           ws_bytes, None)
    return st, lib.dash_attn_last_error().decode()


def good_bwd():
    q, k, v, o = good()
    return q, k, v, o, tensor(1, 256, 8, 128), tensor(1, 256, 8, 128, dtype=0), tensor(1, 256, 2, 128, dtype=0), \
        tensor(1, 256, 2, 128, dtype=0)


@pytest.mark.parametrize(
    "mutate, status, text",
    [
        (lambda a: [setattr(t, "dtype", 0) for t in a[:5]], 2, "f16 or bf16"),
        (lambda a: setattr(a[5], "dtype", 2), 1, "fp32"),
        (lambda a: setattr(a[6], "h", 8), 1, "shape of its input"),
        (lambda a: setattr(a[4], "s", 128), 1, "dout"),
        (lambda a: setattr(a[4], "dtype", 1), 1, "dout"),
        (lambda a: setattr(a[7], "data", FAKE + 4), 1, "aligned"),
    ],
)
def test_bwd_rejects_bad_arguments(mutate, status, text):
    args = list(good_bwd())
    mutate(args)
    st, msg = call_bwd(*args)
    assert st == status, msg
    assert text in msg


def test_bwd_workspace_options_and_outputs():
    lib = dash.load()
    q, k, v, o, do, dq, dk, dv = good_bwd()
    need = lib.dash_attn_bwd_workspace_size(ctypes.byref(q), ctypes.byref(k), 64)
    # at least the per-head routing gradients [B, Hkv, S, T, G] fp32
    assert need >= 1 * 2 * 256 * 4 * 4 * 4
    st, msg = call_bwd(q, k, v, o, do, dq, dk, dv, ws_bytes=need - 1)
    assert st == 3 and "workspace" in msg
    st, msg = call_bwd(q, k, v, o, do, dq, dk, dv, dw_s=None)
    assert st == 1 and "dw_s" in msg
    opts = dash.DashOptions(1.0, FAKE)
    st, msg = call_bwd(q, k, v, o, do, dq, dk, dv, opts=ctypes.byref(opts))
    assert st == 1 and "qbar" in msg
    opts = dash.DashOptions(-1.0, None)
    st, msg = call_bwd(q, k, v, o, do, dq, dk, dv, opts=ctypes.byref(opts))
    assert st == 1 and "sigma" in msg
