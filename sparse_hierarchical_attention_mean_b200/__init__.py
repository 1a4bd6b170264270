"""Python binding of libdashattn (the DashAttention forward and backward for B200).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/dashattn.h``.  PyTorch is used
for device memory and the current CUDA stream.  The library must have been
built (``python -m sparse_hierarchical_attention_mean_b200._build``); loading
fails loudly otherwise -- there is no fallback implementation.

Layouts (FlashAttention convention, last dim contiguous):
q, out [B, S, H, d]; k, v [B, S, Hkv, d]; summaries [B, Hkv, T, d] fp32.
"""

from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdashattn.so")

DASH_OK = 0
_STATUS = {
    0: "DASH_OK",
    1: "DASH_ERR_INVALID_ARGUMENT",
    2: "DASH_ERR_UNSUPPORTED",
    3: "DASH_ERR_WORKSPACE_TOO_SMALL",
    4: "DASH_ERR_CUDA",
    5: "DASH_ERR_DEVICE_TIMEOUT",
}
_DTYPE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}

# Every symbol include/dashattn.h declares.
EXPORTED = (
    "dash_attn_version",
    "dash_attn_last_error",
    "dash_attn_fwd_workspace_size",
    "dash_attn_fwd_workspace_lists",
    "dash_attn_decode_workspace_lists",
    "dash_attn_fwd",
    "dash_attn_summarize",
    "dash_attn_summarize_sdpa",
    "dash_attn_fwd_ex",
    "dash_attn_sparse_ex",
    "dash_attn_sparse_mask",
    "dash_attn_debug_sparse_stalled",
    "dash_attn_decode_ex",
    "dash_attn_lists_to_mask",
    "dash_attn_cp_scores",
    "dash_attn_cp_lists",
    "dash_attn_cp_attend",
    "dash_attn_cp_attend_workspace_size",
    "dash_attn_cp_attend_ex",
    "dash_attn_cp_merge",
    "dash_attn_summarize_paged",
    "dash_attn_decode_paged",
    "dash_attn_decode_workspace_size",
    "dash_attn_decode",
    "dash_attn_route_workspace_size",
    "dash_attn_route",
    "dash_attn_sparse_workspace_size",
    "dash_attn_sparse",
    "dash_attn_get_device_status",
    "dash_attn_decode_noalloc",
    "dash_attn_decode_noalloc_status",
    "dash_attn_bwd_workspace_size",
    "dash_attn_bwd",
)


class DashError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


class DashOptions(ctypes.Structure):
    _fields_ = [("sigma", ctypes.c_float), ("qbar", ctypes.c_void_p)]


class DashTensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("b", ctypes.c_int64),
        ("s", ctypes.c_int64),
        ("h", ctypes.c_int64),
        ("d", ctypes.c_int64),
        ("stride_b", ctypes.c_int64),
        ("stride_s", ctypes.c_int64),
        ("stride_h", ctypes.c_int64),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python -m sparse_hierarchical_attention_mean_b200._build`"
        )
    lib = ctypes.CDLL(_LIB_PATH)
    T = ctypes.POINTER(DashTensor)
    O = ctypes.POINTER(DashOptions)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "dash_attn_version": (i32, []),
        "dash_attn_last_error": (ctypes.c_char_p, []),
        "dash_attn_fwd_workspace_size": (sz, [T, T, i32]),
        "dash_attn_fwd_workspace_lists": (i32, [T, T, i32, vp, vp, vp, vp]),
        "dash_attn_decode_workspace_lists": (i32, [T, T, i32, i64, vp, vp, vp]),
        "dash_attn_fwd": (i32, [T, T, T, vp, f32, i32, i32, T, vp, sz, vp]),
        "dash_attn_summarize": (i32, [T, vp, vp, i32, vp, i64, i64, vp]),
        "dash_attn_summarize_sdpa": (i32, [T, vp, vp, vp, i32, vp, i64, i64, vp]),
        "dash_attn_decode_workspace_size": (sz, [T, T, i32, i64]),
        "dash_attn_decode": (i32, [T, T, T, vp, vp, i64, f32, i32, T, vp, sz, vp]),
        "dash_attn_route_workspace_size": (sz, [T, i64, i64, i32]),
        "dash_attn_route": (i32, [T, vp, i64, i64, vp, f32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]),
        "dash_attn_sparse_workspace_size": (sz, [T, T, i32, i64]),
        "dash_attn_sparse": (i32, [T, T, T, vp, vp, vp, i64, i32, i32, T, vp, sz, vp]),
        "dash_attn_fwd_ex": (i32, [T, T, T, vp, f32, i32, i32, T, vp, sz, O, vp]),
        "dash_attn_sparse_ex": (i32, [T, T, T, vp, vp, vp, i64, i32, i32, T, vp, sz, O, vp]),
        "dash_attn_sparse_mask": (i32, [T, T, T, vp, i64, vp, i64, i32, i32, T, vp, sz, O, vp]),
        "dash_attn_debug_sparse_stalled": (i32, [T, T, T, vp, vp, vp, i64, i32, i32, T, vp, sz, i64, vp]),
        "dash_attn_decode_ex": (i32, [T, T, T, vp, vp, i64, f32, i32, T, vp, sz, O, vp]),
        "dash_attn_lists_to_mask": (i32, [vp, vp, i64, i64, vp, i64, vp]),
        "dash_attn_cp_scores": (i32, [T, i64, vp, i64, i64, i64, vp, i64, f32, i32, vp, i64, vp]),
        "dash_attn_cp_lists": (i32, [T, i64, vp, vp, i64, f32, i32, vp, vp, vp, i64, vp]),
        "dash_attn_cp_attend": (i32, [T, T, T, i64, vp, i64, vp, vp, vp, i64, i32, O, vp, vp]),
        "dash_attn_cp_attend_workspace_size": (sz, [i64, i64, i64, i64, i32, i64]),
        "dash_attn_cp_attend_ex": (i32, [T, T, T, i64, vp, i64, vp, vp, vp, i64, i32, O, vp, vp, sz, vp]),
        "dash_attn_cp_merge": (i32, [vp, i64, T, vp]),
        "dash_attn_summarize_paged": (i32, [T, vp, i64, i64, vp, vp, vp, i32, vp, i64, i64, vp]),
        "dash_attn_decode_paged": (i32, [T, T, T, vp, i64, vp, vp, i64, f32, i32, T, vp, sz, O, vp]),
        "dash_attn_get_device_status": (i32, [vp, vp]),
        "dash_attn_decode_noalloc": (i32, [T, T, T, vp, vp, i64, f32, i32, T, vp]),
        "dash_attn_decode_noalloc_status": (i32, [vp]),
        "dash_attn_bwd_workspace_size": (sz, [T, T, i32]),
        "dash_attn_bwd": (i32, [T, T, T, vp, T, T, f32, i32, i32, O, T, T, T, vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


class _Lazy:
    """Loads the library on first use (so the build step can import this package)."""

    _cdll = None

    def __getattr__(self, name):
        if _Lazy._cdll is None:
            _Lazy._cdll = _load()
        return getattr(_Lazy._cdll, name)


_lib = _Lazy()


def library_path() -> str:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Loads (once) and returns the library; raises ImportError if it is missing."""
    _lib.dash_attn_version  # noqa: B018
    return _Lazy._cdll


def version() -> int:
    return _lib.dash_attn_version()


def _check(status: int) -> None:
    if status != DASH_OK:
        raise DashError(status, _lib.dash_attn_last_error().decode())


def _desc(t: torch.Tensor) -> DashTensor:
    if t.dim() != 4:
        raise ValueError("expected a [B, S, H, d] tensor")
    if not t.is_cuda:
        raise ValueError("tensors must be CUDA device tensors")
    if t.stride(3) != 1:
        raise ValueError("the last dimension must be contiguous")
    if t.dtype not in _DTYPE:
        raise ValueError(f"unsupported dtype {t.dtype}")
    b, s, h, d = t.shape
    return DashTensor(t.data_ptr(), _DTYPE[t.dtype], 0, b, s, h, d, t.stride(0), t.stride(1), t.stride(2))


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _options(sigma: float, qbar: torch.Tensor | None):
    """None for the defaults (sigma 1, mean pooling), else a pointer to DashOptions."""
    if sigma == 1.0 and qbar is None:
        return None
    if qbar is not None:
        assert qbar.is_cuda and qbar.is_contiguous() and qbar.dtype == torch.float32
    return ctypes.byref(DashOptions(float(sigma), None if qbar is None else qbar.data_ptr()))


def _workspace(nbytes: int, device, given: torch.Tensor | None) -> torch.Tensor:
    if given is not None:
        return given
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def n_blocks(seq: int, block: int) -> int:
    return -(-seq // block)


# ------------------------------------------------------------------ stage 0


def summarize(k: torch.Tensor, w_s: torch.Tensor, block: int, seqlens: torch.Tensor | None = None,
              summaries: torch.Tensor | None = None, first_block: int = 0, stream=None,
              qbar: torch.Tensor | None = None) -> torch.Tensor:
    """Block summaries [B, Hkv, t_cap, d] fp32 (see dash_attn_summarize).

    qbar: optional fp32 [Hkv, d] learned summary queries (dash_attn_summarize_sdpa).
    """
    B, S, Hkv, d = k.shape
    if summaries is None:
        summaries = torch.zeros((B, Hkv, n_blocks(S, block), d), dtype=torch.float32, device=k.device)
    assert summaries.is_contiguous() and summaries.dtype == torch.float32
    kd = _desc(k)
    if qbar is None:
        _check(_lib.dash_attn_summarize(ctypes.byref(kd), _ptr(seqlens), w_s.data_ptr(), block,
                                        summaries.data_ptr(), summaries.shape[2], first_block, _stream(stream)))
    else:
        assert qbar.is_contiguous() and qbar.dtype == torch.float32 and tuple(qbar.shape) == (Hkv, d)
        _check(_lib.dash_attn_summarize_sdpa(ctypes.byref(kd), _ptr(seqlens), w_s.data_ptr(), qbar.data_ptr(),
                                             block, summaries.data_ptr(), summaries.shape[2], first_block,
                                             _stream(stream)))
    return summaries


# ------------------------------------------------------------------ stage 1


def route_workspace_size(q: torch.Tensor, kv_heads: int, t_cap: int, decode: bool) -> int:
    qd = _desc(q)
    return _lib.dash_attn_route_workspace_size(ctypes.byref(qd), kv_heads, t_cap, 1 if decode else 0)


def route(q: torch.Tensor, summaries: torch.Tensor, alpha: float, block: int, causal: bool = True,
          seqlens: torch.Tensor | None = None, want_tau: bool = False, want_p: bool = False,
          idx=None, logp=None, cnt=None, workspace=None, stream=None) -> dict:
    """Stage 1 alone; returns idx, logp [B, Hkv, Sq, t_cap], cnt [B, Hkv, Sq] (+ tau, p).

    idx / logp / cnt / workspace may be passed in to reuse buffers.
    """
    B, Sq, H, d = q.shape
    _, Hkv, t_cap, _ = summaries.shape
    dev = q.device
    if idx is None:
        idx = torch.full((B, Hkv, Sq, t_cap), -1, dtype=torch.int32, device=dev)
    if logp is None:
        logp = torch.zeros((B, Hkv, Sq, t_cap), dtype=torch.float32, device=dev)
    if cnt is None:
        cnt = torch.zeros((B, Hkv, Sq), dtype=torch.int32, device=dev)
    tau = torch.zeros((B, H, Sq), dtype=torch.float32, device=dev) if want_tau else None
    p = torch.zeros((B, H, Sq, t_cap), dtype=torch.float32, device=dev) if want_p else None
    ws = None
    if seqlens is not None:
        ws = _workspace(route_workspace_size(q, Hkv, t_cap, True), dev, workspace)
    elif q.dtype != torch.float32:
        ws = _workspace(route_workspace_size(q, Hkv, t_cap, False), dev, workspace)  # split summaries
    qd = _desc(q)
    _check(_lib.dash_attn_route(ctypes.byref(qd), summaries.data_ptr(), Hkv, t_cap, _ptr(seqlens), alpha, block,
                                1 if causal else 0, idx.data_ptr(), logp.data_ptr(), cnt.data_ptr(), _ptr(tau),
                                _ptr(p), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return {"idx": idx, "logp": logp, "cnt": cnt, "tau": tau, "p": p, "workspace": ws}


# ------------------------------------------------------------------ stage 2


def sparse_workspace_size(q: torch.Tensor, k: torch.Tensor, block: int, t_cap: int) -> int:
    qd, kd = _desc(q), _desc(k)
    return _lib.dash_attn_sparse_workspace_size(ctypes.byref(qd), ctypes.byref(kd), block, t_cap)


def sparse(q, k, v, idx, logp, cnt, block: int, causal: bool = True, out=None, workspace=None,
           stream=None, sigma: float = 1.0) -> torch.Tensor:
    """Stage 2 alone on caller-given routing (layout of :func:`route`); sigma: prior strength."""
    out = torch.empty_like(q) if out is None else out
    t_cap = idx.shape[-1]
    ws = _workspace(sparse_workspace_size(q, k, block, t_cap), q.device, workspace)
    qd, kd, vd, od = _desc(q), _desc(k), _desc(v), _desc(out)
    opts = _options(sigma, None)
    args = (ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), idx.data_ptr(), logp.data_ptr(), cnt.data_ptr(),
            t_cap, block, 1 if causal else 0, ctypes.byref(od), ws.data_ptr(), ws.numel())
    if opts is None:
        _check(_lib.dash_attn_sparse(*args, _stream(stream)))
    else:
        _check(_lib.dash_attn_sparse_ex(*args, opts, _stream(stream)))
    return out


def sparse_mask(q, k, v, mask: torch.Tensor, logp_dense: torch.Tensor, block: int, causal: bool = True, out=None,
                workspace=None, sigma: float = 1.0, stream=None) -> torch.Tensor:
    """Stage 2 on bit-packed masks [B, Hkv, S, n_words] (int32 bit patterns) and a dense log p_bar
    [B, Hkv, S, t_cap] (see dash_attn_sparse_mask)."""
    assert mask.is_contiguous() and mask.dtype == torch.int32 and logp_dense.is_contiguous()
    assert logp_dense.dtype == torch.float32
    out = torch.empty_like(q) if out is None else out
    t_cap, n_words = logp_dense.shape[-1], mask.shape[-1]
    ws = _workspace(sparse_workspace_size(q, k, block, t_cap), q.device, workspace)
    qd, kd, vd, od = _desc(q), _desc(k), _desc(v), _desc(out)
    _check(_lib.dash_attn_sparse_mask(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), mask.data_ptr(), n_words,
                                      logp_dense.data_ptr(), t_cap, block, 1 if causal else 0, ctypes.byref(od),
                                      ws.data_ptr(), ws.numel(), ctypes.byref(DashOptions(float(sigma), None)),
                                      _stream(stream)))
    return out


def debug_sparse_stalled(q, k, v, idx, logp, cnt, block: int, causal: bool, out, workspace, wait_cycles: int,
                         stream=None) -> None:
    """Stage 2 with its copies withheld and short waits (see dash_attn_debug_sparse_stalled): a test of
    the timeout path; the workspace status word then reads DASH_ERR_DEVICE_TIMEOUT."""
    qd, kd, vd, od = _desc(q), _desc(k), _desc(v), _desc(out)
    _check(_lib.dash_attn_debug_sparse_stalled(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), idx.data_ptr(),
                                               logp.data_ptr(), cnt.data_ptr(), idx.shape[-1], block,
                                               1 if causal else 0, ctypes.byref(od), workspace.data_ptr(),
                                               workspace.numel(), wait_cycles, _stream(stream)))


def lists_to_mask(idx: torch.Tensor, cnt: torch.Tensor, n_words: int | None = None, stream=None) -> torch.Tensor:
    """Bit-packed active-block masks [..., n_words] (int32 bit patterns) from lists idx [..., t_cap], cnt [...]."""
    t_cap = idx.shape[-1]
    n_words = -(-t_cap // 32) if n_words is None else n_words
    rows = cnt.numel()
    mask = torch.empty(tuple(cnt.shape) + (n_words,), dtype=torch.int32, device=idx.device)
    assert idx.is_contiguous() and cnt.is_contiguous() and idx.dtype == torch.int32 and cnt.dtype == torch.int32
    _check(_lib.dash_attn_lists_to_mask(idx.data_ptr(), cnt.data_ptr(), rows, t_cap, mask.data_ptr(), n_words,
                                        _stream(stream)))
    return mask


# ------------------------------------------------------------------ full forward


def fwd_workspace_size(q: torch.Tensor, k: torch.Tensor, block: int) -> int:
    qd, kd = _desc(q), _desc(k)
    n = _lib.dash_attn_fwd_workspace_size(ctypes.byref(qd), ctypes.byref(kd), block)
    if n == 0:
        raise DashError(1, "arguments rejected by dash_attn_fwd_workspace_size")
    return n


def fwd(q, k, v, w_s, alpha: float, block: int, causal: bool = True, out=None, workspace=None,
        stream=None, sigma: float = 1.0, qbar: torch.Tensor | None = None) -> torch.Tensor:
    """Full prefill forward (stages 0-2); see dash_attn_fwd (and dash_attn_fwd_ex for sigma / qbar)."""
    out = torch.empty_like(q) if out is None else out
    ws = _workspace(fwd_workspace_size(q, k, block), q.device, workspace)
    qd, kd, vd, od = _desc(q), _desc(k), _desc(v), _desc(out)
    opts = _options(sigma, qbar)
    args = (ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), w_s.data_ptr(), alpha, block, 1 if causal else 0,
            ctypes.byref(od), ws.data_ptr(), ws.numel())
    if opts is None:
        _check(_lib.dash_attn_fwd(*args, _stream(stream)))
    else:
        _check(_lib.dash_attn_fwd_ex(*args, opts, _stream(stream)))
    return out


def _view(ws: torch.Tensor, offset: int, shape, dtype) -> torch.Tensor:
    n = 1
    for e in shape:
        n *= e
    nbytes = n * torch.tensor([], dtype=dtype).element_size()
    return ws[offset:offset + nbytes].view(dtype).view(*shape)


def fwd_lists(workspace: torch.Tensor, q: torch.Tensor, k: torch.Tensor, block: int) -> dict:
    """Views into a fwd workspace of the call's summaries and routing lists (dash_attn_fwd_workspace_lists)."""
    qd, kd = _desc(q), _desc(k)
    off = [ctypes.c_size_t() for _ in range(4)]
    _check(_lib.dash_attn_fwd_workspace_lists(ctypes.byref(qd), ctypes.byref(kd), block,
                                              *[ctypes.byref(o) for o in off]))
    B, S, _, d = q.shape
    Hkv, T = k.shape[2], n_blocks(S, block)
    return {"summaries": _view(workspace, off[0].value, (B, Hkv, T, d), torch.float32),
            "idx": _view(workspace, off[1].value, (B, Hkv, S, T), torch.int32),
            "logp": _view(workspace, off[2].value, (B, Hkv, S, T), torch.float32),
            "cnt": _view(workspace, off[3].value, (B, Hkv, S), torch.int32)}


# ------------------------------------------------------------------ backward


def bwd_workspace_size(q: torch.Tensor, k: torch.Tensor, block: int) -> int:
    qd, kd = _desc(q), _desc(k)
    n = _lib.dash_attn_bwd_workspace_size(ctypes.byref(qd), ctypes.byref(kd), block)
    if n == 0:
        raise DashError(1, "arguments rejected by dash_attn_bwd_workspace_size")
    return n


def bwd(q, k, v, w_s, out, dout, alpha: float, block: int, causal: bool = True, sigma: float = 1.0,
        grads=None, workspace=None, stream=None) -> dict:
    """Gradients of sum(dout * out) (see dash_attn_bwd): dq, dk, dv fp32 and dw_s [d, d] fp32.

    grads: optional dict of preallocated fp32 dq / dk / dv / dw_s.
    """
    d = q.shape[-1]
    g = grads or {}
    dq = g.get("dq", torch.empty(q.shape, dtype=torch.float32, device=q.device))
    dk = g.get("dk", torch.empty(k.shape, dtype=torch.float32, device=q.device))
    dv = g.get("dv", torch.empty(v.shape, dtype=torch.float32, device=q.device))
    dw_s = g.get("dw_s", torch.empty((d, d), dtype=torch.float32, device=q.device))
    ws = _workspace(bwd_workspace_size(q, k, block), q.device, workspace)
    descs = [_desc(t) for t in (q, k, v, out, dout, dq, dk, dv)]
    qd, kd, vd, od, dod, dqd, dkd, dvd = descs
    opts = ctypes.byref(DashOptions(float(sigma), None))
    _check(_lib.dash_attn_bwd(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), w_s.data_ptr(), ctypes.byref(od),
                              ctypes.byref(dod), alpha, block, 1 if causal else 0, opts, ctypes.byref(dqd),
                              ctypes.byref(dkd), ctypes.byref(dvd), dw_s.data_ptr(), ws.data_ptr(), ws.numel(),
                              _stream(stream)))
    return {"dq": dq, "dk": dk, "dv": dv, "dw_s": dw_s}


class _DashAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, w_s, alpha, block, causal, sigma):
        out = fwd(q, k, v, w_s, alpha, block, causal, sigma=sigma)
        ctx.save_for_backward(q, k, v, w_s, out)
        ctx.args = (alpha, block, causal, sigma)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, w_s, out = ctx.saved_tensors
        alpha, block, causal, sigma = ctx.args
        g = bwd(q, k, v, w_s, out, dout.contiguous(), alpha, block, causal, sigma)
        return (g["dq"].to(q.dtype), g["dk"].to(k.dtype), g["dv"].to(v.dtype), g["dw_s"].to(w_s.dtype),
                None, None, None, None)


def attention(q, k, v, w_s, alpha: float, block: int, causal: bool = True, sigma: float = 1.0) -> torch.Tensor:
    """Differentiable DashAttention prefill (f16/bf16): forward by dash_attn_fwd_ex, gradients by dash_attn_bwd."""
    return _DashAttention.apply(q, k, v, w_s, alpha, block, causal, sigma)


# ------------------------------------------------------------------ decode


def decode_workspace_size(q: torch.Tensor, kcache: torch.Tensor, block: int, t_cap: int) -> int:
    qd, kd = _desc(q), _desc(kcache)
    n = _lib.dash_attn_decode_workspace_size(ctypes.byref(qd), ctypes.byref(kd), block, t_cap)
    if n == 0:
        raise DashError(1, "arguments rejected by dash_attn_decode_workspace_size")
    return n


def decode(q, kcache, vcache, seqlens, summaries, alpha: float, block: int, out=None, workspace=None,
           stream=None, sigma: float = 1.0) -> torch.Tensor:
    """One decode step for q [B, 1, H, d] (see dash_attn_decode); sigma: prior strength."""
    out = torch.empty_like(q) if out is None else out
    t_cap = summaries.shape[2]
    ws = _workspace(decode_workspace_size(q, kcache, block, t_cap), q.device, workspace)
    qd, kd, vd, od = _desc(q), _desc(kcache), _desc(vcache), _desc(out)
    opts = _options(sigma, None)
    args = (ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), seqlens.data_ptr(), summaries.data_ptr(), t_cap,
            alpha, block, ctypes.byref(od), ws.data_ptr(), ws.numel())
    if opts is None:
        _check(_lib.dash_attn_decode(*args, _stream(stream)))
    else:
        _check(_lib.dash_attn_decode_ex(*args, opts, _stream(stream)))
    return out


def decode_lists(workspace: torch.Tensor, q: torch.Tensor, kcache: torch.Tensor, block: int, t_cap: int) -> dict:
    """Views into a decode workspace of the step's routing lists (dash_attn_decode_workspace_lists)."""
    qd, kd = _desc(q), _desc(kcache)
    off = [ctypes.c_size_t() for _ in range(3)]
    _check(_lib.dash_attn_decode_workspace_lists(ctypes.byref(qd), ctypes.byref(kd), block, t_cap,
                                                 *[ctypes.byref(o) for o in off]))
    B, Hkv = q.shape[0], kcache.shape[2]
    return {"idx": _view(workspace, off[0].value, (B, Hkv, t_cap), torch.int32),
            "logp": _view(workspace, off[1].value, (B, Hkv, t_cap), torch.float32),
            "cnt": _view(workspace, off[2].value, (B, Hkv), torch.int32)}


def decode_noalloc(q, kcache, vcache, seqlens, summaries, alpha: float, block: int, out=None,
                   stream=None) -> torch.Tensor:
    """One decode step without a workspace (see dash_attn_decode_noalloc).

    For callers that may not allocate device memory while they run: the
    library keeps a fixed 16 MiB scratch array per GPU.  Only ``out`` is
    allocated here when it is not given.  Concurrent calls on one device race.
    """
    out = torch.empty_like(q) if out is None else out
    qd, kd, vd, od = _desc(q), _desc(kcache), _desc(vcache), _desc(out)
    _check(_lib.dash_attn_decode_noalloc(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), seqlens.data_ptr(),
                                         summaries.data_ptr(), summaries.shape[2], alpha, block, ctypes.byref(od),
                                         _stream(stream)))
    return out


def decode_noalloc_status(stream=None) -> int:
    """Status word of the last decode_noalloc call on the current device (synchronises)."""
    return _lib.dash_attn_decode_noalloc_status(_stream(stream))


def device_status(workspace: torch.Tensor, stream=None) -> int:
    """Status word of the last call that used ``workspace`` (synchronises)."""
    return _lib.dash_attn_get_device_status(workspace.data_ptr(), _stream(stream))



# ------------------------------------------------------------------ context-parallel decode


def cp_scores(q, summaries, block_lo: int, block_hi: int, seqlens, lmax: int, alpha: float, block: int,
              scores: torch.Tensor, stream=None) -> torch.Tensor:
    """This rank's routing logits into ``scores`` [B, Hkv, G, t_cap] (see dash_attn_cp_scores)."""
    B, Hkv, summ_cap, d = summaries.shape
    qd = _desc(q)
    _check(_lib.dash_attn_cp_scores(ctypes.byref(qd), Hkv, summaries.data_ptr(), summ_cap, block_lo, block_hi,
                                    seqlens.data_ptr(), lmax, alpha, block, scores.data_ptr(), scores.shape[3],
                                    _stream(stream)))
    return scores


def cp_lists(q, kv_heads: int, scores, seqlens, lmax: int, alpha: float, block: int, stream=None) -> dict:
    """alpha-entmax, GQA mean and ascending lists from whole score vectors (see dash_attn_cp_lists)."""
    B, Hkv, G, t_cap = scores.shape
    dev = q.device
    idx = torch.full((B, Hkv, t_cap), -1, dtype=torch.int32, device=dev)
    logp = torch.zeros((B, Hkv, t_cap), dtype=torch.float32, device=dev)
    cnt = torch.zeros((B, Hkv), dtype=torch.int32, device=dev)
    qd = _desc(q)
    _check(_lib.dash_attn_cp_lists(ctypes.byref(qd), kv_heads, scores.data_ptr(), seqlens.data_ptr(), lmax, alpha,
                                   block, idx.data_ptr(), logp.data_ptr(), cnt.data_ptr(), t_cap, _stream(stream)))
    return {"idx": idx, "logp": logp, "cnt": cnt}


def cp_attend(q, kshard, vshard, tok_lo: int, seqlens, lmax: int, lists: dict, block: int, sigma: float = 1.0,
              part=None, stream=None) -> torch.Tensor:
    """Partials [B, H, d + 2] of this rank's tokens (see dash_attn_cp_attend)."""
    B, _, H, d = q.shape
    part = torch.empty((B, H, d + 2), dtype=torch.float32, device=q.device) if part is None else part
    qd, kd, vd = _desc(q), _desc(kshard), _desc(vshard)
    t_cap = lists["idx"].shape[-1]
    _check(_lib.dash_attn_cp_attend(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), tok_lo, seqlens.data_ptr(),
                                    lmax, lists["idx"].data_ptr(), lists["logp"].data_ptr(), lists["cnt"].data_ptr(),
                                    t_cap, block, _options(sigma, None), part.data_ptr(), _stream(stream)))
    return part


def cp_attend_workspace_size(B: int, H: int, Hkv: int, d: int, block: int, t_cap: int) -> int:
    """Bytes of workspace dash_attn_cp_attend_ex needs."""
    return int(_lib.dash_attn_cp_attend_workspace_size(B, H, Hkv, d, block, t_cap))


def cp_attend_ex(q, kshard, vshard, tok_lo: int, seqlens, lmax: int, lists: dict, block: int, sigma: float = 1.0,
                 part=None, workspace=None, stream=None) -> torch.Tensor:
    """Partials [B, H, d + 2] of this rank's tokens on the split-KV path (see dash_attn_cp_attend_ex)."""
    B, _, H, d = q.shape
    Hkv = kshard.shape[2]
    t_cap = lists["idx"].shape[-1]
    part = torch.empty((B, H, d + 2), dtype=torch.float32, device=q.device) if part is None else part
    n_ws = cp_attend_workspace_size(B, H, Hkv, d, block, t_cap)
    if workspace is None:
        workspace = torch.empty(n_ws, dtype=torch.uint8, device=q.device)
    qd, kd, vd = _desc(q), _desc(kshard), _desc(vshard)
    _check(_lib.dash_attn_cp_attend_ex(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), tok_lo,
                                       seqlens.data_ptr(), lmax, lists["idx"].data_ptr(), lists["logp"].data_ptr(),
                                       lists["cnt"].data_ptr(), t_cap, block, _options(sigma, None), part.data_ptr(),
                                       workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                       _stream(stream)))
    return part


def cp_merge(parts: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
    """Merge partials [R, B, H, d + 2] into out [B, 1, H, d] (see dash_attn_cp_merge)."""
    assert parts.is_contiguous() and parts.dtype == torch.float32
    od = _desc(out)
    _check(_lib.dash_attn_cp_merge(parts.data_ptr(), parts.shape[0], ctypes.byref(od), _stream(stream)))
    return out


# ------------------------------------------------------------------ paged KV cache


def summarize_paged(k_pages, block_table, seqlens, w_s, block: int, summaries=None, t_cap: int | None = None,
                    first_block: int = 0, qbar=None, stream=None) -> torch.Tensor:
    """Summaries [B, Hkv, t_cap, d] from a paged cache (see dash_attn_summarize_paged)."""
    n_pages, page, Hkv, d = k_pages.shape
    B, max_blocks = block_table.shape
    t_cap = max_blocks if t_cap is None else t_cap
    if summaries is None:
        summaries = torch.zeros((B, Hkv, t_cap, d), dtype=torch.float32, device=k_pages.device)
    kd = _desc(k_pages)
    _check(_lib.dash_attn_summarize_paged(ctypes.byref(kd), block_table.data_ptr(), max_blocks, B, seqlens.data_ptr(),
                                          w_s.data_ptr(), _ptr(qbar), block, summaries.data_ptr(), summaries.shape[2],
                                          first_block, _stream(stream)))
    return summaries


def decode_paged(q, k_pages, v_pages, block_table, seqlens, summaries, alpha: float, block: int, out=None,
                 workspace=None, sigma: float = 1.0, stream=None) -> torch.Tensor:
    """One decode step against a paged cache (see dash_attn_decode_paged)."""
    out = torch.empty_like(q) if out is None else out
    B, max_blocks = block_table.shape
    t_cap = summaries.shape[2]
    qd, kd, vd, od = _desc(q), _desc(k_pages), _desc(v_pages), _desc(out)
    # the workspace is that of a dense cache of the same B, Hkv, d (only the shape enters the size query)
    dk = DashTensor(k_pages.data_ptr(), kd.dtype, 0, B, max_blocks * block, kd.h, kd.d,
                    kd.h * kd.d * max_blocks * block, kd.h * kd.d, kd.d)
    nbytes = _lib.dash_attn_decode_workspace_size(ctypes.byref(qd), ctypes.byref(dk), block, t_cap)
    ws = _workspace(nbytes, q.device, workspace)
    _check(_lib.dash_attn_decode_paged(ctypes.byref(qd), ctypes.byref(kd), ctypes.byref(vd), block_table.data_ptr(),
                                       max_blocks, seqlens.data_ptr(), summaries.data_ptr(), t_cap, alpha, block,
                                       ctypes.byref(od), ws.data_ptr(), ws.numel(), _options(sigma, None),
                                       _stream(stream)))
    return out
