"""B200-native (sm_100a) forward pass of token-level dynamic local-global attention.

Method (page titles and sections): "LoGo: Token-Level Dynamic Local-Global
Attention", Abstract; "Learning When to Attend", "The Architecture of
Conditional Attention".  Every query token gets causal sliding-window
attention over the previous W keys; a per-sequence budget picks the
ceil(ratio * L) tokens with the largest gate logits (ties to the lower
position); those tokens also get exact full-causal attention, merged as
``local + sigmoid(g) * global``.

This module is a thin ctypes binding over the C ABI in ``include/logo.h``
(``liblogo.so``): it only marshals torch CUDA tensors (device memory, the
current stream) into the C calls.  Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and a missing
library raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# LOGO_LIBRARY may point at another build of the same library (e.g. a tuning variant).
LIB_PATH = os.environ.get("LOGO_LIBRARY") or os.path.join(_HERE, "liblogo.so")
CSRC = os.path.join(_HERE, "csrc")

LOGO_OK = 0
_STATUS = {0: "LOGO_OK", 1: "LOGO_ERR_INVALID_ARG", 2: "LOGO_ERR_UNSUPPORTED", 3: "LOGO_ERR_WORKSPACE",
           4: "LOGO_ERR_CUDA", 5: "LOGO_ERR_DEVICE_TIMEOUT", 6: "LOGO_ERR_CAPACITY",
           7: "LOGO_ERR_BOUNDS"}

EXPORTED = ("logo_num_selected", "logo_workspace_size", "logo_workspace_init", "logo_select",
            "logo_local_attn", "logo_global_attn_sparse", "logo_forward", "logo_check",
            "logo_selftest_timeout", "logo_status_string", "logo_last_error",
            "logo_global_attn_sparse_noalloc", "logo_select_threshold", "logo_threshold_update",
            "logo_decode_workspace_size", "logo_decode", "logo_forward_train", "logo_backward_workspace_size",
            "logo_backward", "logo_forward_host_buffer_size", "logo_forward_host", "logo_build_flags")


class LogoError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{_STATUS.get(status, status)}: {message}")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("L", ctypes.c_int),
                ("d", ctypes.c_int), ("cu_seqlens", ctypes.c_void_p), ("nseq", ctypes.c_int),
                ("max_seqlen", ctypes.c_int)]


_lock = threading.Lock()
_lib = None


def load_library(path: str | None = None):
    """Load liblogo.so (built by ``make -C token_level_dynamic_seq_b200/csrc``); raise if absent."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"CUDA library {p} is missing: build it with `make -C {CSRC}` "
                               "(or __graft_entry__.build()); there is no fallback")
        lib = ctypes.CDLL(p)
        vp, i32, i64, dbl, flt, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double,
                                      ctypes.c_float, ctypes.c_size_t)
        sp = ctypes.POINTER(Shape)
        sig = {
            "logo_num_selected": ([dbl, i64], i64),
            "logo_workspace_size": ([sp, dbl], sz),
            "logo_workspace_init": ([vp, sz, vp], i32),
            "logo_select": ([vp, sp, dbl, vp, vp, vp, sz, vp], i32),
            "logo_local_attn": ([vp, vp, vp, sp, i32, flt, vp, vp, sz, vp], i32),
            "logo_global_attn_sparse": ([vp, vp, vp, vp, vp, vp, sp, i32, flt, i32, vp, vp, sz, vp], i32),
            "logo_forward": ([vp, vp, vp, vp, sp, i32, dbl, flt, vp, vp, vp, vp, sz, vp], i32),
            "logo_check": ([vp, vp], i32),
            "logo_selftest_timeout": ([vp, sz, ctypes.c_uint, vp], i32),
            "logo_status_string": ([i32], ctypes.c_char_p),
            "logo_last_error": ([], ctypes.c_char_p),
            "logo_build_flags": ([], ctypes.c_uint),
            "logo_global_attn_sparse_noalloc": ([vp, vp, vp, vp, vp, vp, sp, i32, flt, i32, vp, vp], i32),
            "logo_select_threshold": ([vp, sp, vp, i32, vp, vp, vp, sz, vp], i32),
            "logo_threshold_update": ([vp, sp, dbl, flt, vp, vp, vp, sz, vp], i32),
            "logo_decode_workspace_size": ([sp], sz),
            "logo_decode": ([vp, vp, vp, vp, vp, vp, sp, i32, flt, vp, vp, vp, sz, vp], i32),
            "logo_forward_train": ([vp, vp, vp, vp, sp, i32, dbl, flt, vp, vp, vp, i32, vp, vp, vp, vp, vp, sz, vp],
                                   i32),
            "logo_backward_workspace_size": ([sp, i32], sz),
            "logo_forward_host_buffer_size": ([sp, dbl], sz),
            "logo_forward_host": ([vp, vp, vp, vp, sp, i32, dbl, flt, vp, vp, vp, vp, sz, vp], i32),
            "logo_backward": ([vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, sp, i32, flt, vp, vp, vp,
                               vp, vp, sz, vp], i32),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        if path is None:
            _lib = lib
        return lib


def _raise(status: int):
    if status != LOGO_OK:
        msg = load_library().logo_last_error().decode()
        raise LogoError(status, msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _bits(x: torch.Tensor) -> torch.Tensor:
    if x.dtype != torch.bfloat16:
        raise TypeError(f"expected bf16, got {x.dtype}")
    if not x.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not x.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return x


def make_shape(q: torch.Tensor, k: torch.Tensor, cu_seqlens=None, max_seqlen=None) -> Shape:
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if cu_seqlens is None:
        return Shape(B, Hq, Hkv, L, d, None, B, L)
    nseq = cu_seqlens.numel() - 1
    if max_seqlen is None:
        raise ValueError("max_seqlen is required with cu_seqlens (the library never reads device data on the host)")
    return Shape(B, Hq, Hkv, L, d, cu_seqlens.data_ptr(), nseq, int(max_seqlen))


def num_selected(ratio: float, length: int) -> int:
    return int(load_library().logo_num_selected(float(ratio), int(length)))


def workspace(shape: Shape, ratio: float, device, stream=None) -> torch.Tensor:
    lib = load_library()
    n = lib.logo_workspace_size(ctypes.byref(shape), float(ratio))
    if n == 0:
        _raise(1)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _raise(lib.logo_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))
    return ws


def check(ws: torch.Tensor, stream=None):
    """Synchronise the stream and raise if a kernel recorded an error."""
    _raise(load_library().logo_check(_ptr(ws), _stream(stream)))


def selection_capacity(shape: Shape, ratio: float, seqlens=None) -> int:
    if shape.cu_seqlens is None or not shape.cu_seqlens:
        return shape.B * num_selected(ratio, shape.L)
    if seqlens is None:
        # upper bound without reading device data: every sequence at max_seqlen, capped by T
        return min(shape.L, shape.nseq * num_selected(ratio, shape.max_seqlen))
    return sum(num_selected(ratio, n) for n in seqlens)


def select(gate: torch.Tensor, shape: Shape, ratio: float, ws: torch.Tensor, sel_idx=None, cu_sel=None,
           stream=None):
    lib = load_library()
    nseq = shape.nseq if shape.cu_seqlens else shape.B
    if sel_idx is None:
        sel_idx = torch.empty(max(1, selection_capacity(shape, ratio)), dtype=torch.int32, device=gate.device)
    if cu_sel is None:
        cu_sel = torch.empty(nseq + 1, dtype=torch.int32, device=gate.device)
    _raise(lib.logo_select(_ptr(gate), ctypes.byref(shape), float(ratio), _ptr(sel_idx), _ptr(cu_sel), _ptr(ws),
                           ws.numel(), _stream(stream)))
    return sel_idx, cu_sel


def select_threshold(gate: torch.Tensor, shape: Shape, tau: torch.Tensor, max_selected: int, ws: torch.Tensor,
                     sel_idx=None, cu_sel=None, stream=None):
    """Threshold form of the budget rule: per sequence, ascending positions with logit > tau."""
    nseq = shape.nseq if shape.cu_seqlens else shape.B
    if sel_idx is None:
        sel_idx = torch.empty(max(1, nseq * int(max_selected)), dtype=torch.int32, device=gate.device)
    if cu_sel is None:
        cu_sel = torch.empty(nseq + 1, dtype=torch.int32, device=gate.device)
    _raise(load_library().logo_select_threshold(_ptr(gate), ctypes.byref(shape), _ptr(tau), int(max_selected),
                                                _ptr(sel_idx), _ptr(cu_sel), _ptr(ws), ws.numel(), _stream(stream)))
    return sel_idx, cu_sel


def threshold_update(gate: torch.Tensor, shape: Shape, ratio: float, beta: float, tau: torch.Tensor,
                     ws: torch.Tensor, target=None, stream=None):
    """One controller step: moves the device threshold `tau` toward the batch target; returns target."""
    if target is None:
        target = torch.empty(1, dtype=torch.float32, device=gate.device)
    _raise(load_library().logo_threshold_update(_ptr(gate), ctypes.byref(shape), float(ratio), float(beta), _ptr(tau),
                                                _ptr(target), _ptr(ws), ws.numel(), _stream(stream)))
    return target


def decode_workspace(shape: Shape, device) -> torch.Tensor:
    n = load_library().logo_decode_workspace_size(ctypes.byref(shape))
    if n == 0:
        _raise(1)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _raise(load_library().logo_workspace_init(_ptr(ws), ws.numel(), _stream()))
    return ws


def decode(q, k_cache, v_cache, cache_len, gate, tau, window: int, ws: torch.Tensor | None = None,
           scale: float = 0.0, out=None, selected=None, stream=None):
    """Decode step: q [B, Hq, d], caches [B, Hkv, Lmax, d] (bf16), cache_len int32 [B], gate fp32 [B],
    tau fp32 [1] (all CUDA).  Returns (out [B, Hq, d], selected int32 [B])."""
    q, k_cache, v_cache = _bits(q), _bits(k_cache), _bits(v_cache)
    B, Hq, d = q.shape
    shape = Shape(B, Hq, k_cache.shape[1], k_cache.shape[2], d, None, B, k_cache.shape[2])
    if ws is None:
        ws = decode_workspace(shape, q.device)
    if out is None:
        out = torch.empty_like(q)
    if selected is None:
        selected = torch.empty(B, dtype=torch.int32, device=q.device)
    _raise(load_library().logo_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_len), _ptr(gate), _ptr(tau),
                                      ctypes.byref(shape), int(window), float(scale), _ptr(out), _ptr(selected),
                                      _ptr(ws), ws.numel(), _stream(stream)))
    return out, selected


def local_attn(q, k, v, window: int, ws: torch.Tensor, scale: float = 0.0, cu_seqlens=None, max_seqlen=None,
               out=None, stream=None):
    q, k, v = _bits(q), _bits(k), _bits(v)
    shape = make_shape(q, k, cu_seqlens, max_seqlen)
    if out is None:
        out = torch.empty_like(q)
    _raise(load_library().logo_local_attn(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(shape), int(window),
                                          float(scale), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def global_attn_sparse(q, k, v, gate, sel_idx, cu_sel, max_selected: int, out, ws: torch.Tensor,
                       scale: float = 0.0, merge: bool = True, cu_seqlens=None, max_seqlen=None, stream=None):
    q, k, v = _bits(q), _bits(k), _bits(v)
    shape = make_shape(q, k, cu_seqlens, max_seqlen)
    _raise(load_library().logo_global_attn_sparse(
        _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(sel_idx), _ptr(cu_sel), ctypes.byref(shape),
        int(max_selected), float(scale), 1 if merge else 0, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def global_attn_sparse_noalloc(q, k, v, gate, sel_idx, cu_sel, max_selected: int, out, scale: float = 0.0,
                               merge: bool = True, cu_seqlens=None, max_seqlen=None, stream=None):
    """global_attn_sparse without a caller workspace: the library's fixed scratch array is used."""
    q, k, v = _bits(q), _bits(k), _bits(v)
    shape = make_shape(q, k, cu_seqlens, max_seqlen)
    _raise(load_library().logo_global_attn_sparse_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(sel_idx), _ptr(cu_sel), ctypes.byref(shape),
        int(max_selected), float(scale), 1 if merge else 0, _ptr(out), _stream(stream)))
    return out


def forward(q, k, v, gate, window: int, ratio: float, ws: torch.Tensor | None = None, scale: float = 0.0,
            cu_seqlens=None, max_seqlen=None, out=None, sel_idx=None, cu_sel=None, stream=None):
    """The whole forward pass; returns (out, sel_idx, cu_sel)."""
    q, k, v = _bits(q), _bits(k), _bits(v)
    shape = make_shape(q, k, cu_seqlens, max_seqlen)
    if ws is None:
        ws = workspace(shape, ratio, q.device, stream)
    if out is None:
        out = torch.empty_like(q)
    nseq = shape.nseq if cu_seqlens is not None else shape.B
    if sel_idx is None:
        sel_idx = torch.empty(max(1, selection_capacity(shape, ratio)), dtype=torch.int32, device=q.device)
    if cu_sel is None:
        cu_sel = torch.empty(nseq + 1, dtype=torch.int32, device=q.device)
    _raise(load_library().logo_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(gate), ctypes.byref(shape), int(window),
                                       float(ratio), float(scale), _ptr(out), _ptr(sel_idx), _ptr(cu_sel),
                                       _ptr(ws), ws.numel(), _stream(stream)))
    return out, sel_idx, cu_sel


def _host_bits(x: torch.Tensor) -> torch.Tensor:
    if x.dtype != torch.bfloat16:
        raise TypeError(f"expected bf16, got {x.dtype}")
    if x.is_cuda:
        raise ValueError("expected a host tensor")
    if not x.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return x


def host_buffer(shape: Shape, ratio: float, device, stream=None) -> torch.Tensor:
    """Device arena of :func:`forward_host` (its first bytes are the workspace, initialised here)."""
    lib = load_library()
    n = lib.logo_forward_host_buffer_size(ctypes.byref(shape), float(ratio))
    if n == 0:
        _raise(1)
    buf = torch.empty(n, dtype=torch.uint8, device=device)
    _raise(lib.logo_workspace_init(_ptr(buf), buf.numel(), _stream(stream)))
    return buf


def forward_host(q, k, v, gate, window: int, ratio: float, buf: torch.Tensor | None = None, device=None,
                 scale: float = 0.0, cu_seqlens=None, max_seqlen=None, out=None, sel_idx=None, cu_sel=None,
                 stream=None):
    """The whole forward pass on HOST tensors (page-locked for asynchronous copies).

    The library copies the inputs in and the output out, one key/value-head group
    at a time, overlapping the copies with the kernels.  ``cu_seqlens`` (packed
    layout) is a host int32 tensor here.  Returns host tensors (out, sel_idx,
    cu_sel) once the work is queued on ``stream``: synchronise the stream before
    reading them.  ``buf`` is the device arena (:func:`host_buffer`)."""
    q, k, v = _host_bits(q), _host_bits(k), _host_bits(v)
    if gate.is_cuda or gate.dtype != torch.float32:
        raise ValueError("gate must be a host fp32 tensor")
    shape = make_shape(q, k, cu_seqlens, max_seqlen)
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    if buf is None:
        buf = host_buffer(shape, ratio, device, stream)
    nseq = shape.nseq if cu_seqlens is not None else shape.B
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if sel_idx is None:
        sel_idx = torch.empty(max(1, nseq * num_selected(ratio, shape.max_seqlen)), dtype=torch.int32,
                              pin_memory=True)
    if cu_sel is None:
        cu_sel = torch.empty(nseq + 1, dtype=torch.int32, pin_memory=True)
    _raise(load_library().logo_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(gate), ctypes.byref(shape),
                                            int(window), float(ratio), float(scale), _ptr(out), _ptr(sel_idx),
                                            _ptr(cu_sel), _ptr(buf), buf.numel(), _stream(stream)))
    return out, sel_idx, cu_sel


def forward_train(q, k, v, gate, window: int, ratio: float, ws: torch.Tensor | None = None, scale: float = 0.0,
                  cu_seqlens=None, max_seqlen=None, stream=None, reuse=None):
    """Forward pass that also saves what :func:`backward` needs.

    Returns (out, ctx): ``ctx`` holds the selection (sel_idx, cu_sel, its
    capacity and the largest per-sequence count) and the saved statistics
    (lse [B*Hq*L], lse_sel [Hq, cap], glob and loc_sel [Hq, cap, d]: the two
    branches of the selected rows).  ``reuse`` = (out, ctx) of an earlier call
    with the same shapes: its buffers are written again instead of new ones."""
    q, k, v = _bits(q), _bits(k), _bits(v)
    shape = make_shape(q, k, cu_seqlens, max_seqlen)
    if ws is None:
        ws = workspace(shape, ratio, q.device, stream)
    dev = q.device
    nseq = shape.nseq if cu_seqlens is not None else shape.B
    cap = max(1, selection_capacity(shape, ratio))
    max_sel = num_selected(ratio, shape.max_seqlen)
    if reuse is not None:
        out, old = reuse
        sel_idx, cu_sel, lse, lse_sel, glob, loc_sel = (old[n] for n in ("sel_idx", "cu_sel", "lse", "lse_sel",
                                                                           "glob", "loc_sel"))
        cap = old["cap"]
    else:
        out = torch.empty_like(q)
        sel_idx = torch.empty(cap, dtype=torch.int32, device=dev)
        cu_sel = torch.empty(nseq + 1, dtype=torch.int32, device=dev)
        lse = torch.empty(q.shape[0] * q.shape[1] * q.shape[2], dtype=torch.float32, device=dev)
        lse_sel = torch.empty(q.shape[1], cap, dtype=torch.float32, device=dev)
        glob = torch.empty(q.shape[1], cap, q.shape[3], dtype=torch.bfloat16, device=dev)
        loc_sel = torch.empty_like(glob)
    _raise(load_library().logo_forward_train(_ptr(q), _ptr(k), _ptr(v), _ptr(gate), ctypes.byref(shape), int(window),
                                             float(ratio), float(scale), _ptr(out), _ptr(sel_idx), _ptr(cu_sel), cap,
                                             _ptr(lse), _ptr(lse_sel), _ptr(glob), _ptr(loc_sel), _ptr(ws),
                                             ws.numel(),
                                             _stream(stream)))
    ctx = {"sel_idx": sel_idx, "cu_sel": cu_sel, "cap": cap, "max_selected": max_sel, "lse": lse,
           "lse_sel": lse_sel, "glob": glob, "loc_sel": loc_sel, "window": int(window), "scale": float(scale),
           "shape": shape, "ws": ws}
    return out, ctx


def backward_workspace(shape: Shape, cap: int, device) -> torch.Tensor:
    n = load_library().logo_backward_workspace_size(ctypes.byref(shape), int(cap))
    if n == 0:
        _raise(1)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def backward(q, k, v, gate, out, dout, ctx, ws: torch.Tensor | None = None, stream=None, grads=None):
    """Gradients (dq, dk, dv, dgate) of a loss with dL/d(out) = dout, for a forward
    pass made by :func:`forward_train` (its ``ctx``).  ``grads`` may hold
    preallocated outputs (dq, dk, dv, dgate)."""
    q, k, v, out, dout = _bits(q), _bits(k), _bits(v), _bits(out), _bits(dout)
    shape = ctx["shape"]
    if ws is None:
        ws = backward_workspace(shape, ctx["cap"], q.device)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 torch.empty(gate.shape, dtype=torch.float32, device=q.device))
    dq, dk, dv, dg = grads
    _raise(load_library().logo_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(out), _ptr(dout),
                                        _ptr(ctx["sel_idx"]), _ptr(ctx["cu_sel"]), ctx["cap"], ctx["max_selected"],
                                        _ptr(ctx["lse"]), _ptr(ctx["lse_sel"]), _ptr(ctx["glob"]),
                                        _ptr(ctx["loc_sel"]), ctypes.byref(shape), ctx["window"], ctx["scale"],
                                        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(ws), ws.numel(),
                                        _stream(stream)))
    return dq, dk, dv, dg, ws


def selftest_timeout(ws: torch.Tensor, limit_us: int = 1000, stream=None):
    _raise(load_library().logo_selftest_timeout(_ptr(ws), ws.numel(), int(limit_us), _stream(stream)))


def useful_flops(d: int, Hq: int, seqlens, window: int, sel_positions) -> tuple[int, int]:
    """Useful FLOPs of one forward pass: (local, global).

    local = 4 d Hq sum_s sum_{i < L_s} min(i + 1, W); global = 4 d Hq sum_{i selected} (i + 1).
    """
    lp = 0
    for n in seqlens:
        n = int(n)
        w = min(int(window), n)
        # sum_{i<n} min(i+1, w) = w(w+1)/2 + (n - w) w
        lp += w * (w + 1) // 2 + (n - w) * w
    sp = int(sum(int(p) + 1 for p in sel_positions))
    return 4 * d * Hq * lp, 4 * d * Hq * sp
