"""fp64 CPU oracle for token-level dynamic local-global attention (LoGo / L2A).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import this package.  The library's product
path never does: it has no CPU fallback.

The arithmetic lives in ``logo_oracle.c`` (plain loops in double precision);
this module only marshals torch CPU tensors into it.  Each function cites the
passage of the pages it follows in the C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liblogo_oracle.so")
_SRC = os.path.join(_HERE, "logo_oracle.c")
_lock = threading.Lock()
_lib = None

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double


def build() -> str:
    """Compile the oracle with the Makefile beside it (gcc, OpenMP if available)."""
    subprocess.run(["make", "-s", "-C", _HERE], check=True)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if (not os.path.exists(_SO)) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
            build()
        lib = ctypes.CDLL(_SO)
        lib.oracle_num_selected.argtypes = [_dbl, _i64]
        lib.oracle_num_selected.restype = _i64
        lib.oracle_select.argtypes = [_p, _i64, _dbl, _p]
        lib.oracle_select.restype = _i64
        lib.oracle_forward.argtypes = [_p, _p, _p, _p, _p, _int, _int, _int, _i64, _int, _i64,
                                       _dbl, _dbl, _p, _p, _p, _p, _p]
        lib.oracle_forward.restype = _i64
        lib.oracle_rows.argtypes = [_p, _p, _p, _p, _p, _int, _int, _int, _i64, _int, _i64, _dbl,
                                    _i64, _p, _p, _p, _p, _p, _p, _p]
        lib.oracle_rows.restype = None
        lib.oracle_threshold_select.argtypes = [_p, _i64, ctypes.c_float, _p]
        lib.oracle_threshold_select.restype = _i64
        lib.oracle_threshold_target.argtypes = [_p, _i64, _dbl]
        lib.oracle_threshold_target.restype = ctypes.c_float
        lib.oracle_threshold_update.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_float]
        lib.oracle_threshold_update.restype = ctypes.c_float
        lib.oracle_decode.argtypes = [_p, _p, _p, _p, _p, ctypes.c_float, _int, _int, _int, _i64, _int, _i64,
                                      _dbl, _p, _p, _p, _p]
        lib.oracle_decode.restype = _i64
        lib.oracle_backward.argtypes = [_p, _p, _p, _p, _p, _p, _int, _int, _int, _i64, _int, _i64, _dbl, _dbl,
                                        _p, _p, _p, _p]
        lib.oracle_backward.restype = _i64
        lib.oracle_backward_rows.argtypes = [_p, _p, _p, _p, _p, _p, _p, _int, _int, _int, _i64, _int, _i64, _dbl,
                                             _i64, _p, _p, _p, _p, _p, _i64, _p, _p, _p, _p, _p]
        lib.oracle_backward_rows.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = _int
        lib.oracle_set_num_threads.argtypes = [_int]
        lib.oracle_set_num_threads.restype = None
        _lib = lib
        return lib


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _bits(x: torch.Tensor) -> torch.Tensor:
    assert x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return x.contiguous().view(torch.int16)


def num_selected(ratio: float, length: int) -> int:
    """k = ceil(ratio * length) with fp noise snapped (see logo_oracle.c)."""
    return int(_load().oracle_num_selected(float(ratio), int(length)))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Thread count of the following oracle calls (n >= 1)."""
    _load().oracle_set_num_threads(int(n))


def select(g: torch.Tensor, ratio: float) -> torch.Tensor:
    """Selected positions (ascending) of one sequence's fp32 gate logits."""
    g = g.detach().to(torch.float32).contiguous()
    k = num_selected(ratio, g.numel())
    out = torch.empty(max(k, 1), dtype=torch.int32)
    got = _load().oracle_select(_ptr(g), g.numel(), float(ratio), _ptr(out))
    assert got == k
    return out[:k].clone()


def _geometry(q, k, cu_seqlens):
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if cu_seqlens is not None:
        assert B == 1
        nseq = cu_seqlens.numel() - 1
    else:
        nseq = B
    return B, Hq, Hkv, L, d, nseq


def forward(q, k, v, g, window: int, ratio: float, scale: float = 0.0, cu_seqlens=None,
            want_branches: bool = False):
    """Whole forward pass in fp64.

    q: bf16 [B, Hq, L, d]; k, v: bf16 [B, Hkv, L, d]; g: fp32 [B, L].
    Varlen: B == 1, L == T and ``cu_seqlens`` int32 [nseq + 1].
    Returns a dict with ``out`` (fp64 [B, Hq, L, d]), ``sel_idx`` (int32, the
    sequences' ascending lists back to back), ``cu_sel`` (int32 [nseq + 1])
    and, if ``want_branches``, ``local`` and ``global`` (global is 0 on rows
    that are not selected).
    """
    B, Hq, Hkv, L, d, nseq = _geometry(q, k, cu_seqlens)
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    g32 = g.detach().to(torch.float32).contiguous()
    cu = None if cu_seqlens is None else cu_seqlens.to(torch.int32).contiguous()
    lens = [L] * B if cu is None else (cu[1:] - cu[:-1]).tolist()
    cap = max(1, sum(num_selected(ratio, n) for n in lens))
    out = torch.empty(B, Hq, L, d, dtype=torch.float64)
    loc = torch.empty_like(out) if want_branches else None
    glo = torch.empty_like(out) if want_branches else None
    sel = torch.empty(cap, dtype=torch.int32)
    cu_sel = torch.empty(nseq + 1, dtype=torch.int32)
    total = _load().oracle_forward(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(g32), _ptr(cu), nseq, Hq, Hkv,
                                   L, d, int(window), float(ratio), float(scale), _ptr(out),
                                   _ptr(loc), _ptr(glo), _ptr(sel), _ptr(cu_sel))
    res = {"out": out, "sel_idx": sel[:total].clone(), "cu_sel": cu_sel}
    if want_branches:
        res["local"] = loc
        res["global"] = glo
    return res


def rows(q, k, v, g, window: int, seq, head, pos, selected, scale: float = 0.0, cu_seqlens=None):
    """fp64 outputs of a sample of rows: (local, global, merged), each [n, d].

    ``seq``, ``head``, ``pos`` (relative to the sequence start) and
    ``selected`` (0/1, from :func:`select`) are 1-D sequences of length n.
    """
    B, Hq, Hkv, L, d, nseq = _geometry(q, k, cu_seqlens)
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    g32 = g.detach().to(torch.float32).contiguous()
    cu = None if cu_seqlens is None else cu_seqlens.to(torch.int32).contiguous()
    seq_t = torch.as_tensor(seq, dtype=torch.int32).contiguous()
    head_t = torch.as_tensor(head, dtype=torch.int32).contiguous()
    pos_t = torch.as_tensor(pos, dtype=torch.int64).contiguous()
    sel_t = torch.as_tensor(selected, dtype=torch.uint8).contiguous()
    n = seq_t.numel()
    loc = torch.empty(n, d, dtype=torch.float64)
    glo = torch.empty(n, d, dtype=torch.float64)
    out = torch.empty(n, d, dtype=torch.float64)
    _load().oracle_rows(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(g32), _ptr(cu), nseq, Hq, Hkv, L, d,
                        int(window), float(scale), n, _ptr(seq_t), _ptr(head_t), _ptr(pos_t),
                        _ptr(sel_t), _ptr(loc), _ptr(glo), _ptr(out))
    return loc, glo, out


def threshold_select(g: torch.Tensor, tau: float) -> torch.Tensor:
    """Ascending positions of one sequence whose fp32 logit is > tau (threshold form)."""
    g = g.detach().to(torch.float32).contiguous()
    out = torch.empty(max(1, g.numel()), dtype=torch.int32)
    n = _load().oracle_threshold_select(_ptr(g), g.numel(), float(tau), _ptr(out))
    return out[:n].clone()


def threshold_target(g: torch.Tensor, ratio: float) -> float:
    """Target threshold: the (k+1)-th largest logit of the whole batch, k = ceil(ratio * n)."""
    g = g.detach().to(torch.float32).contiguous().flatten()
    return float(_load().oracle_threshold_target(_ptr(g), g.numel(), float(ratio)))


def threshold_update(tau: float, q: float, beta: float) -> float:
    """One controller step tau + beta * (q - tau) in fp32 (q when either is not finite)."""
    return float(_load().oracle_threshold_update(float(tau), float(q), float(beta)))


def decode(q, k_cache, v_cache, cache_len, g, tau: float, window: int, scale: float = 0.0):
    """Decode step in fp64: q bf16 [B, Hq, d], caches bf16 [B, Hkv, Lmax, d], cache_len int32 [B]
    (the new token at position cache_len - 1), g fp32 [B].  Returns out, local, global ([B, Hq, d]
    fp64) and the 0/1 selection [B]."""
    B, Hq, d = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    cl = torch.as_tensor(cache_len, dtype=torch.int32).contiguous()
    g32 = torch.as_tensor(g, dtype=torch.float32).contiguous()
    out = torch.empty(B, Hq, d, dtype=torch.float64)
    loc = torch.empty_like(out)
    glo = torch.empty_like(out)
    sel = torch.empty(B, dtype=torch.int32)
    _load().oracle_decode(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(cl), _ptr(g32), float(tau), B, Hq, Hkv, Lmax, d,
                          int(window), float(scale), _ptr(out), _ptr(loc), _ptr(glo), _ptr(sel))
    return out, loc, glo, sel


def backward(q, k, v, g, dout, window: int, ratio: float, scale: float = 0.0, cu_seqlens=None):
    """Whole backward pass in fp64 (chain rule through :func:`forward`).

    ``dout`` is bf16 with the shape of the output.  Returns a dict with
    ``dq`` [B, Hq, L, d], ``dk``, ``dv`` [B, Hkv, L, d] and ``dg`` [B, L]
    (fp64), and the number of selected tokens ``n_sel``.
    """
    B, Hq, Hkv, L, d, nseq = _geometry(q, k, cu_seqlens)
    qb, kb, vb, eb = _bits(q), _bits(k), _bits(v), _bits(dout)
    g32 = g.detach().to(torch.float32).contiguous()
    cu = None if cu_seqlens is None else cu_seqlens.to(torch.int32).contiguous()
    dq = torch.empty(B, Hq, L, d, dtype=torch.float64)
    dk = torch.empty(B, Hkv, L, d, dtype=torch.float64)
    dv = torch.empty_like(dk)
    dg = torch.empty(B, L, dtype=torch.float64)
    n = _load().oracle_backward(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(g32), _ptr(eb), _ptr(cu), nseq, Hq, Hkv, L, d,
                                int(window), float(ratio), float(scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg))
    return {"dq": dq, "dk": dk, "dv": dv, "dg": dg, "n_sel": int(n)}


def selection_flags(g, ratio: float, cu_seqlens=None) -> torch.Tensor:
    """uint8 [B, L]: 1 where the budget rule selects the position (per sequence)."""
    g32 = g.detach().to(torch.float32)
    B, L = g32.shape
    flags = torch.zeros(B, L, dtype=torch.uint8)
    if cu_seqlens is None:
        spans = [(b, 0, L) for b in range(B)]
    else:
        cu = cu_seqlens.tolist()
        spans = [(0, cu[s], cu[s + 1]) for s in range(len(cu) - 1)]
    for b, a, e in spans:
        if e > a:
            flags[b, a + select(g32[b, a:e], ratio).long()] = 1
    return flags


def backward_rows(q, k, v, g, dout, window: int, ratio: float, qrows=(), krows=(), scale: float = 0.0,
                  cu_seqlens=None, flags=None):
    """Sampled gradient rows in fp64.

    ``qrows``: (seq, query head, position) triples -> ``dq`` [nq, d] and the
    gate gradient ``dg`` [nq] at that position (all heads).  ``krows``:
    (seq, key/value head, position) -> ``dk``, ``dv`` [nk, d].  Positions are
    relative to the sequence start.
    """
    B, Hq, Hkv, L, d, nseq = _geometry(q, k, cu_seqlens)
    qb, kb, vb, eb = _bits(q), _bits(k), _bits(v), _bits(dout)
    g32 = g.detach().to(torch.float32).contiguous()
    cu = None if cu_seqlens is None else cu_seqlens.to(torch.int32).contiguous()
    if flags is None:
        flags = selection_flags(g32, ratio, cu)
    flags = flags.to(torch.uint8).contiguous()
    qr = list(qrows)
    kr = list(krows)
    cols = lambda rows, i, dt: torch.tensor([r[i] for r in rows] or [0], dtype=dt)
    qs, qh, qp = cols(qr, 0, torch.int32), cols(qr, 1, torch.int32), cols(qr, 2, torch.int64)
    ks, kh, kp = cols(kr, 0, torch.int32), cols(kr, 1, torch.int32), cols(kr, 2, torch.int64)
    dq = torch.empty(max(1, len(qr)), d, dtype=torch.float64)
    dg = torch.empty(max(1, len(qr)), dtype=torch.float64)
    dk = torch.empty(max(1, len(kr)), d, dtype=torch.float64)
    dv = torch.empty_like(dk)
    _load().oracle_backward_rows(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(g32), _ptr(eb), _ptr(flags), _ptr(cu), nseq,
                                 Hq, Hkv, L, d, int(window), float(scale), len(qr), _ptr(qs), _ptr(qh), _ptr(qp),
                                 _ptr(dq), _ptr(dg), len(kr), _ptr(ks), _ptr(kh), _ptr(kp), _ptr(dk), _ptr(dv))
    return {"dq": dq[:len(qr)], "dg": dg[:len(qr)], "dk": dk[:len(kr)], "dv": dv[:len(kr)]}
