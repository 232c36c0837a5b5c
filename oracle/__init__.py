"""ctypes wrapper over the CPU oracle (libcoli_oracle.so).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the package smoke check and by the
benchmark's CPU-baseline leg.  The product path never imports this package.

All arrays are host numpy arrays (torch CPU tensors are accepted and converted).  Shapes follow
coli_oracle.h.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))


class OracleCfg(C.Structure):
    _fields_ = [
        ("hidden", C.c_int), ("inter", C.c_int), ("n_experts", C.c_int), ("top_k", C.c_int),
        ("n_group", C.c_int), ("topk_group", C.c_int), ("n_shared", C.c_int),
        ("shared_inter", C.c_int), ("routed_scaling", C.c_double), ("fmt", C.c_int),
        ("act", C.c_int), ("group", C.c_int),
    ]


def _load():
    lib = C.CDLL(_build.build())
    P = C.c_void_p
    lib.oracle_record_bytes.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_size_t)]
    lib.oracle_unpack_row.argtypes = [P, C.c_int, C.c_int, P]
    lib.oracle_pack_row.argtypes = [P, C.c_int, C.c_int, P]
    lib.oracle_gate.argtypes = [C.POINTER(OracleCfg), P, P, C.c_int, P]
    lib.oracle_gate.restype = None
    lib.oracle_route.argtypes = [C.POINTER(OracleCfg), P, P, C.c_int, P, P, P, P]
    lib.oracle_group.argtypes = [C.c_int, C.c_int, C.c_int, P, P, P, P, P, P]
    lib.oracle_expert.argtypes = [C.POINTER(OracleCfg), P, C.c_int, P, P]
    lib.oracle_expert.restype = None
    lib.oracle_ffn.argtypes = [C.POINTER(OracleCfg), P, P, P, C.c_int, P, P, P]
    lib.oracle_ffn_union.argtypes = [C.POINTER(OracleCfg), P, P, P, C.c_int, P, P, P]
    lib.oracle_layer.argtypes = [C.POINTER(OracleCfg), P, P, P, P, P, C.c_int, P, P, P, P,
                                 C.c_int]
    lib.oracle_residual.argtypes = [C.POINTER(OracleCfg), P, P, C.c_size_t, P]
    lib.oracle_residual.restype = None
    return lib


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def _np(a, dtype=None):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        t = a.detach().cpu().contiguous()
        if str(t.dtype) == "torch.bfloat16":
            import torch
            t = t.view(torch.int16)
        a = t.numpy()
    a = np.ascontiguousarray(a)
    if dtype is not None and a.dtype != dtype:
        if a.dtype.itemsize == np.dtype(dtype).itemsize and a.dtype.kind in "iu" and \
                np.dtype(dtype).kind in "iu":
            a = a.view(dtype)
        else:
            a = a.astype(dtype)
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def make_cfg(wl) -> OracleCfg:
    """OracleCfg from a synth.Workload (or anything with the same attributes)."""
    return OracleCfg(wl.hidden, wl.inter, wl.n_experts, wl.top_k, wl.n_group, wl.topk_group,
                     wl.n_shared, wl.shared_inter, float(wl.routed_scaling), wl.fmt,
                     0 if wl.act == "f32" else 1, getattr(wl, "group", 0))


def _x(cfg: OracleCfg, x):
    return _np(x, np.float32 if cfg.act == 0 else np.uint16)


def record_bytes(hidden: int, inter: int, fmt: int, group: int = 0) -> int:
    n = C.c_size_t()
    if lib().oracle_record_bytes(hidden, inter, fmt, group, C.byref(n)) != 0:
        raise ValueError("bad record shape")
    return n.value


def unpack_row(row, n: int, fmt: int) -> np.ndarray:
    row = _np(row, np.uint8)
    q = np.zeros(n, np.int8)
    if lib().oracle_unpack_row(_ptr(row), n, fmt, _ptr(q)) != 0:
        raise ValueError("unpack failed")
    return q


def pack_row(q, fmt: int) -> np.ndarray:
    q = _np(q, np.int8)
    n = q.size
    out = np.zeros(n * fmt // 8, np.uint8)
    if lib().oracle_pack_row(_ptr(q), n, fmt, _ptr(out)) != 0:
        raise ValueError("pack failed (code out of range)")
    return out


def gate(cfg: OracleCfg, Wr, x, T: int) -> np.ndarray:
    Wr = _np(Wr, np.float32)
    x = _x(cfg, x)
    out = np.zeros((T, cfg.n_experts), np.float32)
    lib().oracle_gate(C.byref(cfg), _ptr(Wr), _ptr(x), T, _ptr(out))
    return out


def route(cfg: OracleCfg, logits, bias, T: int, margins: bool = False):
    logits = _np(logits, np.float32)
    bias = _np(bias, np.float32)
    ids = np.zeros((T, cfg.top_k), np.int32)
    w = np.zeros((T, cfg.top_k), np.float32)
    me = np.zeros(T, np.float64)
    mg = np.zeros(T, np.float64)
    rc = lib().oracle_route(C.byref(cfg), _ptr(logits), _ptr(bias), T, _ptr(ids), _ptr(w),
                            _ptr(me), _ptr(mg))
    if rc != 0:
        raise ValueError("oracle_route rejected the configuration")
    return (ids, w, me, mg) if margins else (ids, w)


def group(ids, T: int, K: int, E: int):
    ids = _np(ids, np.int32)
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(max(T * K, 1), np.int32)[: T * K]
    uniq = np.zeros(E, np.int32)
    nu = np.zeros(1, np.int32)
    if lib().oracle_group(T, K, E, _ptr(ids), _ptr(counts), _ptr(offsets), _ptr(perm),
                          _ptr(uniq), _ptr(nu)) != 0:
        raise ValueError("oracle_group: expert id out of range")
    return counts, offsets, perm, uniq, int(nu[0])


class Records:
    """Keeps the numpy buffers of the expert records alive and exposes a pointer table."""

    def __init__(self, experts: Sequence, shared=None):
        self.bufs = [None if r is None else _np(r, np.uint8) for r in experts]
        self.table = (C.c_void_p * len(self.bufs))(
            *[None if b is None else b.ctypes.data for b in self.bufs])
        self.shared = None if shared is None else _np(shared, np.uint8)

    @property
    def ptr(self):
        return C.cast(self.table, C.c_void_p)

    @property
    def shared_ptr(self):
        return _ptr(self.shared)


def expert(cfg: OracleCfg, record, inter: int, x) -> np.ndarray:
    rec = _np(record, np.uint8)
    x = _np(x, np.float64)
    y = np.zeros(cfg.hidden, np.float64)
    lib().oracle_expert(C.byref(cfg), _ptr(rec), inter, _ptr(x), _ptr(y))
    return y


def ffn(cfg: OracleCfg, recs: Records, x, T: int, ids, w, union: bool = False) -> np.ndarray:
    x = _x(cfg, x)
    ids = _np(ids, np.int32)
    w = _np(w, np.float32)
    out = np.zeros((T, cfg.hidden), np.float64)
    fn = lib().oracle_ffn_union if union else lib().oracle_ffn
    if fn(C.byref(cfg), recs.ptr, recs.shared_ptr, _ptr(x), T, _ptr(ids), _ptr(w),
          _ptr(out)) != 0:
        raise ValueError("oracle ffn failed (missing record or bad id)")
    return out


def layer(cfg: OracleCfg, Wr, bias, recs: Records, x, T: int, n_threads: int = 1):
    """Returns (out [T,H] float64, ids [T,K], w [T,K], logits [T,E])."""
    Wr = _np(Wr, np.float32)
    bias = _np(bias, np.float32)
    x = _x(cfg, x)
    out = np.zeros((T, cfg.hidden), np.float64)
    ids = np.zeros((T, cfg.top_k), np.int32)
    w = np.zeros((T, cfg.top_k), np.float32)
    lg = np.zeros((T, cfg.n_experts), np.float32)
    if lib().oracle_layer(C.byref(cfg), _ptr(Wr), _ptr(bias), recs.ptr, recs.shared_ptr,
                          _ptr(x), T, _ptr(out), _ptr(ids), _ptr(w), _ptr(lg),
                          n_threads) != 0:
        raise ValueError("oracle layer failed")
    return out, ids, w, lg


def residual(cfg: OracleCfg, x, out) -> np.ndarray:
    """x + out as the next layer's input: float32 sum, rounded to bf16 for bf16 activations.
    Returns bf16 bit patterns (uint16) for bf16 activations, float32 otherwise."""
    x = _x(cfg, x)
    out = _np(out, np.float32)
    if out.shape != x.shape:
        raise ValueError("x and out shapes differ")
    nxt = np.empty_like(x)
    lib().oracle_residual(C.byref(cfg), _ptr(x), _ptr(out), x.size, _ptr(nxt))
    return nxt
