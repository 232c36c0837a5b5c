"""Helpers shared by the GPU tests: resident synthetic layers, oracle calls, tolerances."""
from __future__ import annotations

import concurrent.futures as cf
import os

import numpy as np
import torch

import oracle
import synth

# FFN tolerance of the float32-accumulate (CUDA-core) path: normwise per token,
# max_j |y - y_ref| / max_j |y_ref|.
TOL_GEMV = 1e-4
# Tensor-core path (int8 MMA): x and h are rounded to 16-bit fixed point per row (half a unit of
# 2^-15 of the row maximum); with max/rms ~4.5 for x and ~10 for h the per-element errors are
# ~4e-5 and ~9e-5 of the row rms, and the normwise output error is of that order.
TOL_TC = 3e-4


def tol_for(q, cfg, T) -> float:
    """FFN tolerance of the path coli_moe_layer / coli_moe_ffn take for T tokens."""
    return TOL_TC if q.coli_moe_layer_kernels(cfg, T) == 7 else TOL_GEMV


def normwise_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.abs(got - ref).max(axis=-1)
    den = np.maximum(np.abs(ref).max(axis=-1), 1e-300)
    return float((num / den).max()) if got.size else 0.0


class Layer:
    """One synthetic layer resident on `device`, with host copies made on demand."""

    def __init__(self, wl: synth.Workload, device="cuda", layer: int = 0):
        self.wl = wl
        self.layer = layer
        self.device = device
        self.experts = synth.make_expert_records(wl, device=device, layer=layer)
        self.shared = synth.make_shared_record(wl, device=device, layer=layer)
        self.Wr, self.bias = synth.make_router(wl, device=device, layer=layer)
        self._host = {}

    def weights(self):
        import quantized_routed_expert_noaux_b200 as q
        return q.weights_for(self.Wr, self.bias, self.experts, self.shared)

    def host_records(self, ids) -> oracle.Records:
        need = sorted({int(e) for e in np.asarray(ids).reshape(-1)})
        for e in need:
            if e not in self._host:
                self._host[e] = self.experts[e].cpu().numpy()
        table = [self._host.get(e) for e in range(self.wl.n_experts)]
        sh = None if self.shared is None else self.shared.cpu().numpy()
        return oracle.Records(table, sh)

    def host_router(self):
        return self.Wr.cpu(), self.bias.cpu()


def oracle_gate(cfg, Wr, x_host, T, threads=None):
    """oracle.gate over token blocks on a thread pool (ctypes releases the GIL)."""
    threads = threads or min(16, os.cpu_count() or 1)
    if T <= 8 or threads == 1:
        return oracle.gate(cfg, Wr, x_host, T)
    blocks = np.array_split(np.arange(T), threads)
    out = np.zeros((T, cfg.n_experts), np.float32)

    def run(b):
        if len(b):
            out[b[0]:b[-1] + 1] = oracle.gate(cfg, Wr, x_host[b[0]:b[-1] + 1], len(b))

    with cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(run, blocks))
    return out


def oracle_layer_tokens(layer: Layer, x_host, tokens, threads=None):
    """Oracle output for the listed tokens only (the layer is per-token)."""
    wl = layer.wl
    cfg = oracle.make_cfg(wl)
    Wr, bias = layer.host_router()
    xs = x_host[list(tokens)]
    lg = oracle.gate(cfg, Wr, xs, len(tokens))
    ids, w = oracle.route(cfg, lg, bias, len(tokens))
    recs = layer.host_records(ids)
    out, ids2, w2, lg2 = oracle.layer(cfg, Wr, bias, recs, xs, len(tokens),
                                      n_threads=threads or min(16, os.cpu_count() or 1))
    return out, ids2, w2, lg2


def ulp_diff_f32(a, b):
    a = np.ascontiguousarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.ascontiguousarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b)
