"""Python binding of libcoli_moe.so: the routed-expert MoE layer on B200 (sm_100a).

Argument marshalling only.  Every function has the name of the C entry point it calls
(include/coli_moe.h), takes torch CUDA tensors (or None for a NULL pointer), passes their
device pointers and the current torch CUDA stream, and raises ColiError on a non-OK status.
Every step of the layer runs in the library's CUDA kernels; there is no CPU path.  Importing
this package raises ImportError when the library has not been built.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

__all__ = [
    "ColiError", "MoEConfig", "MoEWeights", "lib", "LIB_PATH",
    "coli_moe_status_str", "coli_moe_last_cuda_error", "coli_moe_record_bytes", "coli_moe_check_config",
    "coli_moe_workspace_size", "coli_moe_clear_error", "coli_moe_error_word",
    "coli_moe_gate", "coli_moe_route", "coli_moe_group", "coli_moe_ffn", "coli_moe_layer",
    "coli_moe_layer_noalloc", "coli_moe_noalloc_error_word", "STATIC_SCRATCH_BYTES", "coli_moe_layer_kernels", "coli_moe_residual",
    "coli_moe_debug_set_wait",
    "coli_moe_set_dispatch_threshold",
    "coli_moe_dispatch_threshold",
    "config_for", "weights_for",
    "COLI_W_INT2", "COLI_W_INT4", "COLI_W_INT8", "COLI_ACT_F32", "COLI_ACT_BF16",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcoli_moe.so")

COLI_W_INT2, COLI_W_INT4, COLI_W_INT8 = 2, 4, 8
COLI_ACT_F32, COLI_ACT_BF16 = 0, 1
DEVERR_EXPERT_ID, DEVERR_GROUPING, DEVERR_TIMEOUT = 0x1, 0x2, 0x4

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python quantized_routed_expert_noaux_b200/build.py` "
        "(there is no CPU fallback for this layer)")


class MoEConfig(C.Structure):
    _fields_ = [
        ("hidden", C.c_int), ("inter", C.c_int), ("n_experts", C.c_int), ("top_k", C.c_int),
        ("n_group", C.c_int), ("topk_group", C.c_int), ("n_shared", C.c_int),
        ("shared_inter", C.c_int), ("routed_scaling", C.c_double), ("wfmt", C.c_int),
        ("act", C.c_int), ("group_size", C.c_int),
    ]


class MoEWeights(C.Structure):
    _fields_ = [
        ("router_w", C.c_void_p), ("router_bias", C.c_void_p), ("experts", C.c_void_p),
        ("expert_stride", C.c_size_t), ("shared", C.c_void_p),
    ]


class ColiError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        extra = ""
        if status == 5:
            extra = " [" + lib.coli_moe_last_cuda_error().decode() + "]"
        super().__init__(f"{fn}: {coli_moe_status_str(status)} (status {status}){extra}")


def _load():
    L = C.CDLL(LIB_PATH)
    P, I, S = C.c_void_p, C.c_int, C.c_size_t
    cfgp, wp = C.POINTER(MoEConfig), C.POINTER(MoEWeights)
    L.coli_moe_status_str.argtypes = [I]
    L.coli_moe_status_str.restype = C.c_char_p
    L.coli_moe_last_cuda_error.argtypes = []
    L.coli_moe_last_cuda_error.restype = C.c_char_p
    L.coli_moe_record_bytes.argtypes = [I, I, I, I, C.POINTER(S)]
    L.coli_moe_check_config.argtypes = [cfgp]
    L.coli_moe_workspace_size.argtypes = [cfgp, I, C.POINTER(S)]
    L.coli_moe_clear_error.argtypes = [P, P]
    L.coli_moe_error_word.argtypes = [P, P, C.POINTER(I)]
    L.coli_moe_gate.argtypes = [cfgp, P, P, I, P, P]
    L.coli_moe_route.argtypes = [cfgp, P, P, I, P, P, P]
    L.coli_moe_group.argtypes = [cfgp, P, I, P, P, P, P, P, P, S, P]
    L.coli_moe_ffn.argtypes = [cfgp, wp, P, I, P, P, P, P, P, P, P, S, P]
    L.coli_moe_layer.argtypes = [cfgp, wp, P, I, P, P, P, P, S, P]
    L.coli_moe_layer_noalloc.argtypes = [cfgp, wp, P, I, P, P, P, P]
    L.coli_moe_noalloc_error_word.argtypes = [P, C.POINTER(I)]
    L.coli_moe_layer_kernels.argtypes = [cfgp, I, C.POINTER(I)]
    L.coli_moe_residual.argtypes = [cfgp, P, P, I, P, P]
    L.coli_moe_debug_set_wait.argtypes = [C.c_longlong, I]
    L.coli_moe_set_dispatch_threshold.argtypes = [I]
    L.coli_moe_dispatch_threshold.argtypes = []
    L.coli_moe_dispatch_threshold.restype = I
    L.coli_moe_layer_kernels.restype = I
    L.coli_moe_layer_noalloc.restype = I
    for name in ("coli_moe_record_bytes", "coli_moe_check_config", "coli_moe_workspace_size",
                 "coli_moe_clear_error", "coli_moe_error_word", "coli_moe_gate",
                 "coli_moe_route", "coli_moe_group", "coli_moe_ffn", "coli_moe_layer",
                 "coli_moe_residual", "coli_moe_debug_set_wait", "coli_moe_set_dispatch_threshold",
                 "coli_moe_noalloc_error_word"):
        getattr(L, name).restype = I
    return L


lib = _load()


def _p(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise ColiError(fn, status)


def coli_moe_status_str(status: int) -> str:
    return lib.coli_moe_status_str(status).decode()


def coli_moe_last_cuda_error() -> str:
    return lib.coli_moe_last_cuda_error().decode()


def coli_moe_record_bytes(hidden: int, inter: int, wfmt: int, group_size: int = 0) -> int:
    n = C.c_size_t()
    _check("coli_moe_record_bytes", lib.coli_moe_record_bytes(hidden, inter, wfmt, group_size, C.byref(n)))
    return n.value


def coli_moe_check_config(cfg: MoEConfig) -> None:
    _check("coli_moe_check_config", lib.coli_moe_check_config(C.byref(cfg)))


def coli_moe_workspace_size(cfg: MoEConfig, max_tokens: int) -> int:
    n = C.c_size_t()
    _check("coli_moe_workspace_size",
           lib.coli_moe_workspace_size(C.byref(cfg), max_tokens, C.byref(n)))
    return n.value


def coli_moe_clear_error(ws, stream=None) -> None:
    _check("coli_moe_clear_error", lib.coli_moe_clear_error(_p(ws), _stream(stream)))


def coli_moe_error_word(ws, stream=None) -> int:
    v = C.c_int()
    _check("coli_moe_error_word", lib.coli_moe_error_word(_p(ws), _stream(stream), C.byref(v)))
    return v.value


def coli_moe_layer_kernels(cfg, T) -> int:
    n = C.c_int()
    _check("coli_moe_layer_kernels", lib.coli_moe_layer_kernels(C.byref(cfg), T, C.byref(n)))
    return n.value


def coli_moe_gate(cfg, router_w, x, T, logits, stream=None) -> None:
    _check("coli_moe_gate", lib.coli_moe_gate(C.byref(cfg), _p(router_w), _p(x), T, _p(logits),
                                              _stream(stream)))


def coli_moe_route(cfg, logits, bias, T, topk_ids, topk_w, stream=None) -> None:
    _check("coli_moe_route", lib.coli_moe_route(C.byref(cfg), _p(logits), _p(bias), T,
                                                _p(topk_ids), _p(topk_w), _stream(stream)))


def coli_moe_group(cfg, topk_ids, T, counts, offsets, perm, unique_ids, n_unique, ws,
                   stream=None) -> None:
    _check("coli_moe_group", lib.coli_moe_group(
        C.byref(cfg), _p(topk_ids), T, _p(counts), _p(offsets), _p(perm), _p(unique_ids),
        _p(n_unique), _p(ws), _nbytes(ws), _stream(stream)))


def coli_moe_ffn(cfg, weights: MoEWeights, x, T, topk_w, offsets, perm, unique_ids, n_unique,
                 out, ws, stream=None) -> None:
    _check("coli_moe_ffn", lib.coli_moe_ffn(
        C.byref(cfg), C.byref(weights), _p(x), T, _p(topk_w), _p(offsets), _p(perm),
        _p(unique_ids), _p(n_unique), _p(out), _p(ws), _nbytes(ws), _stream(stream)))


def coli_moe_layer(cfg, weights: MoEWeights, x, T, out, topk_ids_out, topk_w_out, ws,
                   stream=None) -> None:
    _check("coli_moe_layer", lib.coli_moe_layer(
        C.byref(cfg), C.byref(weights), _p(x), T, _p(out), _p(topk_ids_out), _p(topk_w_out),
        _p(ws), _nbytes(ws), _stream(stream)))


def coli_moe_residual(cfg, x, out, T, x_next, stream=None) -> None:
    """x_next = x + out between chained layers (float32 sum; bf16 activations rounded to bf16)."""
    _check("coli_moe_residual", lib.coli_moe_residual(
        C.byref(cfg), _p(x), _p(out), T, _p(x_next), _stream(stream)))


# Size of the static scratch array behind coli_moe_layer_noalloc (COLI_MOE_STATIC_SCRATCH_BYTES).
STATIC_SCRATCH_BYTES = 8 << 20


def coli_moe_layer_noalloc(cfg, weights: MoEWeights, x, T, out, topk_ids_out=None,
                           topk_w_out=None, stream=None) -> None:
    """The whole layer for callers that cannot allocate device memory (a plugin whose GPU memory
    pool is fixed at start-up, a real-time loop that cannot afford cudaMalloc's synchronisation):
    no workspace argument; the library's static per-GPU scratch array is used instead.  Calls on
    one device share that array, so calls that overlap on the GPU must be ordered."""
    _check("coli_moe_layer_noalloc", lib.coli_moe_layer_noalloc(
        C.byref(cfg), C.byref(weights), _p(x), T, _p(out), _p(topk_ids_out), _p(topk_w_out),
        _stream(stream)))


def coli_moe_noalloc_error_word(stream=None) -> int:
    """Device error word of the static scratch array behind coli_moe_layer_noalloc (synchronises
    the stream): 0 when the last no-allocation call on this device ran clean."""
    v = C.c_int()
    _check("coli_moe_noalloc_error_word", lib.coli_moe_noalloc_error_word(_stream(stream), C.byref(v)))
    return v.value


def coli_moe_debug_set_wait(wait_cycles: int, unreachable: bool) -> None:
    """Testing aid: the fused decode kernel's wait bound (cycles, 0 = default) and whether its
    grid-barrier targets are out of reach (every wait then runs out and reports a timeout)."""
    _check("coli_moe_debug_set_wait", lib.coli_moe_debug_set_wait(wait_cycles, int(bool(unreachable))))


def coli_moe_set_dispatch_threshold(max_tokens: int) -> None:
    """a5' per-expert dispatch on the tensor-core path: work experts with at most max_tokens
    routed tokens take the CUDA-core GEMV kernels, the rest the grouped GEMM (0: all GEMM)."""
    _check("coli_moe_set_dispatch_threshold", lib.coli_moe_set_dispatch_threshold(int(max_tokens)))


def coli_moe_dispatch_threshold() -> int:
    """The current per-expert dispatch threshold."""
    return int(lib.coli_moe_dispatch_threshold())


def config_for(wl) -> MoEConfig:
    """MoEConfig with the shape fields of a workload description (any object with the
    attributes hidden, inter, n_experts, top_k, n_group, topk_group, n_shared, shared_inter,
    routed_scaling, fmt and act = "f32" | "bf16")."""
    return MoEConfig(wl.hidden, wl.inter, wl.n_experts, wl.top_k, wl.n_group, wl.topk_group,
                     wl.n_shared, wl.shared_inter, float(wl.routed_scaling), wl.fmt,
                     COLI_ACT_F32 if wl.act == "f32" else COLI_ACT_BF16, getattr(wl, "group", 0))


def weights_for(router_w, router_bias, experts, shared=None) -> MoEWeights:
    """MoEWeights over device tensors: experts is [E, stride] uint8, shared [stride_s] uint8."""
    return MoEWeights(_p(router_w), _p(router_bias), _p(experts), experts.stride(0),
                      _p(shared))
