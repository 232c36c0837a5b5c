"""Seeded synthetic inputs for the routed-expert MoE layer.

This module is the one source of inputs shared by the CUDA path's tests/benchmark and the CPU
oracle.  It draws random numbers and writes them in the record format the layer reads; it
computes none of the layer's arithmetic (no routing, no dot products, no activation).  Its
quantise-and-pack step plays the part of the pages' offline converter (model preparation,
JustVugg/colibri README, "File: c/tools/README.md"), producing the container the layer
consumes; the layer's own decoders (CUDA and oracle) are written independently of it.

Recipe (shapes and distributions of the five named workloads):
  * activations: N(0,1), float32 for the tiny layer, otherwise rounded to bfloat16 (RNE);
  * router weight Wr[E,H]: N(0, 1/sqrt(H)) float32, so logits are about N(0,1);
  * selection bias[E]: N(0, 0.1) float32 (zero for the OLMoE-shaped layer); the prefill workload
    adds a Zipf(s=1.1) popularity offset (see `zipf_bias_offsets`);
  * expert weights N(0, 0.02), quantised per output row: scale = absmax/qmax (float32),
    code = round-half-even(w/scale) clamped to the format's range (int4 [-8,7] with qmax 7,
    int8 [-127,127] with qmax 127, int2 [-2,1] with qmax 1); an all-zero row gets scale 0.
  * packing: int4 element 2j -> low nibble of byte j, 2j+1 -> high nibble; int2 element 4j+k
    -> bits [2k, 2k+1] of byte j; two's complement.
  * record: Wg codes [I,H] | Wu codes [I,H] | Wd codes [H,I] | sg[I] | su[I] | sd[H] (f32),
    padded to a multiple of 256 bytes.

Expert e of a layer is drawn from its own torch.Generator seeded with (seed, e), so any subset
of experts can be regenerated without the rest.  CPU and CUDA generators give different
streams; a test always feeds both sides the same tensors.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable, Optional

import torch

__all__ = [
    "Workload", "WORKLOADS", "record_layout", "quantize_rows", "pack_codes",
    "make_router", "make_activations", "make_expert_records", "make_shared_record",
    "zipf_bias_offsets",
]

QMAX = {4: 7, 8: 127, 2: 1}
QMIN = {4: -8, 8: -127, 2: -2}
WEIGHT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes, routing constants and recipe of one named synthetic workload."""
    name: str
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    n_group: int
    topk_group: int
    n_shared: int
    shared_inter: int
    routed_scaling: float
    fmt: int                 # 4 packed int4, 8 int8, 2 packed int2
    act: str                 # "f32" or "bf16"
    tokens: tuple            # token counts this workload is run at
    bias_std: float
    seed: int
    zipf_s: float = 0.0      # > 0: Zipf popularity offsets in the selection bias
    n_layers: int = 1        # consecutive layers resident at once (chained workloads)
    group: int = 0           # 0: one scale per weight row; g: one per g consecutive columns

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


_GLM = dict(hidden=6144, inter=2048, n_experts=256, top_k=8, n_group=8, topk_group=4,
            n_shared=1, shared_inter=2048, routed_scaling=2.5, act="bf16", bias_std=0.1)

WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", hidden=256, inter=128, n_experts=16, top_k=4, n_group=2,
                     topk_group=1, n_shared=1, shared_inter=128, routed_scaling=2.5, fmt=4,
                     act="f32", tokens=(8,), bias_std=0.1, seed=0),
    "olmoe": Workload("olmoe", hidden=2048, inter=1024, n_experts=64, top_k=8, n_group=1,
                      topk_group=1, n_shared=0, shared_inter=0, routed_scaling=1.0, fmt=4,
                      act="bf16", tokens=(1, 32), bias_std=0.0, seed=1),
    "glm_decode": Workload("glm_decode", fmt=4, tokens=(1, 4), seed=2, **_GLM),
    "glm_prefill": Workload("glm_prefill", fmt=4, tokens=(2048,), seed=2, zipf_s=1.1, **_GLM),
    # GLM-5.2 expert shapes with 32 experts and uniform routing: a 0.6 GB layer on which the
    # tensor-core kernels run with mostly full token chunks (small enough for ncu captures)
    "glm_e32": Workload("glm_e32", fmt=4, tokens=(1024,), seed=2, **dict(_GLM, n_experts=32)),
    # GLM-5.2 expert shapes with 64 experts (8 groups, 4 kept) and the prefill layer's Zipf(1.1)
    # popularity at 512 tokens: ~64 tokens per expert on average with a long tail of small
    # ones, as on the 2048-token layer, in a 1.2 GB layer (small enough for ncu captures)
    "glm_zipf_e64": Workload("glm_zipf_e64", fmt=4, tokens=(512,), seed=2, zipf_s=1.1,
                             **dict(_GLM, n_experts=64)),
    # the group-scaled int4 container (one scale per 64 consecutive weights of a row) at the
    # GLM-5.2 decode shape: the pages' recommended GLM-5.2 build
    "glm_gs64": Workload("glm_gs64", fmt=4, tokens=(1, 4), seed=5, group=64, **_GLM),
    "glm_int8": Workload("glm_int8", fmt=8, tokens=(64,), seed=4, n_layers=4, **_GLM),
    "glm_int2": Workload("glm_int2", fmt=2, tokens=(64,), seed=4, n_layers=4, **_GLM),
}


def _row_bytes(n: int, fmt: int) -> int:
    return n * fmt // 8


def record_layout(hidden: int, inter: int, fmt: int, group: int = 0) -> dict:
    """Byte offsets of the six parts of one record and the padded record size.  Scales are one
    float32 per row, or with `group` one per `group` consecutive columns of a row."""
    rh, ri = _row_bytes(hidden, fmt), _row_bytes(inter, fmt)
    nh = hidden // group if group else 1
    ni = inter // group if group else 1
    o = {}
    o["wg"] = 0
    o["wu"] = inter * rh
    o["wd"] = 2 * inter * rh
    o["sg"] = o["wd"] + hidden * ri
    o["su"] = o["sg"] + 4 * inter * nh
    o["sd"] = o["su"] + 4 * inter * nh
    o["bytes"] = o["sd"] + 4 * hidden * ni
    o["stride"] = (o["bytes"] + 255) // 256 * 256
    o["row_bytes_h"], o["row_bytes_i"] = rh, ri
    return o


def _gen(device, *key: int) -> torch.Generator:
    g = torch.Generator(device=device)
    h = 0x9E3779B97F4A7C15
    for k in key:
        h = (h ^ (k & 0xFFFFFFFFFFFFFFFF)) * 0xBF58476D1CE4E5B9 & 0xFFFFFFFFFFFFFFFF
        h ^= h >> 31
    g.manual_seed(h & 0x7FFFFFFFFFFFFFFF)
    return g


def quantize_rows(w: torch.Tensor, fmt: int, group: int = 0):
    """Symmetric quantisation per row (group 0: codes int8 [R,C], scales float32 [R]) or per
    group of `group` consecutive columns of a row (scales float32 [R, C/group])."""
    qmax, qmin = QMAX[fmt], QMIN[fmt]
    R, Cn = w.shape
    wg = w.reshape(R, Cn // group, group) if group else w.reshape(R, 1, Cn)
    absmax = wg.abs().amax(dim=2)
    scale = (absmax / qmax).to(torch.float32)
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    q = torch.round(wg / safe[:, :, None]).clamp_(qmin, qmax)
    q = torch.where(scale[:, :, None] > 0, q, torch.zeros_like(q))
    return q.reshape(R, Cn).to(torch.int8), (scale if group else scale[:, 0])


def pack_codes(q: torch.Tensor, fmt: int) -> torch.Tensor:
    """Pack int8 codes [R,C] into the container's bytes [R, C*fmt/8] (uint8)."""
    if fmt == 8:
        return q.view(torch.uint8)
    u = q.to(torch.int32)
    if fmt == 4:
        lo = u[:, 0::2] & 0xF
        hi = u[:, 1::2] & 0xF
        return (lo | (hi << 4)).to(torch.uint8)
    if fmt == 2:
        b = torch.zeros_like(u[:, 0::4])
        for k in range(4):
            b |= (u[:, k::4] & 0x3) << (2 * k)
        return b.to(torch.uint8)
    raise ValueError(f"unsupported fmt {fmt}")


def _one_record(hidden: int, inter: int, fmt: int, g: torch.Generator, device,
                keep_codes: bool = False, group: int = 0):
    lay = record_layout(hidden, inter, fmt, group)
    rec = torch.zeros(lay["stride"], dtype=torch.uint8, device=device)
    parts = {}
    for name, (r, c) in (("g", (inter, hidden)), ("u", (inter, hidden)), ("d", (hidden, inter))):
        w = torch.randn(r, c, generator=g, device=device, dtype=torch.float32) * WEIGHT_STD
        q, s = quantize_rows(w, fmt, group)
        parts[name] = (q, s)
    rec[lay["wg"]:lay["wu"]] = pack_codes(parts["g"][0], fmt).reshape(-1)
    rec[lay["wu"]:lay["wd"]] = pack_codes(parts["u"][0], fmt).reshape(-1)
    rec[lay["wd"]:lay["sg"]] = pack_codes(parts["d"][0], fmt).reshape(-1)
    rec[lay["sg"]:lay["su"]] = parts["g"][1].contiguous().view(torch.uint8).reshape(-1)
    rec[lay["su"]:lay["sd"]] = parts["u"][1].contiguous().view(torch.uint8).reshape(-1)
    rec[lay["sd"]:lay["bytes"]] = parts["d"][1].contiguous().view(torch.uint8).reshape(-1)
    return (rec, parts) if keep_codes else (rec, None)


def make_expert_records(wl: Workload, device="cpu", layer: int = 0,
                        experts: Optional[Iterable[int]] = None, keep_codes: bool = False,
                        out: Optional[torch.Tensor] = None):
    """Routed-expert records [E, stride] uint8 (rows of experts not listed stay zero).

    With keep_codes, also returns {e: {"g"|"u"|"d": (codes int8, scales f32)}} -- the int8
    container view of the same weights, used by the container pins."""
    lay = record_layout(wl.hidden, wl.inter, wl.fmt, wl.group)
    E = wl.n_experts
    recs = out if out is not None else torch.zeros(E, lay["stride"], dtype=torch.uint8,
                                                    device=device)
    codes = {}
    for e in (range(E) if experts is None else experts):
        g = _gen(device, wl.seed, layer, 1, e)
        rec, parts = _one_record(wl.hidden, wl.inter, wl.fmt, g, device, keep_codes, wl.group)
        recs[e].copy_(rec)
        if keep_codes:
            codes[e] = parts
    return (recs, codes) if keep_codes else recs


def make_shared_record(wl: Workload, device="cpu", layer: int = 0, keep_codes: bool = False):
    """The shared expert's record [stride_s] uint8 (None when the workload has none)."""
    if wl.n_shared == 0:
        return (None, None) if keep_codes else None
    g = _gen(device, wl.seed, layer, 2)
    rec, parts = _one_record(wl.hidden, wl.shared_inter, wl.fmt, g, device, keep_codes, wl.group)
    return (rec, parts) if keep_codes else rec


def zipf_bias_offsets(wl: Workload, device="cpu", layer: int = 0) -> torch.Tensor:
    """Zipf(s) popularity offsets for the selection bias: alpha * ln(rank^-s).

    Ranks 1..E are dealt round-robin over the G groups (rank r -> group (r-1) mod G), and a
    seeded shuffle places them inside each group, so every group holds popular and unpopular
    experts.  ZIPF_ALPHA sets the strength of the skew: a fixed recipe constant, chosen so that
    on the 2048-token GLM-shaped layer the most popular expert takes several hundred tokens."""
    E, G = wl.n_experts, wl.n_group
    gs = E // G
    g = _gen("cpu", wl.seed, layer, 3)
    rank_of = torch.empty(E, dtype=torch.float64)
    slots = [torch.randperm(gs, generator=g) for _ in range(G)]
    for r in range(1, E + 1):
        grp = (r - 1) % G
        j = (r - 1) // G
        rank_of[grp * gs + int(slots[grp][j])] = r
    off = ZIPF_ALPHA * (-wl.zipf_s) * torch.log(rank_of)
    return off.to(torch.float32).to(device)


ZIPF_ALPHA = 0.06


def make_router(wl: Workload, device="cpu", layer: int = 0):
    """(Wr [E,H] float32, bias [E] float32)."""
    g = _gen(device, wl.seed, layer, 4)
    Wr = torch.randn(wl.n_experts, wl.hidden, generator=g, device=device,
                     dtype=torch.float32) * (1.0 / math.sqrt(wl.hidden))
    gb = _gen(device, wl.seed, layer, 5)
    bias = torch.randn(wl.n_experts, generator=gb, device=device, dtype=torch.float32)
    bias = bias * wl.bias_std
    if wl.zipf_s > 0:
        bias = (bias + zipf_bias_offsets(wl, device, layer)).to(torch.float32)
    return Wr.contiguous(), bias.contiguous()


def make_activations(wl: Workload, T: int, device="cpu", step: int = 0) -> torch.Tensor:
    """x [T,H]: float32 N(0,1), or that value rounded to bfloat16 for bf16 workloads."""
    g = _gen(device, wl.seed, 1000 + step, 6)
    x = torch.randn(T, wl.hidden, generator=g, device=device, dtype=torch.float32)
    return x if wl.act == "f32" else x.to(torch.bfloat16)
