"""coli_moe_layer_noalloc: the layer for callers that cannot allocate device memory.

Such callers (a plugin inside an engine whose GPU memory pool is fixed at start-up, a real-time
loop that cannot afford cudaMalloc's device-wide synchronisation) pass only their inputs and
outputs; the library keeps its scratch in one static device array.  This file is collected last
so that a run stopping at the first failure has already run every other test; it also passes
when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth
from tests._common import normwise_err

pytestmark = pytest.mark.gpu

q = pytest.importorskip("quantized_routed_expert_noaux_b200")


def _layer(name, device):
    wl = synth.WORKLOADS[name]
    ex = synth.make_expert_records(wl, device=device)
    sh = synth.make_shared_record(wl, device=device)
    Wr, b = synth.make_router(wl, device=device)
    return wl, (ex, sh, Wr, b), q.weights_for(Wr, b, ex, sh)


def _largest_fitting_tokens(cfg):
    T = 1
    while q.coli_moe_workspace_size(cfg, T + 1) <= q.STATIC_SCRATCH_BYTES:
        T += 1
    return T


def _both(cfg, weights, wl, T, step):
    """(out, ids, w) of coli_moe_layer with its own workspace and of coli_moe_layer_noalloc."""
    dev = torch.device("cuda", 0)
    x = synth.make_activations(wl, T, device=dev, step=step)
    ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device=dev)
    res = []
    for noalloc in (False, True):
        out = torch.full((T, wl.hidden), float("nan"), device=dev)
        ids = torch.full((T, wl.top_k), -1, dtype=torch.int32, device=dev)
        w = torch.full((T, wl.top_k), float("nan"), dtype=torch.float32, device=dev)
        if noalloc:
            q.coli_moe_layer_noalloc(cfg, weights, x, T, out, ids, w)
            assert q.coli_moe_noalloc_error_word() == 0  # the static array's error word reads clean
        else:
            q.coli_moe_clear_error(ws)
            q.coli_moe_layer(cfg, weights, x, T, out, ids, w, ws)
            assert q.coli_moe_error_word(ws) == 0
        res.append((out, ids, w))
    torch.cuda.synchronize()
    return res


@pytest.mark.parametrize("name,T", [("tiny", 4), ("glm_decode", 4), ("glm_decode", 1)])
def test_noalloc_matches_workspace_layer_twice(name, T):
    """Two calls in a row (the static scratch keeps the last call's bytes): the same kernels on
    the same inputs, so outputs and routing agree bit for bit."""
    dev = torch.device("cuda", 0)
    wl, keep, weights = _layer(name, dev)
    cfg = q.config_for(wl)
    assert q.coli_moe_layer_kernels(cfg, T) in (1, 5)  # deterministic paths (no float atomics)
    for call in range(2):
        (ref, ids_ref, w_ref), (out, ids, w) = _both(cfg, weights, wl, T, 100 + call)
        assert torch.equal(ids, ids_ref)
        assert torch.equal(w, w_ref)
        assert torch.equal(out, ref), (call, normwise_err(out.cpu().numpy(), ref.cpu().numpy()))


def test_noalloc_at_the_largest_size_and_one_beyond():
    """The largest token count whose scratch fits the static array runs (tensor-core path at the
    GLM shape: its down projection adds with float atomics, so outputs agree to rounding); one
    token more is rejected before any launch."""
    dev = torch.device("cuda", 0)
    wl, keep, weights = _layer("glm_decode", dev)
    cfg = q.config_for(wl)
    T = _largest_fitting_tokens(cfg)
    assert T >= 4
    (ref, ids_ref, w_ref), (out, ids, w) = _both(cfg, weights, wl, T, 7)
    assert torch.equal(ids, ids_ref)
    assert torch.equal(w, w_ref)
    assert normwise_err(out.cpu().numpy(), ref.cpu().numpy()) <= 1e-6
    x = synth.make_activations(wl, T + 1, device=dev, step=8)
    out = torch.empty(T + 1, wl.hidden, device=dev)
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_layer_noalloc(cfg, weights, x, T + 1, out)
    assert ei.value.status == 7


def test_noalloc_rejects_sizes_beyond_the_static_array():
    """Rejected on size before the weights are looked at: null weight pointers are never read."""
    dev = torch.device("cuda", 0)
    wl = synth.WORKLOADS["glm_decode"]
    cfg = q.config_for(wl)
    T = 256
    assert q.coli_moe_workspace_size(cfg, T) > q.STATIC_SCRATCH_BYTES
    x = torch.zeros(T, wl.hidden, dtype=torch.bfloat16, device=dev)
    out = torch.empty(T, wl.hidden, device=dev)
    w = q.MoEWeights(None, None, None, 18915328, None)
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_layer_noalloc(cfg, w, x, T, out)
    assert ei.value.status == 7
