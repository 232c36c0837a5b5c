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
from tests._common import TOL_GEMV, normwise_err

pytestmark = pytest.mark.gpu

q = pytest.importorskip("quantized_routed_expert_noaux_b200")


def _layer(name, device):
    wl = synth.WORKLOADS[name]
    ex = synth.make_expert_records(wl, device=device)
    sh = synth.make_shared_record(wl, device=device)
    Wr, b = synth.make_router(wl, device=device)
    return wl, (ex, sh, Wr, b), q.weights_for(Wr, b, ex, sh)


@pytest.mark.parametrize("name,T", [("tiny", 8), ("glm_decode", 4)])
def test_noalloc_matches_workspace_layer_twice(name, T):
    dev = torch.device("cuda", 0)
    wl, keep, weights = _layer(name, dev)
    cfg = q.config_for(wl)
    ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device=dev)
    for call in range(2):  # two calls in a row: the shared scratch keeps the last call's bytes
        x = synth.make_activations(wl, T, device=dev, step=100 + call)
        ref = torch.empty(T, wl.hidden, device=dev)
        ids_ref = torch.empty(T, wl.top_k, dtype=torch.int32, device=dev)
        q.coli_moe_clear_error(ws)
        q.coli_moe_layer(cfg, weights, x, T, ref, ids_ref, None, ws)
        out = torch.full((T, wl.hidden), float("nan"), device=dev)
        ids = torch.empty(T, wl.top_k, dtype=torch.int32, device=dev)
        w = torch.empty(T, wl.top_k, dtype=torch.float32, device=dev)
        q.coli_moe_layer_noalloc(cfg, weights, x, T, out, ids, w)
        torch.cuda.synchronize()
        assert torch.equal(ids, ids_ref)
        err = normwise_err(out.cpu().numpy(), ref.cpu().numpy())
        assert err <= TOL_GEMV, (call, err)


def test_noalloc_rejects_sizes_beyond_the_static_array():
    dev = torch.device("cuda", 0)
    wl = synth.WORKLOADS["glm_decode"]
    cfg = q.config_for(wl)
    T = 256
    assert q.coli_moe_workspace_size(cfg, T) > q.STATIC_SCRATCH_BYTES
    x = torch.zeros(T, wl.hidden, dtype=torch.bfloat16, device=dev)
    out = torch.empty(T, wl.hidden, device=dev)
    w = q.MoEWeights(256, 512, 1024 * 256, 18915328, 2048 * 256)
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_layer_noalloc(cfg, w, x, T, out)
    assert ei.value.status == 7
