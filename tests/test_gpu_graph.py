"""The layer inside a CUDA graph: a decode server captures its steps once and replays them.

Several layer calls on different inputs are captured into one graph and replayed; every replay
must give what direct calls on the same inputs give. The fused decode kernel keeps its barrier
counters and phase word in the workspace, so back-to-back replays exercise the hand-over between
calls. The GEMV and tensor-core paths are covered too.
"""
import pytest
import torch

import synth
from tests._common import Layer, normwise_err, tol_for

pytestmark = pytest.mark.gpu

q = pytest.importorskip("quantized_routed_expert_noaux_b200")

_LAYERS = {}


def _layer(name):
    if name not in _LAYERS:
        _LAYERS.clear()
        torch.cuda.empty_cache()
        _LAYERS[name] = Layer(synth.WORKLOADS[name], "cuda", 0)
    return _LAYERS[name]


# (workload, tokens, outputs bitwise equal): fused decode kernel (T <= 4), GEMV path (group-scaled
# records above 4 tokens) and tensor-core path (float-atomic combine: equal within tolerance)
@pytest.mark.parametrize("name,T,bitwise", [("glm_decode", 1, True), ("glm_decode", 4, True),
                                            ("glm_gs64", 8, True), ("olmoe", 32, False)])
def test_layer_replays_in_a_cuda_graph(name, T, bitwise):
    L = _layer(name)
    cfg = q.config_for(L.wl)
    n = 3
    xs = [synth.make_activations(L.wl, T, device="cuda", step=40 + i) for i in range(n)]
    ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    q.coli_moe_clear_error(ws)

    def buffers():
        return ([torch.empty(T, L.wl.hidden, dtype=torch.float32, device="cuda") for _ in range(n)],
                [torch.empty(T, L.wl.top_k, dtype=torch.int32, device="cuda") for _ in range(n)],
                [torch.empty(T, L.wl.top_k, dtype=torch.float32, device="cuda") for _ in range(n)])

    ref_o, ref_i, ref_w = buffers()
    for i in range(n):
        q.coli_moe_layer(cfg, L.weights(), xs[i], T, ref_o[i], ref_i[i], ref_w[i], ws)
    torch.cuda.synchronize()
    assert q.coli_moe_error_word(ws) == 0

    got_o, got_i, got_w = buffers()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            q.coli_moe_layer(cfg, L.weights(), xs[i], T, got_o[i], got_i[i], got_w[i], ws)
    try:
        for _ in range(3):
            for t in got_o + got_w:
                t.fill_(float("nan"))
            for t in got_i:
                t.fill_(-1)
            g.replay()
            torch.cuda.synchronize()
            for i in range(n):
                assert torch.equal(got_i[i], ref_i[i])
                assert torch.equal(got_w[i], ref_w[i])
                if bitwise:
                    assert torch.equal(got_o[i], ref_o[i])
                else:
                    err = normwise_err(got_o[i].cpu().numpy(), ref_o[i].cpu().numpy())
                    assert err <= tol_for(q, cfg, T), err
        assert q.coli_moe_error_word(ws) == 0
    finally:
        del g
