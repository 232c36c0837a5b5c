"""GPU parity of the tensor-core grouped-GEMM path (batches above 4 tokens; int4, int8 and int2
weights with per-row scales).

x and h enter the int8 MMAs as 16-bit fixed point per row, so outputs are compared with the
tensor-core tolerance (TOL_TC, normwise per token); routing and grouping stay bit-exact.  The
oracle computes sampled tokens one by one (the layer is per-token).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._common import TOL_TC, Layer, normwise_err, oracle_gate

pytestmark = pytest.mark.gpu

q = pytest.importorskip("quantized_routed_expert_noaux_b200")

_L = {}
TC_KERNELS = 7  # gate, route, group, x quantisation, gate/up GEMM, h quantisation, down GEMM
CHUNK_TOKENS = 96  # tokens of one expert per tile of the grouped GEMM


# f32 activations and four 64-row gate/up m-blocks: the tiny layer's router and expert counts at
# the smallest shape the tensor-core path takes (hidden and inter multiples of 256)
_EXTRA = {"tiny_wide": synth.WORKLOADS["tiny"].replace(name="tiny_wide", hidden=512, inter=256,
                                                      shared_inter=256)}


def layer(name):
    if name not in _L:
        _L.clear()
        torch.cuda.empty_cache()
        wl = _EXTRA[name] if name in _EXTRA else synth.WORKLOADS[name]
        _L[name] = Layer(wl, "cuda", 0)
    return _L[name]


def _group_gpu(cfg, ids_dev, T, E, ws):
    dev = lambda n: torch.empty(n, dtype=torch.int32, device="cuda")
    counts, offsets, perm, uniq, nu = dev(E), dev(E + 1), dev(T * cfg.top_k), dev(E), dev(1)
    q.coli_moe_group(cfg, ids_dev, T, counts, offsets, perm, uniq, nu, ws)
    return offsets, perm, uniq, nu


def _routing(L, ocfg, x, T, routing):
    wl = L.wl
    if routing == "oracle":
        lg = oracle_gate(ocfg, L.Wr.cpu(), x.cpu(), T)
        return oracle.route(ocfg, lg, L.bias.cpu(), T)
    rng = np.random.default_rng(T)
    ids_np = np.zeros((T, wl.top_k), np.int32)
    for t in range(T):
        others = rng.choice([e for e in range(wl.n_experts) if e != 3], wl.top_k - 1, replace=False)
        ids_np[t] = [3] + list(others)
    w_np = rng.uniform(0.1, 1.0, size=(T, wl.top_k)).astype(np.float32)
    return ids_np, w_np


# (workload, tokens, routing): chunks of 1..96 tokens with ragged tails; one expert with 128 and
# with 160 tokens (two chunks each, the second ragged); one token above the fused decode limit (5: chunks of one
# token); f32 activations and four gate/up m-blocks (tiny_wide); no shared expert (olmoe).
CASES = [("glm_decode", 96, "oracle"), ("glm_decode", 300, "oracle"), ("glm_decode", 160, "one_expert"),
         ("glm_decode", 128, "one_expert"), ("glm_decode", 65, "oracle"), ("glm_decode", 5, "oracle"),
         ("olmoe", 200, "oracle"), ("olmoe", 97, "one_expert"), ("olmoe", 8, "oracle"),
         ("tiny_wide", 100, "oracle")]


@pytest.mark.parametrize("name,T,routing", CASES)
def test_tc_ffn_matches_oracle(name, T, routing):
    L = layer(name)
    wl = L.wl
    cfg = q.config_for(wl)
    assert q.coli_moe_layer_kernels(cfg, T) == TC_KERNELS + (2 if q.coli_moe_dispatch_threshold() else 0)
    ocfg = oracle.make_cfg(wl)
    x = synth.make_activations(wl, T, device="cuda", step=30 + T)
    ids_np, w_np = _routing(L, ocfg, x, T, routing)
    ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    q.coli_moe_clear_error(ws)
    offsets, perm, uniq, nu = _group_gpu(cfg, torch.from_numpy(ids_np).cuda(), T, wl.n_experts, ws)
    out = torch.full((T, wl.hidden), float("nan"), device="cuda")
    q.coli_moe_ffn(cfg, L.weights(), x, T, torch.from_numpy(w_np).cuda(), offsets, perm, uniq,
                   nu, out, ws)
    assert q.coli_moe_error_word(ws) == 0
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    toks = sorted(set([0, 1, T // 3, T // 2, T - 2, T - 1]))
    ref = oracle.ffn(ocfg, L.host_records(ids_np[toks]), x.cpu()[toks], len(toks), ids_np[toks],
                     w_np[toks])
    err = normwise_err(got[toks], ref)
    print(f"{name} T={T} {routing}: normwise error {err:.2e}")
    assert err <= TOL_TC, err


def test_tc_layer_olmoe_all_tokens():
    """Every token of a 200-token OLMoE-shaped layer through coli_moe_layer."""
    L = layer("olmoe")
    wl = L.wl
    T = 200
    cfg = q.config_for(wl)
    x = synth.make_activations(wl, T, device="cuda", step=7)
    out = torch.empty(T, wl.hidden, dtype=torch.float32, device="cuda")
    ids = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
    ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    q.coli_moe_clear_error(ws)
    q.coli_moe_layer(cfg, L.weights(), x, T, out, ids, w, ws)
    assert q.coli_moe_error_word(ws) == 0
    ocfg = oracle.make_cfg(wl)
    lg = oracle_gate(ocfg, L.Wr.cpu(), x.cpu(), T)
    ids_ref, w_ref = oracle.route(ocfg, lg, L.bias.cpu(), T)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    np.testing.assert_array_equal(w.cpu().numpy(), w_ref)
    ref = oracle.ffn(ocfg, L.host_records(ids_ref), x.cpu(), T, ids_ref, w_ref)
    err = normwise_err(out.cpu().numpy(), ref)
    print(f"olmoe layer T={T}: normwise error {err:.2e}")
    assert err <= TOL_TC, err


@pytest.mark.parametrize("name,T,all_tokens", [("olmoe", 20, True), ("glm_decode", 40, False)])
def test_tc_ffn_per_expert_dispatch(name, T, all_tokens):
    """a5' per-expert dispatch: with the threshold at 3, the experts with 1..3 tokens take the
    GEMV kernels and the rest (one expert on every token, the shared expert, the 4+-token ones)
    the grouped GEMM, in one call; both add into the same out."""
    L = layer(name)
    wl = L.wl
    cfg = q.config_for(wl)
    ocfg = oracle.make_cfg(wl)
    x = synth.make_activations(wl, T, device="cuda", step=50 + T)
    ids_np, w_np = _routing(L, ocfg, x, T, "one_expert")
    counts = np.bincount(ids_np.ravel(), minlength=wl.n_experts)
    assert counts.max() == T and ((counts >= 1) & (counts <= 3)).sum() >= 10  # mixed sizes
    old = q.coli_moe_dispatch_threshold()
    q.coli_moe_set_dispatch_threshold(3)
    try:
        assert q.coli_moe_layer_kernels(cfg, T) == TC_KERNELS + 2
        ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
        q.coli_moe_clear_error(ws)
        offsets, perm, uniq, nu = _group_gpu(cfg, torch.from_numpy(ids_np).cuda(), T, wl.n_experts, ws)
        out = torch.full((T, wl.hidden), float("nan"), device="cuda")
        q.coli_moe_ffn(cfg, L.weights(), x, T, torch.from_numpy(w_np).cuda(), offsets, perm, uniq,
                       nu, out, ws)
        assert q.coli_moe_error_word(ws) == 0
    finally:
        q.coli_moe_set_dispatch_threshold(old)
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    toks = list(range(T)) if all_tokens else sorted(set([0, 1, T // 3, T // 2, T - 2, T - 1]))
    ref = oracle.ffn(ocfg, L.host_records(ids_np[toks]), x.cpu()[toks], len(toks), ids_np[toks],
                     w_np[toks])
    err = normwise_err(got[toks], ref)
    print(f"{name} T={T} mixed dispatch: normwise error {err:.2e}")
    assert err <= TOL_TC, err


@pytest.mark.parametrize("fmt", [8, 2])
def test_tc_layer_int8_int2_all_tokens(fmt):
    """Every token of a 48-token layer with int8 or int2 records on the tensor-core path: int8
    codes enter the MMA as they are, int2 codes as 64q, each in the order the activations are
    written in (tiny_wide's router and expert counts, 512 x 256 experts)."""
    wl = _EXTRA["tiny_wide"].replace(name=f"tiny_wide_i{fmt}", fmt=fmt)
    L = Layer(wl, "cuda", 0)
    T = 48
    cfg = q.config_for(wl)
    assert q.coli_moe_layer_kernels(cfg, T) == TC_KERNELS
    x = synth.make_activations(wl, T, device="cuda", step=9)
    out = torch.empty(T, wl.hidden, dtype=torch.float32, device="cuda")
    ids = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
    ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    q.coli_moe_clear_error(ws)
    q.coli_moe_layer(cfg, L.weights(), x, T, out, ids, w, ws)
    assert q.coli_moe_error_word(ws) == 0
    ocfg = oracle.make_cfg(wl)
    lg = oracle_gate(ocfg, L.Wr.cpu(), x.cpu(), T)
    ids_ref, w_ref = oracle.route(ocfg, lg, L.bias.cpu(), T)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    np.testing.assert_array_equal(w.cpu().numpy(), w_ref)
    ref = oracle.ffn(ocfg, L.host_records(ids_ref), x.cpu(), T, ids_ref, w_ref)
    err = normwise_err(out.cpu().numpy(), ref)
    print(f"int{fmt} layer T={T}: normwise error {err:.2e}")
    assert err <= TOL_TC, err


def test_prefill_layer_zipf_2048():
    """The GLM-5.2-shaped prefill layer: 2048 tokens, Zipf(1.1) expert popularity."""
    L = layer("glm_prefill")
    wl = L.wl
    T = 2048
    cfg = q.config_for(wl)
    x = synth.make_activations(wl, T, device="cuda", step=0)
    out = torch.empty(T, wl.hidden, dtype=torch.float32, device="cuda")
    ids = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
    ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    q.coli_moe_clear_error(ws)
    q.coli_moe_layer(cfg, L.weights(), x, T, out, ids, w, ws)
    assert q.coli_moe_error_word(ws) == 0
    ocfg = oracle.make_cfg(wl)
    lg = oracle_gate(ocfg, L.Wr.cpu(), x.cpu(), T)
    ids_ref, w_ref = oracle.route(ocfg, lg, L.bias.cpu(), T)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    np.testing.assert_array_equal(w.cpu().numpy(), w_ref)
    counts = np.bincount(ids_ref.reshape(-1), minlength=wl.n_experts)
    assert counts.max() > 200  # Zipf head: several hundred tokens on the most popular expert
    toks = set([0, 7, 511, 1024, 1500, 2047])
    # the first and last token of every chunk of every expert that spans several chunks (the
    # Zipf head: chunks of CHUNK_TOKENS slots in ascending slot order)
    for e in np.flatnonzero(counts > CHUNK_TOKENS):
        slot_tokens = np.flatnonzero((ids_ref == e).any(axis=1))
        for c0 in range(0, len(slot_tokens), CHUNK_TOKENS):
            part = slot_tokens[c0:c0 + CHUNK_TOKENS]
            toks.update((int(part[0]), int(part[-1])))
    toks = sorted(toks)
    assert len(toks) > 12
    recs = L.host_records(ids_ref[toks])
    ref = oracle.ffn(ocfg, recs, x.cpu()[toks], len(toks), ids_ref[toks], w_ref[toks])
    err = normwise_err(out.cpu().numpy()[toks], ref)
    print(f"glm prefill T=2048: {len(toks)} tokens checked, normwise error {err:.2e}")
    assert err <= TOL_TC, err


def test_prefill_layer_repeatable_all_tokens():
    """Every token of the 2048-token layer agrees across repeated calls on the same input.

    The down projection combines with float atomics, so runs may differ in the last bits of a
    sum (~1e-7 relative); a pipeline race would change whole rows of a tile by orders more."""
    L = layer("glm_prefill")
    wl = L.wl
    T = 2048
    cfg = q.config_for(wl)
    x = synth.make_activations(wl, T, device="cuda", step=1)
    ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    q.coli_moe_clear_error(ws)
    outs, idss = [], []
    for _ in range(3):
        out = torch.empty(T, wl.hidden, dtype=torch.float32, device="cuda")
        ids = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
        q.coli_moe_layer(cfg, L.weights(), x, T, out, ids, w, ws)
        assert q.coli_moe_error_word(ws) == 0
        outs.append(out.cpu().numpy())
        idss.append(ids.cpu().numpy())
    for r in (1, 2):
        np.testing.assert_array_equal(idss[r], idss[0])
        assert normwise_err(outs[r], outs[0]) <= 1e-5
