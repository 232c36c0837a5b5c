"""GPU parity: the CUDA path through the C ABI against the CPU oracle, on the same seeded inputs.

Routing (ids, weights) and grouping are compared bit for bit; the float32 logits to the ulp;
the expert outputs within the float32-accumulate tolerance (normwise per token).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._common import (Layer, normwise_err, oracle_gate, oracle_layer_tokens, tol_for,
                           ulp_diff_f32)

pytestmark = pytest.mark.gpu

q = pytest.importorskip("quantized_routed_expert_noaux_b200")

_LAYERS = {}


def layer_for(name, layer=0):
    key = (name, layer)
    if key not in _LAYERS:
        if len(_LAYERS) > 2:
            _LAYERS.clear()
            torch.cuda.empty_cache()
        _LAYERS[key] = Layer(synth.WORKLOADS[name], "cuda", layer)
    return _LAYERS[key]


def workspace(cfg, T):
    return torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")


def run_layer(L: Layer, x, T):
    cfg = q.config_for(L.wl)
    out = torch.empty(T, L.wl.hidden, dtype=torch.float32, device="cuda")
    ids = torch.empty(T, L.wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, L.wl.top_k, dtype=torch.float32, device="cuda")
    ws = workspace(cfg, T)
    q.coli_moe_clear_error(ws)
    q.coli_moe_layer(cfg, L.weights(), x, T, out, ids, w, ws)
    assert q.coli_moe_error_word(ws) == 0
    return out.cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()


# --------------------------------------------------------------------------- a1 gate ------

@pytest.mark.parametrize("name,T", [("tiny", 8), ("tiny", 37), ("olmoe", 1), ("olmoe", 32),
                                    ("glm_decode", 1), ("glm_decode", 4), ("glm_int8", 64),
                                    ("glm_prefill", 2048)])
def test_gate_matches_oracle(name, T):
    L = layer_for(name)
    cfg = q.config_for(L.wl)
    x = synth.make_activations(L.wl, T, device="cuda", step=T)
    lg = torch.empty(T, L.wl.n_experts, dtype=torch.float32, device="cuda")
    q.coli_moe_gate(cfg, L.Wr, x, T, lg)
    got = lg.cpu().numpy()
    ref = oracle_gate(oracle.make_cfg(L.wl), L.Wr.cpu(), x.cpu(), T)
    ulp = ulp_diff_f32(got, ref)
    # double accumulation in another order: equal after rounding to float32 except where the
    # double sum sits within a few double ulps of a float32 rounding boundary
    assert ulp.max() <= 1
    assert (ulp != 0).sum() <= max(1, got.size // 100000)


# --------------------------------------------------------------------------- a2 route -----

@pytest.mark.parametrize("name,T", [("tiny", 8), ("tiny", 37), ("olmoe", 1), ("olmoe", 32),
                                    ("glm_decode", 1), ("glm_decode", 4), ("glm_int8", 64),
                                    ("glm_prefill", 2048)])
def test_route_matches_oracle_bit_exact(name, T):
    wl = synth.WORKLOADS[name]
    cfg = q.config_for(wl)
    ocfg = oracle.make_cfg(wl)
    rng = np.random.default_rng(T)
    logits = rng.standard_normal((T, wl.n_experts)).astype(np.float32)
    _, bias = synth.make_router(wl.replace(hidden=64))
    ids_ref, w_ref = oracle.route(ocfg, logits, bias, T)
    ids = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
    q.coli_moe_route(cfg, torch.from_numpy(logits).cuda(), bias.cuda(), T, ids, w)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    np.testing.assert_array_equal(w.cpu().numpy(), w_ref)


@pytest.mark.parametrize("case", range(5))
def test_route_closed_forms(case):
    import json, os
    c = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "router_closed_form.json")))["cases"][case]
    wl = synth.WORKLOADS["tiny"]
    cfg = q.config_for(wl)
    cfg.n_experts, cfg.top_k, cfg.n_group, cfg.topk_group = c["E"], c["K"], c["G"], c["TG"]
    cfg.routed_scaling = c["rsf"]
    ids = torch.empty(1, c["K"], dtype=torch.int32, device="cuda")
    w = torch.empty(1, c["K"], dtype=torch.float32, device="cuda")
    q.coli_moe_route(cfg, torch.tensor([c["logits"]], dtype=torch.float32, device="cuda"),
                     torch.tensor(c["bias"], dtype=torch.float32, device="cuda"), 1, ids, w)
    assert ids[0].tolist() == c["ids"]
    np.testing.assert_allclose(w[0].cpu().numpy(), np.array(c["w"], np.float32), rtol=0,
                               atol=c["w_tol"] + 1e-7 * (c["w_tol"] > 0))


def test_route_ties_and_degenerate():
    """All-equal logits and biases (every comparison a tie) and a single-group layer."""
    for G, TG in ((8, 4), (1, 1), (8, 8)):
        wl = synth.WORKLOADS["glm_decode"].replace(n_group=G, topk_group=TG)
        cfg = q.config_for(wl)
        T = 5
        logits = np.zeros((T, wl.n_experts), np.float32)
        bias = np.zeros(wl.n_experts, np.float32)
        bias[::7] = 0.25  # a few distinct levels, many exact ties
        ids_ref, w_ref = oracle.route(oracle.make_cfg(wl), logits, bias, T)
        ids = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
        q.coli_moe_route(cfg, torch.from_numpy(logits).cuda(), torch.from_numpy(bias).cuda(),
                         T, ids, w)
        np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
        np.testing.assert_array_equal(w.cpu().numpy(), w_ref)


# --------------------------------------------------------------------------- a3 group -----

@pytest.mark.parametrize("T,K,E,skew", [(1, 8, 256, 0), (4, 8, 256, 0), (37, 4, 16, 0),
                                        (64, 8, 256, 0), (2048, 8, 256, 1), (2048, 8, 256, 0),
                                        (300, 8, 64, 1), (1, 1, 16, 0)])
def test_group_matches_oracle_bit_exact(T, K, E, skew):
    wl = synth.WORKLOADS["glm_decode"].replace(n_experts=E, top_k=K, n_group=1, topk_group=1)
    cfg = q.config_for(wl)
    rng = np.random.default_rng(T + E)
    if skew:
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        ids_np = rng.choice(E, size=(T, K), p=p / p.sum()).astype(np.int32)
    else:
        ids_np = rng.integers(0, E, size=(T, K)).astype(np.int32)
    ref = oracle.group(ids_np, T, K, E)
    dev = lambda n: torch.empty(n, dtype=torch.int32, device="cuda")
    counts, offsets, perm, uniq, nu = dev(E), dev(E + 1), dev(T * K), dev(E), dev(1)
    ws = workspace(cfg, T)
    q.coli_moe_clear_error(ws)
    q.coli_moe_group(cfg, torch.from_numpy(ids_np).cuda(), T, counts, offsets, perm, uniq, nu, ws)
    assert q.coli_moe_error_word(ws) == 0
    np.testing.assert_array_equal(counts.cpu().numpy(), ref[0])
    np.testing.assert_array_equal(offsets.cpu().numpy(), ref[1])
    np.testing.assert_array_equal(perm.cpu().numpy(), ref[2])
    np.testing.assert_array_equal(uniq.cpu().numpy(), ref[3])
    assert int(nu.item()) == ref[4]


def test_group_flags_bad_ids():
    wl = synth.WORKLOADS["tiny"]
    cfg = q.config_for(wl)
    ids = torch.tensor([[0, 3, 99, 1]], dtype=torch.int32, device="cuda")
    dev = lambda n: torch.empty(n, dtype=torch.int32, device="cuda")
    E = wl.n_experts
    counts, offsets, perm, uniq, nu = dev(E), dev(E + 1), dev(4), dev(E), dev(1)
    ws = workspace(cfg, 1)
    q.coli_moe_clear_error(ws)
    q.coli_moe_group(cfg, ids, 1, counts, offsets, perm, uniq, nu, ws)
    assert q.coli_moe_error_word(ws) & q.DEVERR_EXPERT_ID
    assert int(offsets[E].item()) == 3 and int(nu.item()) == 3


# --------------------------------------------------------------------------- a4..a7 ffn ---

def _gpu_group(cfg, ids_dev, T, E, ws):
    dev = lambda n: torch.empty(n, dtype=torch.int32, device="cuda")
    counts, offsets, perm, uniq, nu = dev(E), dev(E + 1), dev(max(T * cfg.top_k, 1)), dev(E), dev(1)
    q.coli_moe_group(cfg, ids_dev, T, counts, offsets, perm, uniq, nu, ws)
    return offsets, perm, uniq, nu


@pytest.mark.parametrize("name,T,routing", [("tiny", 8, "oracle"), ("tiny", 5, "one_expert"),
                                            ("olmoe", 32, "oracle"), ("glm_decode", 4, "oracle"),
                                            ("glm_decode", 4, "one_expert"),
                                            ("glm_decode", 1, "oracle"),
                                            ("glm_decode", 16, "one_expert"),
                                            ("glm_gs64", 4, "one_expert"),
                                            ("glm_gs64", 3, "oracle")])
def test_ffn_matches_oracle(name, T, routing):
    L = layer_for(name)
    wl = L.wl
    cfg = q.config_for(wl)
    ocfg = oracle.make_cfg(wl)
    x = synth.make_activations(wl, T, device="cuda", step=7 + T)
    if routing == "oracle":
        lg = oracle.gate(ocfg, L.Wr.cpu(), x.cpu(), T)
        ids_np, w_np = oracle.route(ocfg, lg, L.bias.cpu(), T)
    else:
        # every token routed to expert 3 in slot 0 and to distinct others: n_e = T for one expert
        rng = np.random.default_rng(T)
        ids_np = np.zeros((T, wl.top_k), np.int32)
        for t in range(T):
            others = rng.choice([e for e in range(wl.n_experts) if e != 3], wl.top_k - 1,
                                replace=False)
            ids_np[t] = [3] + list(others)
        w_np = rng.uniform(0.1, 1.0, size=(T, wl.top_k)).astype(np.float32)
    ref = oracle.ffn(ocfg, L.host_records(ids_np), x.cpu(), T, ids_np, w_np)
    ws = workspace(cfg, T)
    q.coli_moe_clear_error(ws)
    offsets, perm, uniq, nu = _gpu_group(cfg, torch.from_numpy(ids_np).cuda(), T, wl.n_experts, ws)
    out = torch.full((T, wl.hidden), float("nan"), device="cuda")
    q.coli_moe_ffn(cfg, L.weights(), x, T, torch.from_numpy(w_np).cuda(), offsets, perm, uniq,
                   nu, out, ws)
    assert q.coli_moe_error_word(ws) == 0
    err = normwise_err(out.cpu().numpy(), ref)
    assert err <= tol_for(q, cfg, T), err


def test_ffn_flags_bad_unique_list():
    L = layer_for("tiny")
    wl = L.wl
    cfg = q.config_for(wl)
    T = 2
    x = synth.make_activations(wl, T, device="cuda")
    ws = workspace(cfg, T)
    q.coli_moe_clear_error(ws)
    E = wl.n_experts
    offsets = torch.zeros(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.zeros(T * wl.top_k, dtype=torch.int32, device="cuda")
    uniq = torch.full((E,), 999, dtype=torch.int32, device="cuda")
    nu = torch.tensor([2], dtype=torch.int32, device="cuda")
    w = torch.ones(T, wl.top_k, device="cuda")
    out = torch.empty(T, wl.hidden, device="cuda")
    q.coli_moe_ffn(cfg, L.weights(), x, T, w, offsets, perm, uniq, nu, out, ws)
    assert q.coli_moe_error_word(ws) & q.DEVERR_EXPERT_ID


# --------------------------------------------------------------------------- whole layer --

@pytest.mark.parametrize("name,T", [("tiny", 8), ("tiny", 1), ("tiny", 37), ("olmoe", 1),
                                    ("olmoe", 32), ("olmoe", 3), ("glm_decode", 1),
                                    ("glm_decode", 2), ("glm_decode", 3), ("glm_decode", 4),
                                    ("glm_decode", 5), ("glm_gs64", 1), ("glm_gs64", 2),
                                    ("glm_gs64", 4), ("glm_gs64", 5), ("glm_gs64", 24)])
def test_layer_matches_oracle(name, T):
    L = layer_for(name)
    x = synth.make_activations(L.wl, T, device="cuda", step=T)
    out, ids, w = run_layer(L, x, T)
    ref, ids_ref, w_ref, _ = oracle_layer_tokens(L, x.cpu(), range(T))
    np.testing.assert_array_equal(ids, ids_ref)
    np.testing.assert_array_equal(w, w_ref)
    err = normwise_err(out, ref)
    assert err <= tol_for(q, q.config_for(L.wl), T), err


@pytest.mark.parametrize("name", ["glm_int8", "glm_int2"])
def test_layer_alternate_containers_sampled(name):
    """64 tokens at full GLM size; the oracle checks 6 sampled tokens one by one."""
    L = layer_for(name)
    T = 64
    x = synth.make_activations(L.wl, T, device="cuda", step=3)
    out, ids, w = run_layer(L, x, T)
    toks = [0, 1, 17, 31, 32, 63]
    ref, ids_ref, w_ref, _ = oracle_layer_tokens(L, x.cpu(), toks)
    np.testing.assert_array_equal(ids[toks], ids_ref)
    np.testing.assert_array_equal(w[toks], w_ref)
    err = normwise_err(out[toks], ref)
    assert err <= tol_for(q, q.config_for(L.wl), T), err


def test_decode_shapes_take_fused_kernel():
    """Decode shapes run as one fused launch (a fall back to the five-kernel path would give the
    same outputs, only slower, so the launch count is checked here)."""
    for name, Ts in (("glm_decode", (1, 2, 3, 4)), ("olmoe", (1, 2, 4)), ("glm_int2", (1, 4)),
                     ("glm_gs64", (1, 2, 3, 4))):
        cfg = q.config_for(synth.WORKLOADS[name])
        for T in Ts:
            assert q.coli_moe_layer_kernels(cfg, T) == 1, (name, T)


@pytest.mark.parametrize("name", ["glm_int8", "glm_int2"])
@pytest.mark.parametrize("T", [1, 2])
def test_layer_alternate_containers_decode(name, T):
    """One and two tokens on int8 and int2 codes, every token (int2 takes the fused decode
    kernel; int8's down rows per CTA exceed its phase-2 row split, so it takes the GEMV path)."""
    L = layer_for(name)
    assert q.coli_moe_layer_kernels(q.config_for(L.wl), T) == (1 if name == "glm_int2" else 5)
    x = synth.make_activations(L.wl, T, device="cuda", step=20 + T)
    out, ids, w = run_layer(L, x, T)
    ref, ids_ref, w_ref, _ = oracle_layer_tokens(L, x.cpu(), range(T))
    np.testing.assert_array_equal(ids, ids_ref)
    np.testing.assert_array_equal(w, w_ref)
    err = normwise_err(out, ref)
    assert err <= tol_for(q, q.config_for(L.wl), T), err


@pytest.mark.parametrize("name,T", [("tiny", 8), ("glm_decode", 4), ("olmoe", 32)])
def test_batch_union_equals_per_token_bitwise(name, T):
    """The batch reads each unique expert once, yet every token's output is bit-identical to
    the token run alone whenever both calls take the same kernels (the fused decode path and the
    general or tensor-core path differ in their exact rounding; across paths the outputs agree
    within the sum of the two paths' tolerances)."""
    L = layer_for(name)
    cfg = q.config_for(L.wl)
    same_path = q.coli_moe_layer_kernels(cfg, T) == q.coli_moe_layer_kernels(cfg, 1)
    x = synth.make_activations(L.wl, T, device="cuda", step=11)
    out, _, _ = run_layer(L, x, T)
    for t in range(T):
        o1, _, _ = run_layer(L, x[t:t + 1].contiguous(), 1)
        if same_path:
            np.testing.assert_array_equal(o1[0], out[t])
        else:
            assert normwise_err(o1, out[t:t + 1]) <= tol_for(q, cfg, T) + tol_for(q, cfg, 1)


@pytest.mark.parametrize("T", [1, 4])
def test_layer_deterministic_and_repeatable(T):
    """Repeated calls on one workspace give identical bits and leave the error word clean; the
    fused path leaves its header ready for the next call: the phase word names a counter set
    that is all zero (the other set holds the last call's counts)."""
    L = layer_for("glm_decode")
    cfg = q.config_for(L.wl)
    ws = workspace(cfg, T)
    q.coli_moe_clear_error(ws)
    outs = []
    for rep in range(3):
        x = synth.make_activations(L.wl, T, device="cuda", step=5)
        out = torch.empty(T, L.wl.hidden, dtype=torch.float32, device="cuda")
        q.coli_moe_layer(cfg, L.weights(), x, T, out, None, None, ws)
        outs.append(out.cpu().numpy())
    assert q.coli_moe_error_word(ws) == 0
    hdr = ws[:512].view(torch.int32).cpu().numpy()  # header words: phase 8, arrivals 16 + 8 set,
    phase = int(hdr[8])                              # converted chunks 32 + 40 set
    assert phase in (0, 1), hdr
    assert hdr[16 + 8 * phase] == 0, hdr
    assert (hdr[32 + 40 * phase:32 + 40 * phase + 33] == 0).all(), hdr
    assert (hdr[1:8] == 0).all(), hdr
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[0], outs[2])


def test_layer_zero_tokens_is_noop():
    L = layer_for("tiny")
    cfg = q.config_for(L.wl)
    ws = workspace(cfg, 1)
    out = torch.full((1, L.wl.hidden), 7.0, device="cuda")
    x = synth.make_activations(L.wl, 1, device="cuda")
    q.coli_moe_layer(cfg, L.weights(), x, 0, out, None, None, ws)
    torch.cuda.synchronize()
    assert (out == 7.0).all()
