"""Pins of the CPU oracle against things other than itself (CPU only).

* containers: the generator's int8-container codes vs the oracle's decode of the packed bytes
  (the pages' bit-identity rule), exhaustive byte round trips, hand-decoded bytes;
* router: hand-derived closed forms (tests/golden/router_closed_form.json), brute-force
  enumeration of group and expert subsets, the G=1 special case against a library stable sort,
  invariants (sum of weights = routed_scaling, positivity, kept groups);
* grouping: numpy's stable argsort / bincount / unique;
* expert FFN: a hand-derived closed form (tests/golden/expert_closed_form.json) and numpy
  float64 matmuls over the generator's codes x scales;
* gate: numpy float64 matmul rounded to float32;
* layer: batch-union equals per-token bit for bit, and the layer equals the sum of its parts
  computed by numpy;
* residual update: hand-worked ties of the bf16 rounding, and numpy's float32 sum rounded by
  torch's float32-to-bf16 conversion (round to nearest even).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _cfg(**kw):
    base = dict(hidden=8, inter=8, n_experts=4, top_k=2, n_group=1, topk_group=1, n_shared=0,
                shared_inter=0, routed_scaling=1.0, fmt=4, act=0)
    base.update(kw)
    return oracle.OracleCfg(**base)


# ------------------------------------------------------------------ containers -------------

@pytest.mark.parametrize("fmt", [4, 2, 8])
def test_packed_equals_int8_container(fmt):
    """Decoding the packed bytes gives exactly the int8-container codes (bit-identity rule)."""
    wl = synth.WORKLOADS["tiny"].replace(fmt=fmt)
    recs, codes = synth.make_expert_records(wl, experts=[3], keep_codes=True)
    lay = synth.record_layout(wl.hidden, wl.inter, fmt)
    rec = recs[3].numpy()
    for name, off, rows, cols in (("g", lay["wg"], wl.inter, wl.hidden),
                                  ("u", lay["wu"], wl.inter, wl.hidden),
                                  ("d", lay["wd"], wl.hidden, wl.inter)):
        q = codes[3][name][0].numpy()
        rb = cols * fmt // 8
        for r in range(rows):
            got = oracle.unpack_row(rec[off + r * rb: off + (r + 1) * rb], cols, fmt)
            np.testing.assert_array_equal(got, q[r])


def test_int4_all_bytes_round_trip():
    for b in range(256):
        q = oracle.unpack_row(np.array([b], np.uint8), 2, 4)
        assert -8 <= q.min() and q.max() <= 7
        assert oracle.pack_row(q, 4)[0] == b


def test_int2_all_bytes_round_trip():
    for b in range(256):
        q = oracle.unpack_row(np.array([b], np.uint8), 4, 2)
        assert -2 <= q.min() and q.max() <= 1
        assert oracle.pack_row(q, 2)[0] == b


def test_int4_all_code_pairs_round_trip():
    for lo, hi in itertools.product(range(-8, 8), repeat=2):
        b = oracle.pack_row(np.array([lo, hi], np.int8), 4)
        np.testing.assert_array_equal(oracle.unpack_row(b, 2, 4), [lo, hi])


def test_hand_decoded_bytes():
    # int4: 0x7F -> low nibble 0xF = -1 (element 0), high nibble 0x7 = 7 (element 1)
    np.testing.assert_array_equal(oracle.unpack_row(np.array([0x7F], np.uint8), 2, 4), [-1, 7])
    np.testing.assert_array_equal(oracle.unpack_row(np.array([0x80], np.uint8), 2, 4), [0, -8])
    # int2: 0b10_01_11_00 -> elements (bits 0-1, 2-3, 4-5, 6-7) = 0, -1, 1, -2
    np.testing.assert_array_equal(oracle.unpack_row(np.array([0b10011100], np.uint8), 4, 2),
                                  [0, -1, 1, -2])
    # int8 is the byte itself, two's complement (library view)
    raw = np.arange(256, dtype=np.uint8)
    np.testing.assert_array_equal(oracle.unpack_row(raw, 256, 8), raw.view(np.int8))


def test_pack_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.pack_row(np.array([8, 0], np.int8), 4)
    with pytest.raises(ValueError):
        oracle.pack_row(np.array([2, 0, 0, 0], np.int8), 2)


@pytest.mark.parametrize("fmt,H,I", [(4, 6144, 2048), (8, 6144, 2048), (2, 6144, 2048),
                                     (4, 256, 128)])
def test_record_bytes(fmt, H, I):
    n = oracle.record_bytes(H, I, fmt)
    assert n == synth.record_layout(H, I, fmt)["bytes"]
    if (fmt, H, I) == (4, 6144, 2048):
        assert n == 18_915_328          # the pages' "~19 MB each at int4"


# ------------------------------------------------------------------ router -----------------

def _route_case(case):
    cfg = _cfg(n_experts=case["E"], top_k=case["K"], n_group=case["G"],
               topk_group=case["TG"], routed_scaling=case["rsf"])
    lg = np.array([case["logits"]], np.float32)
    b = np.array(case["bias"], np.float32)
    return oracle.route(cfg, lg, b, 1)


@pytest.mark.parametrize("idx", range(5))
def test_router_closed_forms(idx):
    case = json.load(open(os.path.join(GOLD, "router_closed_form.json")))["cases"][idx]
    ids, w = _route_case(case)
    assert ids[0].tolist() == case["ids"], case["name"]
    np.testing.assert_allclose(w[0], np.array(case["w"], np.float32), rtol=0,
                               atol=case["w_tol"] + 1e-7 * (case["w_tol"] > 0))
    if case["w_tol"] == 0.0:
        np.testing.assert_array_equal(w[0], np.array(case["w"], np.float32))


def _brute_force(logits, bias, E, K, G, TG, rsf):
    """Enumerate every TG-subset of groups and every K-subset of their experts; keep the one
    no outside element beats under (value desc, index asc).  Independent of the oracle."""
    s = [1.0 / (1.0 + math.exp(-float(v))) for v in logits]
    c = [s[e] + float(bias[e]) for e in range(E)]
    gs = E // G

    if G == 1 or TG == G:
        kept = list(range(G))
    else:
        gsc = []
        for g in range(G):
            vals = sorted((c[e] for e in range(g * gs, (g + 1) * gs)), reverse=True)
            gsc.append(vals[0] + vals[1])
        kept = None
        for sub in itertools.combinations(range(G), TG):
            out = [g for g in range(G) if g not in sub]
            if all(gsc[i] > gsc[o] or (gsc[i] == gsc[o] and i < o)
                   for i in sub for o in out):
                kept = sub
                break
    allowed = [e for e in range(E) if (e // gs) in kept]
    chosen = None
    for sub in itertools.combinations(allowed, K):
        out = [e for e in allowed if e not in sub]
        if all(c[i] > c[o] or (c[i] == c[o] and i < o) for i in sub for o in out):
            chosen = sub
            break
    order = sorted(chosen, key=lambda e: (-c[e], e))
    tot = sum(s[e] for e in order)
    w = [np.float32((s[e] / tot) * rsf) for e in order]
    return order, w


@pytest.mark.parametrize("seed", range(40))
def test_router_brute_force(seed):
    rng = np.random.default_rng(seed)
    G = int(rng.choice([1, 2, 4]))
    gs = int(rng.choice([2, 3, 4]))
    E = G * gs
    TG = int(rng.integers(1, G + 1))
    K = int(rng.integers(1, TG * gs + 1))
    rsf = float(rng.choice([1.0, 2.5]))
    # coarse values make exact ties common
    logits = (rng.integers(-3, 4, size=E) * 0.5).astype(np.float32)
    bias = (rng.integers(-2, 3, size=E) * 0.125).astype(np.float32)
    cfg = _cfg(n_experts=E, top_k=K, n_group=G, topk_group=TG, routed_scaling=rsf)
    ids, w = oracle.route(cfg, logits[None], bias, 1)
    order, wb = _brute_force(logits, bias, E, K, G, TG, rsf)
    assert ids[0].tolist() == order
    np.testing.assert_array_equal(w[0], np.array(wb, np.float32))


def test_router_single_group_is_plain_topk():
    """G = 1: the selection is the first K of a stable sort by descending biased score."""
    rng = np.random.default_rng(7)
    E, K, T = 64, 8, 50
    logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.1).astype(np.float32)
    cfg = _cfg(n_experts=E, top_k=K, routed_scaling=1.0)
    ids, w = oracle.route(cfg, logits, bias, T)
    for t in range(T):
        c = 1.0 / (1.0 + np.exp(-logits[t].astype(np.float64))) + bias.astype(np.float64)
        ref = np.argsort(-c, kind="stable")[:K]
        assert ids[t].tolist() == ref.tolist()


def test_router_invariants_glm_shape():
    wl = synth.WORKLOADS["glm_decode"]
    cfg = oracle.make_cfg(wl)
    rng = np.random.default_rng(3)
    T = 64
    logits = rng.standard_normal((T, wl.n_experts)).astype(np.float32)
    _, bias = synth.make_router(wl.replace(hidden=16))
    ids, w, me, mg = oracle.route(cfg, logits, bias, T, margins=True)
    gs = wl.n_experts // wl.n_group
    for t in range(T):
        assert len(set(ids[t].tolist())) == wl.top_k
        assert len({int(e) // gs for e in ids[t]}) <= wl.topk_group
        assert (w[t] > 0).all()
        assert abs(float(w[t].astype(np.float64).sum()) - wl.routed_scaling) <= \
            wl.top_k * np.spacing(np.float32(wl.routed_scaling))
        assert me[t] >= 0 and mg[t] >= 0


def test_router_rejects_bad_config():
    with pytest.raises(ValueError):
        oracle.route(_cfg(n_experts=6, n_group=4), np.zeros((1, 6), np.float32),
                     np.zeros(6, np.float32), 1)
    with pytest.raises(ValueError):
        oracle.route(_cfg(n_experts=4, top_k=3, n_group=2, topk_group=1),
                     np.zeros((1, 4), np.float32), np.zeros(4, np.float32), 1)


# ------------------------------------------------------------------ grouping ---------------

@pytest.mark.parametrize("T,K,E", [(1, 8, 256), (4, 8, 256), (37, 4, 16), (2048, 8, 256),
                                   (0, 8, 256)])
def test_group_against_numpy(T, K, E):
    rng = np.random.default_rng(T)
    ids = rng.integers(0, E, size=(T, K)).astype(np.int32)
    counts, offsets, perm, uniq, nu = oracle.group(ids, T, K, E)
    flat = ids.reshape(-1)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    np.testing.assert_array_equal(perm, np.argsort(flat, kind="stable"))
    u = np.unique(flat)
    assert nu == len(u)
    np.testing.assert_array_equal(uniq[:nu], u)
    assert (uniq[nu:] == -1).all()


def test_group_rejects_bad_id():
    with pytest.raises(ValueError):
        oracle.group(np.array([[0, 5]], np.int32), 1, 2, 4)


# ------------------------------------------------------------------ expert FFN -------------

def _record_from_codes(H, I, fmt, parts):
    lay = synth.record_layout(H, I, fmt)
    rec = np.zeros(lay["stride"], np.uint8)
    for name, key in (("g", "wg"), ("u", "wu"), ("d", "wd")):
        q = torch.tensor(parts[name][0], dtype=torch.int8)
        b = synth.pack_codes(q, fmt).numpy().reshape(-1)
        rec[lay[key]:lay[key] + b.size] = b
    for name, key in (("g", "sg"), ("u", "su"), ("d", "sd")):
        s = np.asarray(parts[name][1], np.float32).view(np.uint8)
        rec[lay[key]:lay[key] + s.size] = s
    return rec


@pytest.mark.parametrize("fmt", [4, 8])
def test_expert_closed_form(fmt):
    g = json.load(open(os.path.join(GOLD, "expert_closed_form.json")))
    H, I = g["hidden"], g["inter"]
    parts = {"g": (g["wg_codes"], g["sg"]), "u": (g["wu_codes"], g["su"]),
             "d": (g["wd_codes"], g["sd"])}
    rec = _record_from_codes(H, I, fmt, parts)
    cfg = _cfg(hidden=H, inter=I, fmt=fmt)
    y = oracle.expert(cfg, rec, I, np.array(g["x"]))
    np.testing.assert_allclose(y, g["y"], rtol=0, atol=g["tol"])


def _np_expert(parts, x):
    """numpy float64 reference over the generator's codes x scales."""
    Wg = parts["g"][0].numpy().astype(np.float64) * parts["g"][1].numpy()[:, None]
    Wu = parts["u"][0].numpy().astype(np.float64) * parts["u"][1].numpy()[:, None]
    Wd = parts["d"][0].numpy().astype(np.float64) * parts["d"][1].numpy()[:, None]
    gg = Wg @ x
    a = gg / (1.0 + np.exp(-gg)) * (Wu @ x)
    return Wd @ a


@pytest.mark.parametrize("fmt", [4, 8, 2])
def test_expert_against_numpy(fmt):
    wl = synth.WORKLOADS["tiny"].replace(fmt=fmt)
    recs, codes = synth.make_expert_records(wl, experts=[5], keep_codes=True)
    cfg = oracle.make_cfg(wl)
    x = np.random.default_rng(1).standard_normal(wl.hidden)
    y = oracle.expert(cfg, recs[5], wl.inter, x)
    ref = _np_expert(codes[5], x)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15 * np.abs(ref).max())


def test_expert_special_cases():
    wl = synth.WORKLOADS["tiny"]
    cfg = oracle.make_cfg(wl)
    recs = synth.make_expert_records(wl, experts=[0])
    rec = recs[0].numpy().copy()
    lay = synth.record_layout(wl.hidden, wl.inter, 4)
    # zero activation -> SiLU(0) * 0 -> zero output
    assert (oracle.expert(cfg, rec, wl.inter, np.zeros(wl.hidden)) == 0).all()
    # zero up-projection scales -> u = 0 -> y = 0
    r2 = rec.copy()
    r2[lay["su"]:lay["sd"]] = 0
    x = np.random.default_rng(0).standard_normal(wl.hidden)
    assert (oracle.expert(cfg, r2, wl.inter, x) == 0).all()
    # doubling the down scales doubles y exactly (per-row scales factor out)
    r3 = rec.copy()
    sd = r3[lay["sd"]:lay["bytes"]].view(np.float32) * 2
    r3[lay["sd"]:lay["bytes"]] = sd.view(np.uint8)
    np.testing.assert_array_equal(oracle.expert(cfg, r3, wl.inter, x),
                                  2 * oracle.expert(cfg, rec, wl.inter, x))


# ------------------------------------------------------------------ gate and layer ---------

@pytest.mark.parametrize("name", ["tiny", "olmoe"])
def test_gate_against_numpy(name):
    wl = synth.WORKLOADS[name]
    Wr, _ = synth.make_router(wl)
    x = synth.make_activations(wl, 16)
    cfg = oracle.make_cfg(wl)
    lg = oracle.gate(cfg, Wr, x, 16)
    ref = (x.to(torch.float64).numpy() @ Wr.to(torch.float64).numpy().T).astype(np.float32)
    ulp = np.abs(lg.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1
    assert (ulp == 0).mean() > 0.99


@pytest.mark.parametrize("name", ["tiny", "olmoe"])
def test_layer_is_sum_of_parts(name):
    wl = synth.WORKLOADS[name]
    T = 3
    recs, codes = synth.make_expert_records(wl, keep_codes=True)
    sh, shc = synth.make_shared_record(wl, keep_codes=True)
    Wr, bias = synth.make_router(wl)
    x = synth.make_activations(wl, T)
    cfg = oracle.make_cfg(wl)
    R = oracle.Records(list(recs), sh)
    out, ids, w, _ = oracle.layer(cfg, Wr, bias, R, x, T)
    xs = x.to(torch.float64).numpy()
    for t in range(T):
        ref = np.zeros(wl.hidden)
        for k in range(wl.top_k):
            ref += float(w[t, k]) * _np_expert(codes[int(ids[t, k])], xs[t])
        if wl.n_shared:
            ref += _np_expert(shc, xs[t])
        np.testing.assert_allclose(out[t], ref, rtol=1e-11, atol=1e-13 * np.abs(ref).max())
    # batch-union visits each unique expert once and still gives the per-token result exactly
    np.testing.assert_array_equal(oracle.ffn(cfg, R, x, T, ids, w, union=True), out)


def test_layer_threads_do_not_change_result():
    wl = synth.WORKLOADS["tiny"]
    T = 8
    recs = synth.make_expert_records(wl)
    sh = synth.make_shared_record(wl)
    Wr, bias = synth.make_router(wl)
    x = synth.make_activations(wl, T)
    cfg = oracle.make_cfg(wl)
    R = oracle.Records(list(recs), sh)
    a = oracle.layer(cfg, Wr, bias, R, x, T, n_threads=1)[0]
    b = oracle.layer(cfg, Wr, bias, R, x, T, n_threads=4)[0]
    np.testing.assert_array_equal(a, b)


# ------------------------------------------------------------------------ residual update --

def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_residual_hand_worked_ties():
    """bf16 keeps 8 significant bits: at 1.0 its spacing is 2^-7, so 1 + 2^-8 is a tie that
    rounds to the even 1.0 (0x3f80) and 1 + 3*2^-8 one that rounds to 1 + 2^-6 (0x3f82);
    1 + 2^-8 + 2^-20 lies above the tie and rounds up to 0x3f81."""
    cfg = oracle.make_cfg(synth.WORKLOADS["olmoe"])
    x = _bf16_bits([1.0, 1.0, 1.0, -1.0, 0.0])
    out = np.array([2.0 ** -8, 3 * 2.0 ** -8, 2.0 ** -8 + 2.0 ** -20, -(2.0 ** -8), -0.0], np.float32)
    got = oracle.residual(cfg, x, out)
    assert [int(v) for v in got] == [0x3F80, 0x3F82, 0x3F81, 0xBF80, 0x0000]


def test_residual_against_torch_rounding():
    """numpy's IEEE float32 sum, rounded by torch's float32 -> bf16 conversion, on random values,
    exact ties, the overflow edge and NaN."""
    cfg = oracle.make_cfg(synth.WORKLOADS["olmoe"])
    rng = np.random.default_rng(5)
    n = 50000
    x = _bf16_bits(rng.normal(0, 1, n).astype(np.float32))
    out = (rng.normal(0, 1, n) * 10.0 ** rng.integers(-6, 3, n)).astype(np.float32)
    # exact ties: x = 0 and out with its low 16 bits 0x8000 (odd and even kept halves)
    ties = (rng.integers(0x3000, 0x4800, 2000).astype(np.uint32) << 16) | 0x8000
    x = np.concatenate([x, np.zeros(2000, np.uint16), _bf16_bits([3.3895313892515355e38, 1.0])])
    out = np.concatenate([out, ties.view(np.float32), np.array([1.0e36, np.nan], np.float32)])
    got = oracle.residual(cfg, x, out)
    xs = (x.astype(np.uint32) << 16).view(np.float32)
    s = (xs + out).astype(np.float32)
    want = torch.from_numpy(s).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    nan = np.isnan(s)
    np.testing.assert_array_equal(got[~nan], want[~nan])
    assert ((got[nan] & 0x7F80) == 0x7F80).all() and ((got[nan] & 0x7F) != 0).all()
    assert got[-2] == 0x7F80  # the largest bf16 plus 1e36 (past half a bf16 step there) rounds to +inf


def test_residual_f32_is_ieee_sum():
    cfg = oracle.make_cfg(synth.WORKLOADS["tiny"])
    rng = np.random.default_rng(6)
    x = rng.normal(0, 1, 4096).astype(np.float32)
    out = rng.normal(0, 1e-3, 4096).astype(np.float32)
    np.testing.assert_array_equal(oracle.residual(cfg, x, out), x + out)



# ------------------------------------------------------------------ group-scaled int4 -------
# The group-scaled container (one scale per 64 consecutive weights of a row; JustVugg/colibri
# README, "Get started -> 2. Get the model" recommends the gs64 GLM-5.2 build).

def test_record_bytes_gs64_glm():
    # codes as in the per-row container (18,874,368 B) + float32 scales: Wg and Wu 2048 rows x
    # 96 groups each, Wd 6144 rows x 32 groups -> 4 * (2 * 196,608 + 196,608) = 2,359,296 B
    assert oracle.record_bytes(6144, 2048, 4, 64) == 18_874_368 + 2_359_296 == 21_233_664
    assert synth.record_layout(6144, 2048, 4, 64)["bytes"] == 21_233_664
    with pytest.raises(ValueError):
        oracle.record_bytes(6144 + 32, 2048, 4, 64)  # a group must not straddle a row end


def _np_expert_grouped(parts, x, group):
    """numpy float64 reference over the generator's codes x group scales (each scale repeated
    over its `group` columns)."""
    def w(name):
        q, s = parts[name]
        return q.numpy().astype(np.float64) * np.repeat(s.numpy().astype(np.float64), group, axis=1)
    gg = w("g") @ x
    a = gg / (1.0 + np.exp(-gg)) * (w("u") @ x)
    return w("d") @ a


def test_expert_gs64_against_numpy():
    wl = synth.WORKLOADS["tiny"].replace(group=64)
    recs, codes = synth.make_expert_records(wl, experts=[3], keep_codes=True)
    assert codes[3]["g"][1].shape == (wl.inter, wl.hidden // 64)
    cfg = oracle.make_cfg(wl)
    x = np.random.default_rng(4).standard_normal(wl.hidden)
    y = oracle.expert(cfg, recs[3], wl.inter, x)
    ref = _np_expert_grouped(codes[3], x, 64)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15 * np.abs(ref).max())


def test_expert_gs64_with_equal_group_scales_is_the_per_row_expert():
    """A group-scaled record whose group scales all equal their row's scale dequantises to the
    same weights as the per-row record: the outputs agree bit for bit."""
    wl = synth.WORKLOADS["tiny"]
    H, I = wl.hidden, wl.inter
    recs, codes = synth.make_expert_records(wl, experts=[1], keep_codes=True)
    lay_r = synth.record_layout(H, I, 4)
    lay_g = synth.record_layout(H, I, 4, 64)
    rec_g = np.zeros(lay_g["stride"], np.uint8)
    rec_r = recs[1].numpy()
    rec_g[:lay_g["sg"]] = rec_r[:lay_r["sg"]]  # the codes are the same bytes
    for name, key, cols in (("g", "sg", H), ("u", "su", H), ("d", "sd", I)):
        s = np.repeat(codes[1][name][1].numpy()[:, None], cols // 64, axis=1).astype(np.float32)
        b = s.reshape(-1).view(np.uint8)
        rec_g[lay_g[key]:lay_g[key] + b.size] = b
    x = np.random.default_rng(5).standard_normal(H)
    y_r = oracle.expert(oracle.make_cfg(wl), rec_r, I, x)
    y_g = oracle.expert(oracle.make_cfg(wl.replace(group=64)), rec_g, I, x)
    np.testing.assert_array_equal(y_g, y_r)


def test_expert_gs64_group_scales_act_on_their_group_only():
    """Doubling one group's down-projection scale in every row changes y by exactly the part of
    the dot product that the group's 64 columns carry: y' - y equals y restricted to that group
    (computed with the other group's scales set to zero)."""
    wl = synth.WORKLOADS["tiny"].replace(group=64)   # inter 128: two groups per down row
    cfg = oracle.make_cfg(wl)
    recs = synth.make_expert_records(wl, experts=[2])
    rec = recs[2].numpy().copy()
    lay = synth.record_layout(wl.hidden, wl.inter, 4, 64)
    x = np.random.default_rng(6).standard_normal(wl.hidden)
    y = oracle.expert(cfg, rec, wl.inter, x)
    sd = rec[lay["sd"]:lay["bytes"]].view(np.float32).reshape(wl.hidden, 2)
    r_dbl = rec.copy()
    r_dbl[lay["sd"]:lay["bytes"]] = (sd * np.array([1.0, 2.0], np.float32)).reshape(-1).view(np.uint8)
    r_only = rec.copy()
    r_only[lay["sd"]:lay["bytes"]] = (sd * np.array([0.0, 1.0], np.float32)).reshape(-1).view(np.uint8)
    d = oracle.expert(cfg, r_dbl, wl.inter, x) - y
    np.testing.assert_allclose(d, oracle.expert(cfg, r_only, wl.inter, x), rtol=1e-12,
                               atol=1e-14 * np.abs(y).max())
