"""GPU parity of the residual update and of chained layers (int8 / int2 records, 64 tokens, four
layers): x_{l+1} = bf16(x_l + out_l) on the device between the layers.

The residual update is compared bit for bit with the oracle.  Each layer is compared with the
oracle fed the device's own input (teacher forcing): routing bit-exact on sampled tokens, the
output within the tolerance of the path it takes.  The oracle also runs the chain on its own from
the first input for two tokens; that end-to-end difference is printed, not gated.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._common import Layer, normwise_err, oracle_layer_tokens, tol_for

pytestmark = pytest.mark.gpu

q = pytest.importorskip("quantized_routed_expert_noaux_b200")


def _bits(t):
    """bf16 tensor -> uint16 bit patterns (numpy); float32 passes through."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def _from_bits(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
    return torch.from_numpy(a.copy())


@pytest.mark.parametrize("name,T", [("olmoe", 37), ("tiny", 9), ("glm_decode", 64)])
def test_residual_matches_oracle_bitwise(name, T):
    wl = synth.WORKLOADS[name]
    cfg, ocfg = q.config_for(wl), oracle.make_cfg(wl)
    x = synth.make_activations(wl, T, device="cuda", step=40)
    out = synth.make_activations(wl.replace(act="f32"), T, device="cuda", step=41) * 0.05
    if wl.act == "bf16":
        # hand-picked rounding cases in the first row: ties to even both ways, above a tie,
        # the overflow edge (largest bf16 + 1e36 -> +inf), a NaN
        xs = torch.tensor([1.0, 1.0, 1.0, 3.3895313892515355e38, 2.0], dtype=torch.bfloat16)
        os_ = torch.tensor([2.0 ** -8, 3 * 2.0 ** -8, 2.0 ** -8 + 2.0 ** -20, 1.0e36, float("nan")])
        x[0, :5] = xs.cuda()
        out[0, :5] = os_.cuda()
    x_next = torch.empty_like(x)
    q.coli_moe_residual(cfg, x, out, T, x_next)
    torch.cuda.synchronize()
    want = oracle.residual(ocfg, x.cpu(), out.cpu())
    got = _bits(x_next)
    if wl.act == "bf16":
        nan = ((want & 0x7F80) == 0x7F80) & ((want & 0x7F) != 0)
        np.testing.assert_array_equal(got[~nan], want[~nan])
        assert (((got[nan] & 0x7F80) == 0x7F80) & ((got[nan] & 0x7F) != 0)).all()
        assert [int(v) for v in got[0, :4]] == [0x3F80, 0x3F82, 0x3F81, 0x7F80]
    else:
        np.testing.assert_array_equal(got, want)
    # in place (x_next = x) gives the same bits
    xi = x.clone()
    q.coli_moe_residual(cfg, xi, out, T, xi)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_bits(xi), got)


@pytest.mark.parametrize("name", ["glm_int8", "glm_int2"])
def test_chained_layers_teacher_forced(name):
    wl = synth.WORKLOADS[name]
    T = 64
    cfg, ocfg = q.config_for(wl), oracle.make_cfg(wl)
    toks = [0, 21, 63]
    chain_toks = [5, 40]
    x = synth.make_activations(wl, T, device="cuda", step=9)
    x_own = x.cpu()[chain_toks]  # the oracle's own chain, from the same first input
    ws = torch.empty(q.coli_moe_workspace_size(cfg, T), dtype=torch.uint8, device="cuda")
    flips = 0
    for layer in range(wl.n_layers):
        L = Layer(wl, "cuda", layer)
        out = torch.empty(T, wl.hidden, dtype=torch.float32, device="cuda")
        ids = torch.empty(T, wl.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, wl.top_k, dtype=torch.float32, device="cuda")
        q.coli_moe_clear_error(ws)
        q.coli_moe_layer(cfg, L.weights(), x, T, out, ids, w, ws)
        assert q.coli_moe_error_word(ws) == 0
        # teacher forcing: the oracle takes the device's input of this layer
        ref, ids_ref, w_ref, _ = oracle_layer_tokens(L, x.cpu(), toks)
        np.testing.assert_array_equal(ids.cpu().numpy()[toks], ids_ref)
        np.testing.assert_array_equal(w.cpu().numpy()[toks], w_ref)
        err = normwise_err(out.cpu().numpy()[toks], ref)
        assert err <= tol_for(q, cfg, T), (layer, err)
        x_next = torch.empty_like(x)
        q.coli_moe_residual(cfg, x, out, T, x_next)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_bits(x_next), oracle.residual(ocfg, x.cpu(), out.cpu()))
        # the oracle's own chain
        own, ids_own, _, _ = oracle_layer_tokens(L, x_own, range(len(chain_toks)))
        flips += int((np.sort(ids_own, axis=1) != np.sort(ids.cpu().numpy()[chain_toks], axis=1)).any(axis=1).sum())
        x_own = _from_bits(oracle.residual(ocfg, x_own, own.astype(np.float32)))
        x = x_next
        del L
        torch.cuda.empty_cache()
    end = normwise_err(x.cpu()[chain_toks].float().numpy(), x_own.float().numpy())
    print(f"{name}: {wl.n_layers} chained layers, end-to-end normwise difference {end:.2e} on "
          f"tokens {chain_toks}, routing differences along the chain: {flips}")
