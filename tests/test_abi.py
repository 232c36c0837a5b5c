"""The C-ABI library loads, exports every entry point include/coli_moe.h declares, and
validates arguments on the host before touching the GPU (CPU only: no compute calls)."""
import ctypes
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "coli_moe.h")

q = pytest.importorskip("quantized_routed_expert_noaux_b200")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(coli_moe_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    syms = declared_symbols()
    assert len(syms) >= 10
    lib = ctypes.CDLL(q.LIB_PATH)
    missing = [s for s in syms if not hasattr(lib, s)]
    assert not missing, missing


def test_binding_names_match_header():
    for s in declared_symbols():
        assert hasattr(q, s), f"binding lacks {s}"
        assert s in q.__all__, f"{s} missing from __all__"


def test_status_strings():
    assert q.coli_moe_status_str(0) == "ok"
    assert "workspace" in q.coli_moe_status_str(7)
    assert q.coli_moe_status_str(99) == "unknown status"


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_workload_configs_are_accepted(name):
    wl = synth.WORKLOADS[name]
    cfg = q.config_for(wl)
    q.coli_moe_check_config(cfg)
    assert q.coli_moe_record_bytes(wl.hidden, wl.inter, wl.fmt, wl.group) == \
        synth.record_layout(wl.hidden, wl.inter, wl.fmt, wl.group)["bytes"]
    assert q.coli_moe_workspace_size(cfg, 64) % 256 == 0


@pytest.mark.parametrize("field,value,status", [
    ("wfmt", 3, 1), ("act", 5, 1), ("group_size", 32, 1), ("group_size", -64, 1), ("n_group", 3, 2), ("topk_group", 9, 2),
    ("top_k", 33, 4), ("top_k", 200, 2), ("hidden", 100, 2), ("n_shared", 2, 4), ("n_experts", 2048, 4), ("n_experts", 250, 2),
    ("shared_inter", 1024, 4), ("routed_scaling", 0.0, 1),
])
def test_bad_config_rejected(field, value, status):
    cfg = q.config_for(synth.WORKLOADS["glm_decode"])
    setattr(cfg, field, value)
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_check_config(cfg)
    assert ei.value.status == status


def test_host_validation_before_launch():
    cfg = q.config_for(synth.WORKLOADS["tiny"])
    # T = 0 is a no-op and negative T a shape error: both decided without a device
    q.coli_moe_gate(cfg, None, None, 0, None, stream=0)
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_gate(cfg, None, None, -1, None, stream=0)
    assert ei.value.status == 2
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_gate(cfg, None, None, 3, None, stream=0)
    assert ei.value.status == 1
    # misaligned activation pointer
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_gate(cfg, 256, 258, 3, 512, stream=0)
    assert ei.value.status == 3
    # layer without a workspace
    w = q.MoEWeights(256, 512, 1024, 51200, 2048)
    rc = q.lib.coli_moe_layer(ctypes.byref(cfg), ctypes.byref(w), 4096, 2, 8192, None, None,
                              None, 0, None)
    assert rc == 7
    # misaligned record stride
    w.expert_stride = 51200 + 16
    rc = q.lib.coli_moe_layer(ctypes.byref(cfg), ctypes.byref(w), 4096, 2, 8192, None, None,
                              None, 0, None)
    assert rc == 3
    # stride smaller than a record
    w.expert_stride = 256
    rc = q.lib.coli_moe_layer(ctypes.byref(cfg), ctypes.byref(w), 4096, 2, 8192, None, None,
                              None, 0, None)
    assert rc == 2


def test_residual_host_validation():
    cfg = q.config_for(synth.WORKLOADS["olmoe"])
    q.coli_moe_residual(cfg, None, None, 0, None, stream=0)  # T = 0: no-op
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_residual(cfg, None, None, -1, None, stream=0)
    assert ei.value.status == 2
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_residual(cfg, None, 256, 2, 512, stream=0)
    assert ei.value.status == 1
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_residual(cfg, 264, 256, 2, 512, stream=0)  # x not 16-byte aligned
    assert ei.value.status == 3



def test_dispatch_rule_on_the_host():
    """Batches above 4 tokens take the tensor-core path (7 launches) for per-row int4, int8 and
    int2 records whose hidden and inter sizes are multiples of 128; group-scaled records and
    other sizes take the GEMV path (5); an empty batch launches nothing.  (Up to 4 tokens the
    fused decode kernel needs the device's shared-memory size, so that choice is checked by the
    GPU tests.)"""
    for name in ("tiny", "olmoe", "glm_decode", "glm_prefill"):
        cfg = q.config_for(synth.WORKLOADS[name])
        assert q.coli_moe_layer_kernels(cfg, 0) == 0
        for T in (5, 8, 64, 65, 2048):
            assert q.coli_moe_layer_kernels(cfg, T) == 7, (name, T)
    for name in ("glm_int8", "glm_int2"):  # int8 and int2 records take the tensor-core path too
        cfg = q.config_for(synth.WORKLOADS[name])
        for T in (5, 64, 256):
            assert q.coli_moe_layer_kernels(cfg, T) == 7, (name, T)
    gs = q.config_for(synth.WORKLOADS["glm_gs64"])  # group scales: the GEMV path above 4 tokens
    assert q.coli_moe_layer_kernels(gs, 64) == 5
    odd = q.config_for(synth.WORKLOADS["tiny"].replace(inter=64, shared_inter=64))
    assert q.coli_moe_layer_kernels(odd, 32) == 5  # inter not a multiple of 128


def test_per_expert_dispatch_threshold():
    """The threshold is process-wide, defaults to 0 (every expert on the grouped GEMM), and a
    positive value adds the two GEMV launches to the tensor-core path's count; negative values
    are rejected."""
    assert q.coli_moe_dispatch_threshold() == 0
    cfg = q.config_for(synth.WORKLOADS["glm_prefill"])
    try:
        q.coli_moe_set_dispatch_threshold(4)
        assert q.coli_moe_dispatch_threshold() == 4
        assert q.coli_moe_layer_kernels(cfg, 2048) == 9
        assert q.coli_moe_layer_kernels(cfg, 0) == 0
        with pytest.raises(q.ColiError):
            q.coli_moe_set_dispatch_threshold(-1)
        assert q.coli_moe_dispatch_threshold() == 4
    finally:
        q.coli_moe_set_dispatch_threshold(0)
    assert q.coli_moe_layer_kernels(cfg, 2048) == 7


def test_noalloc_error_word_rejects_null_code():
    """The static array's error-word accessor checks its output pointer before touching the
    device (status 1, COLI_ERR_INVALID_ARG)."""
    assert q.lib.coli_moe_noalloc_error_word(None, None) == 1


def test_group_scaled_container_is_int4_only():
    wl = synth.WORKLOADS["glm_int8"].replace(group=64)
    with pytest.raises(q.ColiError) as ei:
        q.coli_moe_check_config(q.config_for(wl))
    assert ei.value.status == 4
    with pytest.raises(q.ColiError):
        q.coli_moe_record_bytes(6144, 2048, 8, 64)
    assert q.coli_moe_record_bytes(6144, 2048, 4, 64) == 21_233_664
