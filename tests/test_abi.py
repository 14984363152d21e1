"""The C-ABI library loads, exports every entry point its header declares, and
rejects bad arguments before touching a GPU (these tests run without one)."""
import ctypes
import glob
import os
import re

import pytest

from dynamic_expert_routing_router_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(beam_\w+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


def test_library_exports_every_declared_entry_point():
    names = _declared_functions()
    assert "beam_moe_forward" in names and "beam_moe_route" in names
    L = abi.lib()
    for n in names:
        assert hasattr(L, n), n


def test_status_and_stage_names():
    assert abi.status_str(0) == "BEAM_OK"
    assert abi.status_str(5) == "BEAM_ERR_TIMEOUT"
    assert [abi.stage_name(i) for i in range(abi.FORWARD_STAGES)] == [
        "router_gemm", "topk_mask", "permute", "gather", "gemm1_gate_up_swiglu",
        "gemm2_down", "combine"]
    assert abi.stage_name(abi.FORWARD_STAGES) is None


def test_plan_layout_is_consistent():
    for T in (0, 1, 8, 32, 128, 8192):
        dsc = abi.desc(T, 2048, 128, 768, 8, "bf16", 1)
        P = abi.plan(dsc)
        assert P["BN"] in (16, 32, 64, 128, 256)
        assert P["p_cap"] == T * 8 + 128 * (P["BN"] - 1)
        offs = [P[k] for k in ("off_counts", "off_hist", "off_partial", "off_idx", "off_w",
                               "off_pair", "off_pair_pos", "off_tiles", "off_xp", "off_h",
                               "off_y")]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        assert P["off_y"] + 2 * P["p_cap"] * 2048 <= P["workspace_bytes"]
        assert abi.workspace_size(dsc) == P["workspace_bytes"]
        assert (2048 // 64) % P["router_splits"] == 0
    assert abi.plan(abi.desc(8192, 2048, 128, 768, 8))["BN"] == 256
    assert abi.plan(abi.desc(2048, 2048, 128, 768, 8))["BN"] == 128
    assert abi.plan(abi.desc(8192, 2048, 128, 768, 8, "f32"))["BN"] == 128
    assert abi.plan(abi.desc(128, 2048, 128, 768, 8))["BN"] == 16


@pytest.mark.parametrize("bad,code", [
    (dict(K=0), 1), (dict(K=17, E=32), 1), (dict(E=300, K=8), 1), (dict(K=9, E=8), 1),
    (dict(dtype=7), 1), (dict(renorm=2), 1), (dict(T=-1), 1),
    (dict(d=2000), 2), (dict(I=700), 2),
])
def test_bad_descriptors_are_rejected(bad, code):
    args = dict(T=4, d=2048, E=128, I=768, K=8, dtype="bf16", renorm=1)
    args.update(bad)
    dsc = abi.desc(**args)
    assert abi.workspace_size(dsc) == 0
    with pytest.raises(abi.BeamError) as ei:
        abi.plan(dsc)
    assert ei.value.status == code


def test_f32_shape_rule():
    assert abi.workspace_size(abi.desc(4, 128, 8, 256, 2, "f32", 0)) > 0
    assert abi.workspace_size(abi.desc(4, 132, 8, 256, 2, "f32", 0)) == 0  # d % 8


def _call_forward(dsc, ptrs, ws_bytes):
    L = abi.lib()
    vp = ctypes.c_void_p
    return L.beam_moe_forward(ctypes.byref(dsc), *[vp(p) if p else None for p in ptrs],
                              ctypes.c_size_t(ws_bytes), None)


def test_argument_errors_return_before_any_launch():
    dsc = abi.desc(4, 2048, 128, 768, 8, "bf16", 1)
    need = abi.workspace_size(dsc)
    good = [4096 * (i + 1) for i in range(8)]  # x Wg Wm W1 W3 W2 out ws (never dereferenced)
    # NULL weight
    p = list(good)
    p[3] = 0
    assert _call_forward(dsc, p, need) == 1
    # misaligned x
    p = list(good)
    p[0] += 8
    assert _call_forward(dsc, p, need) == 1
    # workspace too small, NULL, misaligned
    assert _call_forward(dsc, good, need - 1) == 3
    p = list(good)
    p[7] = 0
    assert _call_forward(dsc, p, need) == 3
    p = list(good)
    p[7] += 16
    assert _call_forward(dsc, p, need) == 3


def test_kernel_count_per_path():
    assert abi.kernel_count(abi.desc(128, 2048, 128, 768, 8, "bf16", 1)) == 5  # fused, no gather
    # prefill and fp32: the grouping in two launches (per-chunk counts, placement)
    assert abi.kernel_count(abi.desc(8192, 2048, 128, 768, 8, "bf16", 1)) == 8
    assert abi.kernel_count(abi.desc(64, 128, 8, 256, 2, "f32", 0)) == 8
    assert abi.kernel_count(abi.desc(0, 2048, 128, 768, 8, "bf16", 1)) == 0
    assert abi.kernel_count(abi.desc(4, 2000, 128, 768, 8, "bf16", 1)) == 0


def test_one_launch_path_selection():
    """bf16 batches of at most 16 tokens whose token rows, logits and weight
    stages fit one CTA's shared memory can run the whole layer as one kernel
    (by default up to 4 tokens: beam_moe_set_one_launch_tokens); the router of
    every bf16 call at those sizes then runs unsplit (one partial)."""
    prev = abi.set_one_launch_tokens(16)
    try:
        for T in (1, 8, 16):
            dsc = abi.desc(T, 2048, 128, 768, 8, "bf16", 1)
            P = abi.plan(dsc)
            assert P["one_launch"] == 1 and abi.kernel_count(dsc) == 1
            assert P["router_splits"] == 1
            # counters: one per (expert, 128 columns of H), one per (token, 16
            # columns of the output)
            assert P["off_ctl"] + 4 * (128 * 6 + T * 2048 // 16) <= P["workspace_bytes"]
            assert P["off_ctl"] >= P["off_tiles_sub"] and P["off_ctl"] % 256 == 0
        big = abi.plan(abi.desc(17, 2048, 128, 768, 8, "bf16", 1))
        assert big["one_launch"] == 0 and big["off_ctl"] + 0 <= big["workspace_bytes"]
        assert abi.kernel_count(abi.desc(17, 2048, 128, 768, 8, "bf16", 1)) == 5
        # d = 7168, E = 256: one token fits, sixteen do not (their rows take 224 KB)
        assert abi.plan(abi.desc(1, 7168, 256, 2048, 8, "bf16", 0))["one_launch"] == 1
        assert abi.plan(abi.desc(16, 7168, 256, 2048, 8, "bf16", 0))["one_launch"] == 0
        # the switch: 0 turns the path off; the default takes up to 4 tokens
        abi.set_one_launch_tokens(0)
        assert abi.plan(abi.desc(1, 2048, 128, 768, 8, "bf16", 1))["one_launch"] == 0
        assert abi.plan(abi.desc(1, 2048, 128, 768, 8, "bf16", 1))["router_splits"] == 1
        abi.set_one_launch_tokens(4)
        assert abi.plan(abi.desc(4, 2048, 128, 768, 8, "bf16", 1))["one_launch"] == 1
        assert abi.plan(abi.desc(5, 2048, 128, 768, 8, "bf16", 1))["one_launch"] == 0
        assert abi.set_one_launch_tokens(99) == 4 and abi.set_one_launch_tokens(4) == 16
    finally:
        abi.set_one_launch_tokens(prev)
    # fp32, shared experts and the backward's plan keep the multi-kernel path
    assert abi.plan(abi.desc(4, 128, 8, 256, 2, "f32", 0))["one_launch"] == 0
    sh = abi.desc(4, 2048, 64, 1408, 6, "bf16", 1, n_shared=2, I_shared=1408)
    assert abi.plan(sh)["one_launch"] == 0 and abi.plan(sh)["router_splits"] == 1


def test_nan_mask_threshold_is_rejected():
    dsc = abi.desc(4, 2048, 128, 768, 8, "bf16", 1)
    dsc.mask_logit_threshold = float("nan")
    assert abi.workspace_size(dsc) == 0
    assert abi.tau_logit(0.5) == 0.0 and abi.tau_logit(0.9) > 2.19


def test_shared_expert_descriptor_rules():
    ok = abi.desc(64, 2048, 64, 1408, 6, "bf16", 1, n_shared=2, I_shared=1408)
    P = abi.plan(ok)
    assert P["off_ys"] > P["off_hs"] > P["off_tile_done"]
    # one token tile of 64 rows; the gate/up reduction (32 k-blocks) split 4
    # ways over 22 units, the down reduction (22 k-blocks) 3 ways over 32 units
    # (about half the SMs): gate/up GEMM, SwiGLU of the partials, down GEMM
    assert (P["sh_bn"], P["sh_split1"], P["sh_split2"]) == (64, 4, 3)
    assert P["off_sp"] + 4 * 2 * 4 * 2 * 64 * 1408 <= P["workspace_bytes"]
    assert P["off_tiles_sub"] >= P["off_ys"] + 4 * 3 * 2 * 64 * 2048
    assert abi.kernel_count(ok) == abi.kernel_count(abi.desc(64, 2048, 64, 1408, 6)) + 3
    big = abi.plan(abi.desc(8192, 2048, 64, 1408, 6, "bf16", 1, n_shared=2, I_shared=1408))
    assert (big["sh_bn"], big["sh_split1"], big["sh_split2"]) == (128, 1, 1)
    for bad, code in ((dict(n_shared=17, I_shared=128), 1), (dict(n_shared=2, I_shared=0), 1),
                      (dict(n_shared=2, I_shared=100), 2), (dict(n_shared=-1), 1)):
        with pytest.raises(abi.BeamError) as ei:
            abi.plan(abi.desc(8, 2048, 64, 1408, 6, "bf16", 1, **bad))
        assert ei.value.status == code
    with pytest.raises(abi.BeamError):
        abi.plan(abi.desc(8, 128, 8, 256, 2, "f32", 0, n_shared=1, I_shared=256))
    # beam_moe_forward refuses a descriptor with shared experts before any launch
    L = abi.lib()
    vp = ctypes.c_void_p
    ptrs = [vp(4096 * (i + 1)) for i in range(8)]
    assert L.beam_moe_forward(ctypes.byref(ok), *ptrs, ctypes.c_size_t(1 << 40), None) == 1


def test_backward_split_limit_applies_to_fp32_only():
    """The CUDA-core kept-row products (fp32) hold a split of their A rows in
    shared memory, so an fp32 layer with d > 7168 at 128-token tiles has no
    backward; the bf16 layer runs them on the tensor cores and has one."""
    big_bf16 = abi.desc(1024, 8192, 8, 256, 2, "bf16", 1)
    big_f32 = abi.desc(1024, 8192, 8, 256, 2, "f32", 1)
    assert abi.plan(big_bf16)["BN"] in (128, 256) and abi.workspace_size(big_f32) > 0
    assert abi.backward_workspace_size(big_bf16) > abi.workspace_size(big_bf16)
    assert abi.backward_kernel_count(big_bf16) == 15
    assert abi.backward_workspace_size(big_f32) == 0
    assert abi.backward_kernel_count(big_f32) == 0


def test_backward_descriptor_and_argument_checks():
    dsc = abi.desc(8, 2048, 128, 768, 8, "bf16", 1)
    assert abi.backward_workspace_size(dsc) > abi.workspace_size(dsc)
    assert abi.backward_kernel_count(dsc) == 15  # bf16: dy W2 on the tensor cores
    assert abi.backward_kernel_count(abi.desc(8, 128, 8, 256, 2, "f32", 0)) == 14
    assert abi.backward_kernel_count(abi.desc(0, 2048, 128, 768, 8, "bf16", 1)) == 0
    shared = abi.desc(8, 2048, 64, 1408, 6, "bf16", 1, n_shared=2, I_shared=1408)
    assert abi.backward_workspace_size(shared) == 0  # shared experts: forward only
    L = abi.lib()
    p = [ctypes.c_void_p(4096 * (i + 1)) for i in range(13)]
    big = ctypes.c_size_t(1 << 40)

    def call(desc, beta, dWm):
        return L.beam_moe_backward(ctypes.byref(desc), p[0], p[1], p[2], p[3], p[4], p[5], p[6],
                                   ctypes.c_float(beta), p[7], p[8], dWm, p[9], p[10], p[11],
                                   p[12], big, None)
    assert call(dsc, 0.1, None) == 1            # W_mask given, dW_mask missing
    assert call(dsc, float("nan"), p[0]) == 1   # beta must be finite
    assert call(shared, 0.1, p[0]) == 2         # unsupported: shared experts


def test_tau_to_logit_behind_the_abi():
    """beam_moe_tau_to_logit: ln(tau / (1 - tau)) rounded once to float32; the
    paper's tau = 0.5 is exactly 0 (sigmoid(0) = 1/2)."""
    import math

    import numpy as np
    f = abi.lib().beam_moe_tau_to_logit
    assert f(0.5) == 0.0
    for tau in (0.1, 0.3, 0.7, 0.9):
        t = float(np.float32(tau))  # the value the float argument carries
        assert f(tau) == float(np.float32(math.log(t / (1.0 - t))))
        assert f(tau) == -f(float(np.float32(1.0 - t))) or abs(f(tau) + f(1.0 - t)) < 1e-6
    assert f(0.0) == -math.inf and f(1.0) == math.inf
    for bad in (-0.1, 1.5, float("nan")):
        assert math.isnan(f(bad))
    assert abi.desc(4, 2048, 128, 768, 8, tau=0.3).mask_logit_threshold == f(0.3)


def test_fault_injection_switch_checks_its_mode():
    with pytest.raises(abi.BeamError) as ei:
        abi.set_fault_injection(7)
    assert ei.value.status == 1
    abi.set_fault_injection(abi.FAULT_NONE, 0)  # the default, idempotent
