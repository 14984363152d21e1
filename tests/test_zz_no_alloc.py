"""beam_moe_route_noalloc: routing for callers that cannot allocate device
memory -- for example code running inside a CUDA-graph capture, where
cudaMalloc is illegal, or a plugin whose host runtime owns all device memory.
Its scratch is a fixed array inside the library instead of a caller
workspace.  Checked against beam_moe_route (which takes a workspace) on two
calls in a row with different batches, so the second call runs over the
first call's leftover scratch contents.  This file is collected last.
"""
import numpy as np
import pytest
import torch

from dynamic_expert_routing_router_b200 import abi, inputs

pytestmark = pytest.mark.gpu


def _outputs(T, E, K, dev):
    return (torch.empty((T, K), dtype=torch.int32, device=dev),
            torch.empty((T, K), dtype=torch.float32, device=dev),
            torch.empty((E,), dtype=torch.int32, device=dev),
            torch.empty((K + 1,), dtype=torch.int32, device=dev),
            torch.full((T, 2 * E), float("nan"), dtype=torch.float32, device=dev))


def test_route_noalloc_matches_route_on_two_calls():
    dev = "cuda"
    sh = inputs.QWEN3
    Wg = inputs.make_gate(sh, seed=0, device=dev)
    for T, f, seed in ((128, 0.15, 1), (37, 0.6, 2)):  # second call smaller, other data
        x = inputs.make_tokens(sh, T, seed=seed, device=dev)
        Wm = inputs.make_mask(sh, f, seed=0, device=dev)
        dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
        ref = _outputs(T, sh.E, sh.K, dev)
        ws = abi.alloc_workspace(dsc, dev)
        abi.route(dsc, x, Wg, Wm, *ref, workspace=ws)
        got = _outputs(T, sh.E, sh.K, dev)
        abi.route_noalloc(dsc, x, Wg, Wm, *got)
        torch.cuda.synchronize()
        r = [t.cpu().numpy() for t in ref]
        g = [t.cpu().numpy() for t in got]
        assert np.array_equal(g[0], r[0])  # candidates and mask: bit-exact
        assert np.array_equal(g[2], r[2]) and np.array_equal(g[3], r[3])
        np.testing.assert_allclose(g[1], r[1], rtol=2e-6, atol=1e-7)
        np.testing.assert_allclose(g[4], r[4], rtol=0, atol=1e-5)
        assert g[3].sum() == T and (g[0] >= 0).sum() == g[2].sum()


def test_route_noalloc_rejects_batches_beyond_its_array():
    dev = "cuda"
    sh = inputs.QWEN3
    T = 20000  # the router partials alone need ~20 MB > 16 MiB
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    assert abi.plan(dsc)["off_idx"] > abi.NOALLOC_SCRATCH_BYTES
    small = torch.zeros(64, dtype=torch.float32, device=dev)  # never read: rejected first
    with pytest.raises(abi.BeamError) as ei:
        abi.route_noalloc(dsc, small, small, small, small, small, small, small, small)
    assert ei.value.status == 3  # BEAM_ERR_WORKSPACE
