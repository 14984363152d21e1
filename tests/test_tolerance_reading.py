"""Why the bf16 value bar is read per token and net of the output's rounding.

The stated bar is max-abs-error <= 2e-2 x RMS(ref output).  Here the exact
fp64 oracle output of a Qwen3-shaped layer (d=2048, I=768, top-8, 16 experts
to keep the CPU run short) is simply rounded to bf16 -- the best any bf16
output can be -- and the literal batch-wide reading already fails, while the
adopted reading (per token, net of half an ulp) leaves the whole 2e-2 budget
to the computation.  CPU only.
"""
import numpy as np
import torch

import oracle
from dynamic_expert_routing_router_b200 import inputs

from _parity import BF16_TOL_RMS, bf16_excess


def test_rounding_the_exact_result_breaks_the_literal_bar():
    sh = inputs.Shape(d=2048, E=16, K=8, I=768, renorm=1, dtype="bf16")
    x = inputs.make_tokens(sh, 64, seed=5)
    Wg = inputs.make_gate(sh, seed=0)
    Wm = inputs.make_mask(sh, 0.35, seed=0)
    W1, W3, W2 = inputs.make_experts(sh, seed=0)
    h = [inputs.host_array(t) for t in (x, Wg, Wm, W1, W3, W2)]
    y, rt, _, _ = oracle.forward(*h, sh.K, sh.renorm, "bf16")
    act = (rt["idx"] >= 0).any(axis=1)
    ya = y[act]
    yb = torch.as_tensor(ya).to(torch.bfloat16).double().numpy()  # ideal bf16 output
    literal = np.abs(yb - ya).max() / np.sqrt((ya ** 2).mean())
    assert literal > BF16_TOL_RMS  # no bf16 output can meet the literal reading
    # adopted reading: the rounding costs nothing (up to the fp64->fp32->bf16
    # double rounding of the conversion, ~1e-8)
    assert bf16_excess(yb, ya).max() <= 1e-6
