"""Expert parallelism on one GPU: G ranks emulated in one process.

Each emulated rank owns E/G experts and routes its own token batch through
the library's kernels (route, dispatch, expert rows, combine).  The exchange
between ranks is a device copy that moves the same row chunks an all-to-all
would move (chunk j of rank s's send buffer lands, in source-rank order, in
rank j's receive buffer), so no kernel ever waits for another rank.  The
collective itself is covered on CPU with gloo (test_dist_gloo_ep.py).

Checked per rank: the dispatch lists exactly the kept pairs in the oracle's
permutation order with the right split sizes, local expert ids and token
rows (bit for bit); the reassembled output matches the oracle at the bf16
bar; and it equals the one-GPU layer on the same tokens bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_expert_routing_router_b200 import abi, ep, inputs

from _parity import assert_values, host, oracle_from_logits, report

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _a2a(chunks_by_src, splits_by_src):
    """Emulated all-to-all: rank j receives, from every source s in order,
    rows [sum(splits_s[:j]), + splits_s[j]) of source s's buffer."""
    G = len(chunks_by_src)
    recv = []
    for j in range(G):
        parts = []
        for s in range(G):
            o = sum(splits_by_src[s][:j])
            parts.append(chunks_by_src[s][o:o + splits_by_src[s][j]])
        recv.append(torch.cat(parts, 0))
    return recv


def _run_ep(sh, G, Ts, f, seed=0):
    E = sh.E
    El = E // G
    Wg = inputs.make_gate(sh, seed=seed, device=DEV)
    Wm = inputs.make_mask(sh, f, seed=seed, device=DEV) if f is not None else None
    W1, W3, W2 = inputs.make_experts(sh, seed=seed, device=DEV)
    layers = [ep.ExpertParallelLayer(Ts[r], sh.d, E, sh.I, sh.K, sh.renorm, r, G, Wg, Wm,
                                     W1[r * El:(r + 1) * El], W3[r * El:(r + 1) * El],
                                     W2[r * El:(r + 1) * El]) for r in range(G)]
    xs = [inputs.make_tokens(sh, Ts[r], seed=900 + r, device=DEV) for r in range(G)]
    disp = [layers[r].dispatch(xs[r]) for r in range(G)]
    splits = [d.send_splits for d in disp]
    recv_rows = _a2a([d.send_rows for d in disp], splits)
    recv_exp = _a2a([d.send_expert for d in disp], splits)
    recv_splits = [[splits[s][j] for s in range(G)] for j in range(G)]
    y_recv = [layers[j].local_experts(recv_rows[j], recv_exp[j]) for j in range(G)]
    y_back = _a2a(y_recv, recv_splits)
    outs = []
    for r in range(G):
        out = torch.empty((Ts[r], sh.d), dtype=torch.bfloat16, device=DEV)
        layers[r].combine(disp[r], y_back[r], out)
        layers[r].check()
        outs.append(out)
    torch.cuda.synchronize()
    return dict(Wg=Wg, Wm=Wm, W=(W1, W3, W2), xs=xs, disp=disp, outs=outs, layers=layers)


EP_CASES = [
    # (name, shape, G, tokens per rank, kept fraction)
    ("qwen3_G2_decode", inputs.QWEN3, 2, [32, 17], 0.35),
    ("qwen3_G4_decode", inputs.QWEN3, 4, [64, 1, 33, 8], 0.15),
    ("qwen3_G8_prefill_tiles", inputs.QWEN3, 8, [2048, 1500, 96, 0, 7, 300, 2100, 64], 0.35),
    ("qwen15_E60_G4", inputs.QWEN15_MOE, 4, [40, 9, 0, 23], 0.5),
    ("qwen3_G4_unmasked", inputs.QWEN3, 4, [16, 16, 16, 16], None),
    ("qwen3_G2_all_masked", inputs.QWEN3, 2, [16, 8], 0.0),
]


@pytest.mark.parametrize("name,sh,G,Ts,f", EP_CASES, ids=[c[0] for c in EP_CASES])
def test_expert_parallel_matches_oracle_and_one_gpu(name, sh, G, Ts, f):
    R = _run_ep(sh, G, Ts, f)
    E, K, El = sh.E, sh.K, sh.E // G
    W1, W3, W2 = R["W"]
    h1, h3, h2 = (host(W) for W in R["W"])
    sent = kept_total = 0
    for r in range(G):
        T = Ts[r]
        d = R["disp"][r]
        x = R["xs"][r]
        idx = d.idx.cpu().numpy()
        # routing as the one-GPU layer takes it (oracle fed the same logits)
        lg = torch.empty((T, 2 * E), dtype=torch.float32, device=DEV)
        dsc = abi.desc(T, sh.d, E, sh.I, K, "bf16", sh.renorm)
        if T:
            ws = abi.alloc_workspace(dsc, DEV)
            i2 = torch.empty((T, K), dtype=torch.int32, device=DEV)
            w2 = torch.empty((T, K), dtype=torch.float32, device=DEV)
            c2 = torch.empty((E,), dtype=torch.int32, device=DEV)
            abi.route(dsc, x, R["Wg"], R["Wm"], i2, w2, c2, None, lg, ws)
            o = oracle_from_logits(lg.cpu().numpy(), E, K, sh.renorm, R["Wm"] is not None)
            assert np.array_equal(o["idx"], idx)
        # dispatch: kept pairs in the oracle's permutation order, split by rank
        offsets, pairs = oracle.permutation(idx, E)
        P = len(pairs)
        assert d.send_splits == [int(offsets[(j + 1) * El] - offsets[j * El]) for j in range(G)]
        assert np.array_equal(d.send_pair.cpu().numpy(), pairs)
        assert np.array_equal(d.send_expert.cpu().numpy(), idx.reshape(-1)[pairs] % El)
        if P:
            assert torch.equal(d.send_rows, x[torch.as_tensor(pairs // K, device=DEV)])
            pos = d.pair_pos.cpu().numpy().reshape(-1)
            assert np.array_equal(pos[pairs], np.arange(P))
        sent += P
        kept_total += int((idx >= 0).sum())
        out = R["outs"][r]
        if T == 0:
            continue
        # values: oracle at the bf16 bar, every token
        ref = oracle.experts(host(x), h1, h3, h2, idx, o["w"], "bf16")
        worst = assert_values(out, ref, idx, "bf16")
        # and the one-GPU layer on the same tokens, on the multi-kernel path
        # (the one the expert-parallel steps distribute; the one-launch path
        # of small batches computes the same values in another order)
        one = torch.empty_like(out)
        prev = abi.set_one_launch_tokens(0)
        try:
            abi.forward(dsc, x, R["Wg"], R["Wm"], W1, W3, W2, one, ws)
        finally:
            abi.set_one_launch_tokens(prev)
        abi.check(dsc, ws)
        report(name=f"ep_{name}_rank{r}", kind="ep", T=T, worst_token_excess=worst,
               bitwise_equal_to_one_gpu=bool(torch.equal(out, one)),
               max_abs_diff_one_gpu=float((out.float() - one.float()).abs().max()))
        # the per-pair rows are the same tensor-core dot products in the same k
        # order (whatever the tile a row lands in), and the combine adds them
        # in the same slot order: bit for bit
        assert torch.equal(out, one)
    assert sent == kept_total  # only kept pairs crossed
    if f == 0.0:
        assert sent == 0 and all((o_.float() == 0).all() for o_ in R["outs"])


def test_expert_rows_entry_against_the_oracle():
    """beam_moe_expert_rows alone: ragged expert ids (with -1 rows) on 300
    rows of an 8-expert shard; fp32 rows vs the oracle's E_e(x)."""
    sh = inputs.QWEN3
    El, N = 8, 300
    W1, W3, W2 = (W[:El].contiguous() for W in inputs.make_experts(sh, seed=4, device=DEV))
    x = inputs.make_tokens(sh, N, seed=4, device=DEV)
    g = torch.Generator(device="cpu").manual_seed(4)
    eid = torch.randint(-1, El, (N,), generator=g).to(torch.int32)
    eid[:40] = 3  # one hot expert spanning several tiles
    dsc = abi.desc(N, sh.d, El, sh.I, 1, "bf16", 1)
    ws = abi.alloc_workspace(dsc, DEV)
    y = torch.full((N, sh.d), float("nan"), dtype=torch.float32, device=DEV)
    abi.expert_rows(dsc, x, eid.to(DEV), W1, W3, W2, y, ws)
    abi.check(dsc, ws)
    e = eid.numpy().reshape(N, 1)
    ref = oracle.experts(host(x), host(W1), host(W3), host(W2), e,
                         (e >= 0).astype(np.float64), "bf16")
    got = y.double().cpu().numpy()
    assert (got[e[:, 0] < 0] == 0).all()
    rows = e[:, 0] >= 0
    rms = np.sqrt((ref[rows] ** 2).mean(axis=1))
    assert ((np.abs(got[rows] - ref[rows]).max(axis=1) / rms) <= 2e-2).all()
    # an id outside [-1, E) is reported, not followed
    bad = eid.clone()
    bad[5] = El
    abi.expert_rows(dsc, x, bad.to(DEV), W1, W3, W2, y, ws)
    with pytest.raises(abi.BeamError) as ei:
        abi.check(dsc, ws)
    assert ei.value.status == 6  # BEAM_ERR_INTERNAL
