"""Expert parallelism on CPU: real gloo all-to-alls through the product's
exchange functions (dynamic_expert_routing_router_b200.ep), with G ranks
(G = 2 and 4) each owning E/G experts of the tiny fp32 layer.

The kernels need a GPU, so each rank's local steps are taken by the oracle
here, in the conventions the CUDA dispatch kernel implements (and
tests/test_gpu_ep.py checks on the GPU bit for bit): kept pairs in the
oracle's permutation order (expert, then token), split by expert block,
tagged with the expert's local id; fp32 rows come back in the order they
went.  Each rank's reassembled output must equal the single-rank oracle
layer on its own tokens, and only kept pairs may cross.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    from dynamic_expert_routing_router_b200 import inputs
    L = inputs.make_tiny(T=16, seed=0, gamma=0.0, device="cpu")
    return {k: v.numpy() for k, v in L.items()}


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from dynamic_expert_routing_router_b200 import ep, inputs
        sh = inputs.TINY
        E, K, d = sh.E, sh.K, sh.d
        El = E // world
        L = _layer()
        # this rank's own tokens (seeded per rank), the shared router and experts
        x = inputs.make_tiny(T=16 + 3 * rank, seed=100 + rank, device="cpu")["x"].numpy()
        r, z = oracle.logits(x, L["W_gate"], L["W_mask"], "f32")
        rt = oracle.route(r, z, K, sh.renorm)
        idx, w = rt["idx"], rt["w"]
        # dispatch (the kernel's convention): kept pairs by expert then token
        offsets, pairs = oracle.permutation(idx, E)
        send_splits = [int(offsets[(j + 1) * El] - offsets[j * El]) for j in range(world)]
        assert sum(send_splits) == int((idx >= 0).sum())  # kept pairs only
        send_rows = torch.from_numpy(x[pairs // K])
        send_expert = torch.from_numpy((idx.reshape(-1)[pairs] % El).astype(np.int32))
        pos = -np.ones(idx.size, np.int64)
        pos[pairs] = np.arange(len(pairs))
        # exchange (product code): counts, rows, local expert ids
        recv_splits = ep.exchange_counts(send_splits, world, "cpu")
        recv_rows = ep.exchange_rows(send_rows, send_splits, recv_splits)
        recv_expert = ep.exchange_rows(send_expert, send_splits, recv_splits)
        # this rank's experts on the received rows (oracle stands in for the kernels)
        sl = slice(rank * El, (rank + 1) * El)
        N = recv_rows.shape[0]
        y = oracle.experts(recv_rows.numpy(), L["W1"][sl], L["W3"][sl], L["W2"][sl],
                           recv_expert.numpy().reshape(N, 1), np.ones((N, 1)), "f32") \
            if N else np.zeros((0, d))
        # rows back in the order they came, then the combine at the source
        y_back = ep.exchange_rows(torch.from_numpy(np.ascontiguousarray(y)), recv_splits,
                                  send_splits).numpy()
        got = np.zeros((x.shape[0], d))
        for t in range(x.shape[0]):
            for k in range(K):
                if idx[t, k] >= 0:
                    got[t] += w[t, k] * y_back[pos[t * K + k]]
        ref = oracle.experts(x, L["W1"], L["W3"], L["W2"], idx, w, "f32")
        out[rank] = (float(np.abs(got - ref).max()), float(np.abs(ref).max()),
                     sum(send_splits), sum(recv_splits), int(idx.size))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_exchange_reassembles_the_single_rank_layer(world):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    sent = recv = 0
    for rank in range(world):
        err, mx, s, r, cand = out[rank]
        assert err <= 1e-12 * mx, (rank, err, mx)
        assert s < cand  # the mask kept some candidates back: fewer rows than T*K
        sent += s
        recv += r
    assert sent == recv  # every row sent was received once
