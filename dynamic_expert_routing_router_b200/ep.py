"""Expert parallelism for the BEAM-masked MoE layer: one process per GPU, G
ranks, rank r owning the experts [r E/G, (r+1) E/G).

Every step of the layer runs in the library's kernels (C ABI); this module only
sequences the calls and the two exchanges, which go through torch.distributed
(NCCL between GPUs):

1. route (every rank, its own tokens, the full router): candidates, mask, g*m;
2. dispatch: the KEPT pairs only, listed by expert then token, so grouped by
   destination rank; their token rows are copied into a send buffer, each row
   tagged with its expert's local id on the destination.  A masked pair never
   leaves its rank: the mask cuts the rows that cross the interconnect by the
   same fraction as the expert work (the news article on BEAM, §5: masked
   entries are left out of the expert-token grouping);
3. all-to-all of the per-destination row counts, then of the rows and ids;
4. the destination runs its local experts on the received rows
   (beam_moe_expert_rows: the layer's grouping, tensor-core GEMMs and an fp32
   Y per row);
5. all-to-all of the fp32 Y rows back, in the order they came;
6. the source combines out_t = sum_k g_k m_k Y[row(t, k)] in slot order with
   one rounding (beam_moe_ep_combine), exactly as the one-GPU layer does.

The exchanges need the counts on the host (split sizes): one small
device-to-host copy per step.  No load uses cluster multicast, and no library
kernel is given another GPU's memory: rows land in local buffers first.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import abi


@dataclass
class Dispatch:
    """Per-step state of one rank between the phases."""
    idx: torch.Tensor          # [T, K] candidate or -1
    w: torch.Tensor            # [T, K] g * m
    counts: torch.Tensor       # [E] kept pairs per expert
    send_rows: torch.Tensor    # [P, d] kept pairs' token rows, grouped by destination
    send_pair: torch.Tensor    # [P] t*K + k of each send row
    send_expert: torch.Tensor  # [P] local expert id on the destination
    send_counts: torch.Tensor  # [G] rows per destination (device)
    pair_pos: torch.Tensor     # [T, K] send row of each kept pair
    send_splits: list          # host copy of send_counts


class ExpertParallelLayer:
    """One rank's share of an expert-parallel BEAM layer.

    Wg, Wm: the full routers [E, d] (every rank routes its own tokens);
    W1, W3 [E/G, I, d], W2 [E/G, d, I]: this rank's experts."""

    def __init__(self, T, d, E, I, K, renorm, rank, world, Wg, Wm, W1, W3, W2, dtype="bf16",
                 tau=0.5, group=None):
        if E % world:
            raise ValueError("E must be a multiple of the number of ranks")
        self.T, self.d, self.E, self.I, self.K = T, d, E, I, K
        self.rank, self.world, self.group = rank, world, group
        self.El = E // world
        self.Wg, self.Wm, self.W1, self.W3, self.W2 = Wg, Wm, W1, W3, W2
        self.dtype = dtype
        self.dsc = abi.desc(T, d, E, I, K, dtype, renorm, tau=tau)
        dev = Wg.device
        self.device = dev
        self.ws = abi.alloc_workspace(self.dsc, dev)
        self.tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        cap = max(T * K, 1)
        self.idx = torch.empty((T, K), dtype=torch.int32, device=dev)
        self.w = torch.empty((T, K), dtype=torch.float32, device=dev)
        self.counts = torch.empty((E,), dtype=torch.int32, device=dev)
        self.send_rows = torch.empty((cap, d), dtype=self.tdtype, device=dev)
        self.send_pair = torch.empty((cap,), dtype=torch.int32, device=dev)
        self.send_expert = torch.empty((cap,), dtype=torch.int32, device=dev)
        self.send_counts = torch.empty((max(world, 4),), dtype=torch.int32, device=dev)
        self.pair_pos = torch.empty((T, K), dtype=torch.int32, device=dev)
        self._rows_ws = {}

    # ---- phase 1 (local) ----------------------------------------------------
    def dispatch(self, x) -> Dispatch:
        if self.T == 0:  # nothing to route or send
            z = [0] * self.world
            return Dispatch(self.idx, self.w, self.counts, self.send_rows[:0],
                            self.send_pair[:0], self.send_expert[:0],
                            self.send_counts[: self.world].zero_(), self.pair_pos, z)
        abi.route(self.dsc, x, self.Wg, self.Wm, self.idx, self.w, self.counts,
                  workspace=self.ws)
        abi.ep_dispatch(self.dsc, self.world, x, self.idx, self.counts, self.send_rows,
                        self.send_pair, self.send_expert, self.send_counts, self.pair_pos,
                        self.ws)
        splits = self.send_counts[: self.world].tolist()  # host copy: the split sizes
        P = sum(splits)
        return Dispatch(self.idx, self.w, self.counts, self.send_rows[:P], self.send_pair[:P],
                        self.send_expert[:P], self.send_counts[: self.world], self.pair_pos,
                        splits)

    # ---- phase 3 (local): this rank's experts on the rows it received -------
    def local_experts(self, recv_rows, recv_expert):
        N = recv_rows.shape[0]
        y = torch.empty((N, self.d), dtype=torch.float32, device=self.device)
        if N == 0:
            return y
        dsc = abi.desc(N, self.d, self.El, self.I, 1, self.dtype, 1)
        n = abi.workspace_size(dsc)
        ws = self._rows_ws.get("ws")
        if ws is None or ws.numel() < n:
            ws = abi.alloc_workspace(dsc, self.device)
            self._rows_ws["ws"] = ws
        abi.expert_rows(dsc, recv_rows, recv_expert, self.W1, self.W3, self.W2, y, ws)
        self._rows_ws["dsc"] = dsc
        return y

    # ---- phase 5 (local): weighted sum at the source ------------------------
    def combine(self, disp: Dispatch, y_back, out):
        if self.T == 0:
            return out
        if y_back.shape[0] == 0:  # every pair masked: no row is read, but pass storage
            y_back = torch.zeros((1, self.d), dtype=torch.float32, device=self.device)
        abi.ep_combine(self.dsc, y_back, disp.idx, disp.w, disp.pair_pos, out)
        return out

    def check(self):
        """Device error words of this rank's calls (synchronises).  A rank
        with no tokens launched nothing on its routing workspace."""
        if self.T > 0:
            abi.check(self.dsc, self.ws)
        if "dsc" in self._rows_ws:
            abi.check(self._rows_ws["dsc"], self._rows_ws["ws"])

    # ---- the whole step with torch.distributed exchanges -------------------
    def forward(self, x, out=None):
        if out is None:
            out = torch.empty((self.T, self.d), dtype=self.tdtype, device=self.device)
        disp = self.dispatch(x)
        recv_splits = exchange_counts(disp.send_splits, self.world, self.device, self.group)
        recv_rows = exchange_rows(disp.send_rows, disp.send_splits, recv_splits, self.group)
        recv_expert = exchange_rows(disp.send_expert, disp.send_splits, recv_splits, self.group)
        y_recv = self.local_experts(recv_rows, recv_expert)
        y_back = exchange_rows(y_recv, recv_splits, disp.send_splits, self.group)
        return self.combine(disp, y_back, out)


def exchange_counts(send_splits, world, device, group=None):
    """All-to-all of the per-destination row counts: returns how many rows
    this rank receives from each source rank (host list)."""
    import torch.distributed as dist
    if world == 1:
        return list(send_splits)
    s = torch.tensor(send_splits, dtype=torch.int64, device=device)
    r = torch.empty_like(s)
    dist.all_to_all_single(r, s, group=group)
    return r.tolist()


def exchange_rows(send, send_splits, recv_splits, group=None):
    """All-to-all of rows: chunk j of `send` (send_splits[j] rows) goes to rank
    j; the result holds the chunks received from ranks 0, 1, ... in order."""
    import torch.distributed as dist
    world = len(send_splits)
    recv = torch.empty((sum(recv_splits),) + tuple(send.shape[1:]), dtype=send.dtype,
                       device=send.device)
    if world == 1:
        recv.copy_(send)
        return recv
    dist.all_to_all_single(recv, send.contiguous(), output_split_sizes=list(recv_splits),
                           input_split_sizes=list(send_splits), group=group)
    return recv
