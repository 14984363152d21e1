"""ctypes binding of libbeam_moe.so (include/beam_moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch tensors on the current CUDA device; streams default
to torch's current stream.  Loading fails loudly when the library is missing:
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbeam_moe.so")

BEAM_BF16 = 0
BEAM_F32 = 1
FORWARD_STAGES = 7

STATUS = {0: "BEAM_OK", 1: "BEAM_ERR_INVALID_ARG", 2: "BEAM_ERR_UNSUPPORTED_SHAPE",
          3: "BEAM_ERR_WORKSPACE", 4: "BEAM_ERR_CUDA", 5: "BEAM_ERR_TIMEOUT",
          6: "BEAM_ERR_INTERNAL"}


class BeamError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class Desc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("d", ctypes.c_int), ("E", ctypes.c_int),
                ("I", ctypes.c_int), ("K", ctypes.c_int), ("dtype", ctypes.c_int),
                ("renorm_topk", ctypes.c_int), ("mask_logit_threshold", ctypes.c_float),
                ("n_shared", ctypes.c_int), ("I_shared", ctypes.c_int)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("BN", ctypes.c_int), ("router_bn", ctypes.c_int),
                ("router_splits", ctypes.c_int), ("p_cap", ctypes.c_int),
                ("tiles_cap", ctypes.c_int), ("sub_bn", ctypes.c_int),
                ("one_launch", ctypes.c_int), ("sh_bn", ctypes.c_int),
                ("sh_split1", ctypes.c_int), ("sh_split2", ctypes.c_int)] + \
               [(n, ctypes.c_size_t) for n in (
                   "off_err", "off_meta", "off_counts", "off_hist", "off_partial", "off_idx",
                   "off_w", "off_pair", "off_pair_pos", "off_tiles", "off_xp", "off_h", "off_y",
                   "off_tile_done", "off_hs", "off_ys", "off_tiles_sub", "off_ctl", "off_sp",
                   "workspace_bytes")]


_lib = None


def lib():
    """The loaded library; raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m dynamic_expert_routing_router_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        pd = ctypes.POINTER(Desc)
        L.beam_moe_workspace_size.argtypes = [pd]
        L.beam_moe_workspace_size.restype = sz
        L.beam_moe_plan.argtypes = [pd, ctypes.POINTER(PlanInfo)]
        L.beam_moe_route.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.beam_moe_forward.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.beam_moe_forward_shared.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                              vp]
        L.beam_moe_forward_shared.restype = i32
        L.beam_moe_forward_profiled.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                                ctypes.POINTER(vp)]
        L.beam_moe_check.argtypes = [pd, vp, vp]
        L.beam_moe_route_noalloc.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.beam_moe_route_noalloc.restype = i32
        L.beam_moe_set_one_launch_tokens.argtypes = [i32]
        L.beam_moe_set_one_launch_tokens.restype = i32
        L.beam_moe_forward_kernel_count.argtypes = [pd]
        L.beam_moe_forward_kernel_count.restype = i32
        L.beam_moe_backward_workspace_size.argtypes = [pd]
        L.beam_moe_backward_workspace_size.restype = sz
        L.beam_moe_backward.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp,
                                        vp, vp, vp, vp, sz, vp]
        L.beam_moe_backward.restype = i32
        L.beam_moe_backward_kernel_count.argtypes = [pd]
        L.beam_moe_backward_kernel_count.restype = i32
        L.beam_moe_ep_dispatch.argtypes = [pd, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.beam_moe_ep_dispatch.restype = i32
        L.beam_moe_expert_rows.argtypes = [pd, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.beam_moe_expert_rows.restype = i32
        L.beam_moe_ep_combine.argtypes = [pd, vp, vp, vp, vp, vp, vp]
        L.beam_moe_ep_combine.restype = i32
        L.beam_moe_route_noalloc_check.argtypes = [vp]
        L.beam_moe_route_noalloc_check.restype = i32
        L.beam_moe_tau_to_logit.argtypes = [ctypes.c_float]
        L.beam_moe_tau_to_logit.restype = ctypes.c_float
        L.beam_moe_set_fault_injection.argtypes = [i32, ctypes.c_ulonglong]
        L.beam_moe_set_fault_injection.restype = i32
        L.beam_status_str.argtypes = [i32]
        L.beam_status_str.restype = ctypes.c_char_p
        L.beam_moe_stage_name.argtypes = [i32]
        L.beam_moe_stage_name.restype = ctypes.c_char_p
        for f in ("beam_moe_plan", "beam_moe_route", "beam_moe_forward",
                  "beam_moe_forward_profiled", "beam_moe_check"):
            getattr(L, f).restype = i32
        _lib = L
    return _lib


def tau_logit(tau: float) -> float:
    """The descriptor's mask threshold for sigmoid(z) >= tau (beam_moe_tau_to_logit)."""
    return float(lib().beam_moe_tau_to_logit(ctypes.c_float(tau)))


def desc(T, d, E, I, K, dtype="bf16", renorm=1, tau=0.5, n_shared=0, I_shared=0) -> Desc:
    """Layer descriptor; `tau` is the mask threshold of sigmoid(x W_mask);
    n_shared always-on shared experts of width I_shared."""
    code = dtype if isinstance(dtype, int) else (BEAM_BF16 if dtype == "bf16" else BEAM_F32)
    return Desc(int(T), int(d), int(E), int(I), int(K), int(code), int(renorm),
                tau_logit(tau), int(n_shared), int(I_shared))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ok(status, what):
    if status != 0:
        raise BeamError(status, what)


def status_str(status: int) -> str:
    return lib().beam_status_str(int(status)).decode()


def stage_name(i: int):
    s = lib().beam_moe_stage_name(int(i))
    return None if s is None else s.decode()


def workspace_size(dsc: Desc) -> int:
    return int(lib().beam_moe_workspace_size(ctypes.byref(dsc)))


def set_one_launch_tokens(max_tokens: int) -> int:
    """Largest batch run as one launch (0 = never); returns the previous value."""
    return int(lib().beam_moe_set_one_launch_tokens(int(max_tokens)))


def kernel_count(dsc: Desc) -> int:
    """Kernel launches of one forward call for this descriptor."""
    return int(lib().beam_moe_forward_kernel_count(ctypes.byref(dsc)))


def backward_workspace_size(dsc: Desc) -> int:
    return int(lib().beam_moe_backward_workspace_size(ctypes.byref(dsc)))


def backward_kernel_count(dsc: Desc) -> int:
    """Kernel launches of one backward call for this descriptor."""
    return int(lib().beam_moe_backward_kernel_count(ctypes.byref(dsc)))


def alloc_backward_workspace(dsc: Desc, device=None):
    """A uint8 torch tensor of backward_workspace_size(dsc) bytes on `device`."""
    import torch
    n = backward_workspace_size(dsc)
    if n == 0:
        raise BeamError(1, "beam_moe_backward_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def backward(dsc, x, W_gate, W_mask, W1, W3, W2, dy, beta, dx, dW_gate, dW_mask, dW1, dW3, dW2,
             workspace, stream=None):
    """Training-mode gradients (straight-through estimator, beta-weighted
    penalty on the candidates' mask scores).  dx is overwritten; the weight
    gradients (fp32, shaped like their weights) are accumulated into."""
    _ok(lib().beam_moe_backward(ctypes.byref(dsc), _ptr(x), _ptr(W_gate), _ptr(W_mask),
                                _ptr(W1), _ptr(W3), _ptr(W2), _ptr(dy), ctypes.c_float(beta),
                                _ptr(dx), _ptr(dW_gate), _ptr(dW_mask), _ptr(dW1), _ptr(dW3),
                                _ptr(dW2), _ptr(workspace), workspace.numel(), _stream(stream)),
        "beam_moe_backward")


def plan(dsc: Desc) -> dict:
    info = PlanInfo()
    _ok(lib().beam_moe_plan(ctypes.byref(dsc), ctypes.byref(info)), "beam_moe_plan")
    return {name: getattr(info, name) for name, _ in PlanInfo._fields_}


def alloc_workspace(dsc: Desc, device=None):
    """A uint8 torch tensor of workspace_size(dsc) bytes on `device`."""
    import torch
    n = workspace_size(dsc)
    if n == 0:
        raise BeamError(1, "beam_moe_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def route(dsc, x, W_gate, W_mask, topk_idx, topk_w, counts, hist=None, logits=None,
          workspace=None, stream=None):
    _ok(lib().beam_moe_route(ctypes.byref(dsc), _ptr(x), _ptr(W_gate), _ptr(W_mask),
                             _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(hist),
                             _ptr(logits), _ptr(workspace),
                             workspace.numel() if workspace is not None else 0,
                             _stream(stream)), "beam_moe_route")


NOALLOC_SCRATCH_BYTES = 16 << 20


def route_noalloc(dsc, x, W_gate, W_mask, topk_idx, topk_w, counts, hist=None, logits=None,
                  stream=None):
    """beam_moe_route without a caller workspace (scratch in the library's own
    fixed device array); for callers that cannot allocate device memory."""
    _ok(lib().beam_moe_route_noalloc(ctypes.byref(dsc), _ptr(x), _ptr(W_gate), _ptr(W_mask),
                                     _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(hist),
                                     _ptr(logits), _stream(stream)), "beam_moe_route_noalloc")


def route_noalloc_check(stream=None):
    """Synchronise and read the error word of the last route_noalloc call."""
    _ok(lib().beam_moe_route_noalloc_check(_stream(stream)), "beam_moe_route_noalloc_check")


FAULT_NONE, FAULT_EXPERT_STAGE, FAULT_ROUTER_STAGE, FAULT_SHARED_STAGE = 0, 1, 2, 3


def set_fault_injection(mode: int, wait_limit_ns: int = 0):
    """Testing aid (beam_moe_set_fault_injection): make a bounded device wait
    expire in later calls; mode 0 and wait_limit_ns 0 restore the defaults."""
    _ok(lib().beam_moe_set_fault_injection(int(mode), int(wait_limit_ns)),
        "beam_moe_set_fault_injection")


def forward(dsc, x, W_gate, W_mask, W1, W3, W2, out, workspace, stream=None):
    _ok(lib().beam_moe_forward(ctypes.byref(dsc), _ptr(x), _ptr(W_gate), _ptr(W_mask),
                               _ptr(W1), _ptr(W3), _ptr(W2), _ptr(out), _ptr(workspace),
                               workspace.numel(), _stream(stream)), "beam_moe_forward")


def forward_shared(dsc, x, W_gate, W_mask, W1, W3, W2, W1s, W3s, W2s, out, workspace,
                   stream=None):
    """The layer with dsc.n_shared always-on shared experts (weights W1s, W3s
    [S, I_shared, d], W2s [S, d, I_shared])."""
    _ok(lib().beam_moe_forward_shared(ctypes.byref(dsc), _ptr(x), _ptr(W_gate), _ptr(W_mask),
                                      _ptr(W1), _ptr(W3), _ptr(W2), _ptr(W1s), _ptr(W3s),
                                      _ptr(W2s), _ptr(out), _ptr(workspace), workspace.numel(),
                                      _stream(stream)), "beam_moe_forward_shared")


def forward_profiled(dsc, x, W_gate, W_mask, W1, W3, W2, out, workspace, events, stream=None):
    """`events`: FORWARD_STAGES + 1 torch.cuda.Event(enable_timing=True) or None
    (None records nothing at that point)."""
    arr = (ctypes.c_void_p * len(events))(*[None if e is None else e.cuda_event
                                             for e in events])
    _ok(lib().beam_moe_forward_profiled(ctypes.byref(dsc), _ptr(x), _ptr(W_gate), _ptr(W_mask),
                                        _ptr(W1), _ptr(W3), _ptr(W2), _ptr(out),
                                        _ptr(workspace), workspace.numel(), _stream(stream),
                                        arr), "beam_moe_forward_profiled")


def ep_dispatch(dsc, n_ranks, x, topk_idx, counts, send_rows, send_pair, send_expert,
                send_counts, pair_pos, workspace, stream=None):
    """Kept pairs grouped by destination rank (expert-parallel dispatch)."""
    _ok(lib().beam_moe_ep_dispatch(ctypes.byref(dsc), int(n_ranks), _ptr(x), _ptr(topk_idx),
                                   _ptr(counts), _ptr(send_rows), _ptr(send_pair),
                                   _ptr(send_expert), _ptr(send_counts), _ptr(pair_pos),
                                   _ptr(workspace), workspace.numel(), _stream(stream)),
        "beam_moe_ep_dispatch")


def expert_rows(dsc, x_rows, expert_id, W1, W3, W2, y_rows, workspace, stream=None):
    """y_rows[i] = E_{expert_id[i]}(x_rows[i]) in fp32 (dsc.K == 1, dsc.T rows)."""
    _ok(lib().beam_moe_expert_rows(ctypes.byref(dsc), _ptr(x_rows), _ptr(expert_id), _ptr(W1),
                                   _ptr(W3), _ptr(W2), _ptr(y_rows), _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "beam_moe_expert_rows")


def ep_combine(dsc, y_rows, topk_idx, topk_w, pair_pos, out, stream=None):
    """out_t = sum over kept k of topk_w[t,k] * y_rows[pair_pos[t,k]] (slot order)."""
    _ok(lib().beam_moe_ep_combine(ctypes.byref(dsc), _ptr(y_rows), _ptr(topk_idx),
                                  _ptr(topk_w), _ptr(pair_pos), _ptr(out), _stream(stream)),
        "beam_moe_ep_combine")


def check(dsc, workspace, stream=None):
    _ok(lib().beam_moe_check(ctypes.byref(dsc), _ptr(workspace), _stream(stream)),
        "beam_moe_check")


def workspace_views(dsc, workspace) -> dict:
    """Typed views of the intermediate arrays inside a forward workspace."""
    import torch
    P = plan(dsc)
    T, K, E = dsc.T, dsc.K, dsc.E
    dt = torch.bfloat16 if dsc.dtype == BEAM_BF16 else torch.float32
    es = 2 if dsc.dtype == BEAM_BF16 else 4

    def view(off, n, dtype, size):
        return workspace[off: off + n * size].view(dtype)

    return dict(
        err=view(P["off_err"], 1, torch.int32, 4),
        meta=view(P["off_meta"], 4, torch.int32, 4),
        counts=view(P["off_counts"], E, torch.int32, 4),
        hist=view(P["off_hist"], K + 1, torch.int32, 4),
        partial=view(P["off_partial"], P["router_splits"] * T * 2 * E, torch.float32, 4).view(
            P["router_splits"], T, 2 * E),
        idx=view(P["off_idx"], T * K, torch.int32, 4).view(T, K),
        w=view(P["off_w"], T * K, torch.float32, 4).view(T, K),
        pair=view(P["off_pair"], P["p_cap"], torch.int32, 4),
        pair_pos=view(P["off_pair_pos"], T * K, torch.int32, 4).view(T, K),
        tiles=view(P["off_tiles"], 4 * P["tiles_cap"], torch.int32, 4).view(-1, 4),
        xp=view(P["off_xp"], P["p_cap"] * dsc.d, dt, es).view(P["p_cap"], dsc.d),
        h=view(P["off_h"], P["p_cap"] * dsc.I, dt, es).view(P["p_cap"], dsc.I),
        y=view(P["off_y"], P["p_cap"] * dsc.d, torch.float32, 4).view(P["p_cap"], dsc.d),
        ys=view(P["off_ys"], max(1, P["sh_split2"]) * dsc.n_shared * T * dsc.d, torch.float32,
                4).view(max(1, P["sh_split2"]) * dsc.n_shared * T, dsc.d),
        plan=P,
    )
