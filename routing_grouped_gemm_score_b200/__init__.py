"""Python binding of libmoe_b200.so, the B200 (sm_100a) MoE layer.

The functions carry the names of the C entry points in include/moe_b200.h.
They only marshal arguments: they check dtypes and shapes, allocate outputs
and workspace with torch, and pass raw device pointers and the current CUDA
stream to the library. Every step of the layer runs in the library's CUDA
kernels. If the library is missing or cannot be loaded, importing it raises;
there is no fallback.

Stages (Transformer Engine "Mixture of Experts": Router, Token dispatch,
Grouped MLP, Token combine):
    moe_router_topk -> moe_permute -> moe_grouped_mlp -> moe_unpermute_combine
fused as moe_layer_forward, with moe_grouped_mlp_backward for training and
moe_router_backward for the gradient through the score function.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

__all__ = [
    "MoEError", "RouterOpts", "SCORE_SOFTMAX", "SCORE_SIGMOID", "library_path", "lib",
    "moe_status_string", "moe_get_device_status", "moe_router_topk", "moe_permute",
    "moe_grouped_mlp", "moe_unpermute_combine", "moe_layer_forward", "moe_grouped_mlp_backward",
    "moe_grouped_mlp_scaled_backward",
    "moe_trace_set", "moe_router_topk_noalloc", "moe_router_backward", "moe_expert_bias_update", "LayerWorkspace", "ABI_FUNCTIONS",
]

SCORE_SOFTMAX = 0
SCORE_SIGMOID = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_build", "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA = 1, 2, 3
MOE_ERR_WORKSPACE, MOE_ERR_DEVICE_CHECK, MOE_ERR_TIMEOUT = 4, 5, 6
_STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
                 4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_DEVICE_CHECK", 6: "MOE_ERR_TIMEOUT"}


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {moe_status_string(status)}")


class _RouterOptsC(ctypes.Structure):
    _fields_ = [("score_fn", ctypes.c_int), ("renormalize", ctypes.c_int),
                ("scaling", ctypes.c_float), ("expert_bias", ctypes.c_void_p)]


@dataclass
class RouterOpts:
    """Router options: score function, renormalisation, scaling factor and
    optional selection-only expert bias (device fp32 [E], sigmoid only)."""
    score_fn: int = SCORE_SOFTMAX
    renormalize: bool = True
    scaling: float = 1.0
    expert_bias: Optional[torch.Tensor] = None

    def c(self) -> _RouterOptsC:
        bias = self.expert_bias
        if bias is not None:
            _need(bias, torch.float32, "expert_bias")
        return _RouterOptsC(int(self.score_fn), int(bool(self.renormalize)), float(self.scaling),
                            bias.data_ptr() if bias is not None else None)


P, I64, I32, F32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

# name -> (restype, argtypes), mirroring include/moe_b200.h
ABI_FUNCTIONS = {
    "moe_status_string": (ctypes.c_char_p, [I32]),
    "moe_get_device_status": (I32, [P]),
    "moe_trace_set": (I32, [ctypes.POINTER(ctypes.c_void_p), I32]),
    "moe_router_workspace_size": (SZ, [I64, I32, I32]),
    "moe_router_topk": (I32, [P, I64, I32, I32, ctypes.POINTER(_RouterOptsC), P, P, P, P, P, P, SZ, P]),
    "moe_router_backward": (I32, [P, I64, I32, I32, ctypes.POINTER(_RouterOptsC), P, P, P, P]),
    "moe_expert_bias_update": (I32, [P, I32, ctypes.c_float, P, P]),
    "moe_aux_loss_workspace_size": (SZ, [I64, I32]),
    "moe_aux_loss": (I32, [P, I64, I32, I32, I32, P, F32, P, P, P, SZ, P]),
    "moe_aux_loss_backward": (I32, [P, I64, I32, I32, I32, P, F32, P, P, I32, P]),
    "moe_router_topk_noalloc": (I32, [P, I64, I32, I32, ctypes.POINTER(_RouterOptsC), P, P, P, P,
                                       P, P]),
    "moe_permute_workspace_size": (SZ, [I64, I32, I32]),
    "moe_permute": (I32, [P, I64, I32, P, I32, P, I32, P, P, P, P, SZ, P]),
    "moe_permute_padded_max_rows": (I64, [I64, I32, I32, I32]),
    "moe_permute_padded": (I32, [P, I64, I32, P, P, I32, P, I32, I32, P, P, P, P, P, P, SZ, P]),
    "moe_grouped_mlp_workspace_size": (SZ, [I64, I32, I32, I32]),
    "moe_grouped_mlp": (I32, [P, I64, P, I32, I32, I32, P, P, P, P, P, P, SZ, P]),
    "moe_grouped_mlp_scaled": (I32, [P, I64, P, I32, I32, I32, P, P, P, P, P, P, P, SZ, P]),
    "moe_unpermute_combine": (I32, [P, P, P, I64, I32, I32, P, P, P]),
    "moe_unpermute_combine_rows": (I32, [P, I64, P, P, I64, I32, I32, P, P, P]),
    "moe_layer_forward_workspace_size": (SZ, [I64, I32, I32, I32, I32, I32]),
    "moe_layer_forward": (I32, [P, P, I64, I32, I32, I32, I32, ctypes.POINTER(_RouterOptsC), P, P, P,
                                P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]),
    "moe_grouped_mlp_backward_workspace_size": (SZ, [I64, I32, I32, I32, I32]),
    "moe_grouped_mlp_backward": (I32, [P, I64, I32, I32, I32, I32, P, P, P, P, P, P, P, P, P, P, P,
                                       P, P, P, SZ, P]),
    "moe_grouped_mlp_scaled_backward_workspace_size": (SZ, [I64, I32, I32]),
    "moe_grouped_mlp_scaled_backward": (I32, [P, I64, I32, I32, I32, I32, P, P, P, P, P, P, I64, P, P, P,
                                              P, P, P, P, P, SZ, P]),
    "moe_testing_set_kernels": (I32, [I32, I32, I32, I32]),
    "moe_testing_wait_timeout": (I32, [I64, P]),
}

_lib = None


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded library. Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with "
                              "`python -m routing_grouped_gemm_score_b200.build`")
        l = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in ABI_FUNCTIONS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def moe_status_string(status: int) -> str:
    try:
        return lib().moe_status_string(int(status)).decode()
    except Exception:
        return _STATUS_NAMES.get(int(status), f"status {status}")


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, where)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def moe_get_device_status() -> int:
    """Synchronise the current stream and return (and clear) the device error
    status: MOE_OK, or the code of the first problem a kernel recorded."""
    return int(lib().moe_get_device_status(_stream()))


def moe_trace_set(events) -> None:
    """Record the given torch.cuda.Event objects (timing enabled, already
    recorded once so that they exist) at the stage boundaries of the next
    calls; None turns tracing off. Order of stages: see include/moe_b200.h."""
    if not events:
        _check(lib().moe_trace_set(None, 0), "moe_trace_set")
        return
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(lib().moe_trace_set(arr, len(events)), "moe_trace_set")


# kernel variants for moe_testing_set_kernels (include/moe_b200.h, testing hooks)
TESTING_AUTO = 0
GEMM_SINGLE, GEMM_PAIR, GEMM_SWAP, GEMM_SWAP_UNFUSED = 1, 2, 3, 4
ROUTER_WARP, ROUTER_LANE = 1, 2
PERMUTE_TOKENS, PERMUTE_WARP = 1, 2


def moe_testing_set_kernels(gemm_tiles: int = 0, router: int = 0, permute: int = 0,
                            fold_permute: int = 0) -> None:
    """Force kernel variants for later calls in this process (tests compare
    the variants on the same inputs); all zero restores the library's choice."""
    _check(lib().moe_testing_set_kernels(int(gemm_tiles), int(router), int(permute), int(fold_permute)),
           "moe_testing_set_kernels")


def moe_testing_wait_timeout(limit_ns: int) -> None:
    """Launch the bounded wait that runs out after limit_ns (1 .. 1e9) on the
    current stream; the next moe_get_device_status returns MOE_ERR_TIMEOUT."""
    _check(lib().moe_testing_wait_timeout(int(limit_ns), _stream()), "moe_testing_wait_timeout")


class forced_kernels:
    """Context manager around moe_testing_set_kernels that restores the
    library's own choice on exit."""

    def __init__(self, **kw):
        self.kw = kw

    def __enter__(self):
        moe_testing_set_kernels(**self.kw)
        return self

    def __exit__(self, *exc):
        moe_testing_set_kernels()
        return False


def moe_router_topk(logits: torch.Tensor, k: int, opts: Optional[RouterOpts] = None,
                    routing_map: bool = False) -> dict:
    """Score function + top-k + routing weights + per-expert counts/offsets."""
    _need(logits, torch.float32, "logits")
    T, E = logits.shape
    dev = logits.device
    opts = opts or RouterOpts()
    out = {
        "topk_idx": torch.empty((T, k), dtype=torch.int32, device=dev),
        "topk_prob": torch.empty((T, k), dtype=torch.float32, device=dev),
        "routing_map": torch.empty((T, E), dtype=torch.uint8, device=dev) if routing_map else None,
        "counts": torch.empty(E, dtype=torch.int32, device=dev),
        "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
    }
    ws = _workspace(lib().moe_router_workspace_size(T, E, k), dev)
    oc = opts.c()
    _check(lib().moe_router_topk(_ptr(logits), T, E, k, ctypes.byref(oc), _ptr(out["topk_idx"]),
                                 _ptr(out["topk_prob"]), _ptr(out["routing_map"]), _ptr(out["counts"]),
                                 _ptr(out["offsets"]), _ptr(ws), ws.numel(), _stream()),
           "moe_router_topk")
    return out


def moe_router_topk_noalloc(logits: torch.Tensor, k: int, opts: Optional[RouterOpts] = None,
                            routing_map: bool = False, out: Optional[dict] = None) -> dict:
    """moe_router_topk through the entry point that takes no workspace. It is
    for callers that cannot allocate device memory while routing. Pass `out`
    with preallocated topk_idx, topk_prob, counts, offsets (and routing_map)
    tensors to allocate nothing at all; the library's fixed scratch limits T
    to 32768 and T * k to 262144."""
    _need(logits, torch.float32, "logits")
    T, E = logits.shape
    dev = logits.device
    if out is None:
        out = {
            "topk_idx": torch.empty((T, k), dtype=torch.int32, device=dev),
            "topk_prob": torch.empty((T, k), dtype=torch.float32, device=dev),
            "routing_map": torch.empty((T, E), dtype=torch.uint8, device=dev) if routing_map else None,
            "counts": torch.empty(E, dtype=torch.int32, device=dev),
            "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
        }
    oc = (opts or RouterOpts()).c()
    _check(lib().moe_router_topk_noalloc(_ptr(logits), T, E, k, ctypes.byref(oc),
                                         _ptr(out["topk_idx"]), _ptr(out["topk_prob"]),
                                         _ptr(out.get("routing_map")), _ptr(out["counts"]),
                                         _ptr(out["offsets"]), _stream()),
           "moe_router_topk_noalloc")
    return out


def moe_router_backward(logits: torch.Tensor, topk_idx: torch.Tensor, dprob: torch.Tensor,
                        opts: Optional[RouterOpts] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """dL/dlogits [T,E] (fp32) from dL/dtopk_prob for the experts the forward
    chose, through the score function and the weight normalisation."""
    _need(logits, torch.float32, "logits")
    _need(topk_idx, torch.int32, "topk_idx")
    _need(dprob, torch.float32, "dprob")
    T, E = logits.shape
    k = topk_idx.shape[1]
    if out is None:
        out = torch.empty((T, E), dtype=torch.float32, device=logits.device)
    oc = (opts or RouterOpts()).c()
    _check(lib().moe_router_backward(_ptr(logits), T, E, k, ctypes.byref(oc), _ptr(topk_idx), _ptr(dprob),
                                     _ptr(out), _stream()), "moe_router_backward")
    return out


def moe_expert_bias_update(counts: torch.Tensor, expert_bias: torch.Tensor, coeff: float) -> torch.Tensor:
    """Aux-loss-free load balancing between steps: updates expert_bias in place
    from the per-expert token counts of the last step, and returns it."""
    _need(counts, torch.int32, "counts")
    _need(expert_bias, torch.float32, "expert_bias")
    _check(lib().moe_expert_bias_update(_ptr(counts), counts.numel(), float(coeff), _ptr(expert_bias), _stream()),
           "moe_expert_bias_update")
    return expert_bias


def moe_aux_loss(logits: torch.Tensor, counts: torch.Tensor, k: int, coeff: float,
                 score_fn: int = 0, want_scores: bool = False,
                 workspace: Optional[torch.Tensor] = None) -> tuple:
    """Auxiliary load-balancing loss: (loss as a 0-d fp32 device tensor, the
    dense scores [T,E] or None). counts: tokens per expert from the router."""
    _need(logits, torch.float32, "logits")
    _need(counts, torch.int32, "counts")
    T, E = logits.shape
    dev = logits.device
    loss = torch.empty((), dtype=torch.float32, device=dev)
    scores = torch.empty((T, E), dtype=torch.float32, device=dev) if want_scores else None
    need = lib().moe_aux_loss_workspace_size(T, E)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _check(lib().moe_aux_loss(_ptr(logits), T, E, int(k), int(score_fn), _ptr(counts), float(coeff), _ptr(loss),
                              _ptr(scores), _ptr(workspace), workspace.numel(), _stream()), "moe_aux_loss")
    return loss, scores


def moe_aux_loss_backward(logits: torch.Tensor, counts: torch.Tensor, k: int, coeff: float,
                          score_fn: int = 0, grad_loss: Optional[torch.Tensor] = None,
                          dlogits: Optional[torch.Tensor] = None, accumulate: bool = False) -> torch.Tensor:
    """d(grad_loss * aux loss)/dlogits [T,E] (fp32), counts held fixed. With
    accumulate, adds to the given dlogits."""
    _need(logits, torch.float32, "logits")
    _need(counts, torch.int32, "counts")
    T, E = logits.shape
    if grad_loss is not None:
        _need(grad_loss, torch.float32, "grad_loss")
    if dlogits is None:
        if accumulate:
            raise ValueError("accumulate needs the dlogits to add to")
        dlogits = torch.empty((T, E), dtype=torch.float32, device=logits.device)
    _check(lib().moe_aux_loss_backward(_ptr(logits), T, E, int(k), int(score_fn), _ptr(counts), float(coeff),
                                       _ptr(grad_loss), _ptr(dlogits), int(bool(accumulate)), _stream()),
           "moe_aux_loss_backward")
    return dlogits


def moe_permute(x: torch.Tensor, topk_idx: torch.Tensor, offsets: torch.Tensor) -> dict:
    """Token dispatch into expert-contiguous order (token-ascending in a block)."""
    _need(x, torch.bfloat16, "x")
    _need(topk_idx, torch.int32, "topk_idx")
    _need(offsets, torch.int32, "offsets")
    T, H = x.shape
    k = topk_idx.shape[1]
    E = offsets.numel() - 1
    dev = x.device
    out = {
        "x_perm": torch.empty((T * k, H), dtype=torch.bfloat16, device=dev),
        "sorted_token": torch.empty(T * k, dtype=torch.int32, device=dev),
        "row_of": torch.empty((T, k), dtype=torch.int32, device=dev),
    }
    ws = _workspace(lib().moe_permute_workspace_size(T, E, k), dev)
    _check(lib().moe_permute(_ptr(x), T, H, _ptr(topk_idx), k, _ptr(offsets), E, _ptr(out["x_perm"]),
                             _ptr(out["sorted_token"]), _ptr(out["row_of"]), _ptr(ws), ws.numel(),
                             _stream()), "moe_permute")
    return out


def moe_permute_padded_max_rows(T: int, E: int, k: int, align: int) -> int:
    """Rows a padded dispatch may use, T*k + E*(align-1), with no host sync."""
    return int(lib().moe_permute_padded_max_rows(T, E, k, int(align)))


def moe_permute_padded(x: torch.Tensor, topk_idx: torch.Tensor, offsets: torch.Tensor, align: int,
                       topk_prob: Optional[torch.Tensor] = None) -> dict:
    """Token dispatch with each expert block rounded up to a multiple of align
    rows (zero pad rows). x_perm, prob_perm and sorted_token have the dropless
    bound T*k + E*(align-1) rows; padded_offsets[E] says how many are used."""
    _need(x, torch.bfloat16, "x")
    _need(topk_idx, torch.int32, "topk_idx")
    _need(offsets, torch.int32, "offsets")
    if topk_prob is not None:
        _need(topk_prob, torch.float32, "topk_prob")
    T, H = x.shape
    k = topk_idx.shape[1]
    E = offsets.numel() - 1
    dev = x.device
    R = max(moe_permute_padded_max_rows(T, E, k, align), 1)
    out = {
        "padded_offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "x_perm": torch.empty((R, H), dtype=torch.bfloat16, device=dev),
        "prob_perm": torch.empty(R, dtype=torch.float32, device=dev) if topk_prob is not None else None,
        "sorted_token": torch.empty(R, dtype=torch.int32, device=dev),
        "row_of": torch.empty((T, k), dtype=torch.int32, device=dev),
    }
    ws = _workspace(lib().moe_permute_workspace_size(T, E, k), dev)
    _check(lib().moe_permute_padded(_ptr(x), T, H, _ptr(topk_idx), _ptr(topk_prob), k, _ptr(offsets), E,
                                    int(align), _ptr(out["padded_offsets"]), _ptr(out["x_perm"]),
                                    _ptr(out["prob_perm"]), _ptr(out["sorted_token"]), _ptr(out["row_of"]),
                                    _ptr(ws), ws.numel(), _stream()), "moe_permute_padded")
    return out


def moe_grouped_mlp(x_perm: torch.Tensor, offsets: torch.Tensor, w_gate_up: torch.Tensor,
                    w_down: torch.Tensor, save: bool = False, row_scale: Optional[torch.Tensor] = None) -> dict:
    """Grouped SwiGLU expert MLP over expert-contiguous rows. With row_scale
    (fp32 [A]) the activation of row r is multiplied by row_scale[r] before
    FC2 (ScaledSwiGLU), and the combine must then run without weights."""
    for t, n in ((x_perm, "x_perm"), (w_gate_up, "w_gate_up"), (w_down, "w_down")):
        _need(t, torch.bfloat16, n)
    if row_scale is not None:
        _need(row_scale, torch.float32, "row_scale")
    _need(offsets, torch.int32, "offsets")
    A, H = x_perm.shape
    E, _, I2 = w_gate_up.shape
    I = I2 // 2
    dev = x_perm.device
    out = {"y_perm": torch.empty((A, H), dtype=torch.bfloat16, device=dev),
           "gu": torch.empty((A, 2 * I), dtype=torch.bfloat16, device=dev) if save else None,
           "h": torch.empty((A, I), dtype=torch.bfloat16, device=dev) if save else None}
    ws = _workspace(0 if save else lib().moe_grouped_mlp_workspace_size(A, E, H, I), dev)
    _check(lib().moe_grouped_mlp_scaled(_ptr(x_perm), A, _ptr(offsets), E, H, I, _ptr(w_gate_up),
                                        _ptr(w_down), _ptr(row_scale), _ptr(out["y_perm"]), _ptr(out["gu"]),
                                        _ptr(out["h"]), _ptr(ws), ws.numel(), _stream()), "moe_grouped_mlp")
    return out


def moe_grouped_mlp_scaled(x_perm: torch.Tensor, offsets: torch.Tensor, w_gate_up: torch.Tensor,
                           w_down: torch.Tensor, row_scale: torch.Tensor, save: bool = False) -> dict:
    """Grouped MLP with ScaledSwiGLU: the routing weight of each row applied to
    the activation before FC2 (combine then runs without weights)."""
    return moe_grouped_mlp(x_perm, offsets, w_gate_up, w_down, save=save, row_scale=row_scale)


def moe_unpermute_combine(y_perm: torch.Tensor, row_of: torch.Tensor,
                          topk_prob: Optional[torch.Tensor] = None,
                          shared_out: Optional[torch.Tensor] = None,
                          out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Token combine: out[t] = shared[t] + sum_j p[t,j] y_perm[row_of[t,j]]."""
    _need(y_perm, torch.bfloat16, "y_perm")
    _need(row_of, torch.int32, "row_of")
    if topk_prob is not None:
        _need(topk_prob, torch.float32, "topk_prob")
    if shared_out is not None:
        _need(shared_out, torch.bfloat16, "shared_out")
    T, k = row_of.shape
    A, H = y_perm.shape
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=y_perm.device)
    else:
        _need(out, torch.bfloat16, "out")
        if tuple(out.shape) != (T, H):
            raise ValueError(f"out: expected shape {(T, H)}, got {tuple(out.shape)}")
    _check(lib().moe_unpermute_combine_rows(_ptr(y_perm), A, _ptr(row_of), _ptr(topk_prob), T, k, H,
                                            _ptr(shared_out), _ptr(out), _stream()),
           "moe_unpermute_combine")
    return out


def moe_unpermute_combine_rows(y_perm: torch.Tensor, row_of: torch.Tensor,
                               topk_prob: Optional[torch.Tensor] = None,
                               shared_out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """moe_unpermute_combine for a y_perm with any number of rows (for example
    a padded dispatch's); the binding's moe_unpermute_combine already passes
    y_perm's row count."""
    return moe_unpermute_combine(y_perm, row_of, topk_prob, shared_out)


class LayerWorkspace:
    """A reusable workspace for moe_layer_forward / moe_grouped_mlp_backward,
    sized once for a shape, so repeated calls allocate nothing."""

    def __init__(self, T, H, I, E, k, has_shared=False, backward=False, device="cuda"):
        n = lib().moe_layer_forward_workspace_size(T, H, I, E, k, int(has_shared))
        self.fwd = _workspace(n, device)
        self.bwd = None
        if backward:
            self.bwd = _workspace(lib().moe_grouped_mlp_backward_workspace_size(T, H, I, E, k), device)


def moe_layer_forward(logits: torch.Tensor, x: torch.Tensor, w_gate_up: torch.Tensor,
                      w_down: torch.Tensor, k: int, opts: Optional[RouterOpts] = None,
                      shared_gate_up: Optional[torch.Tensor] = None,
                      shared_down: Optional[torch.Tensor] = None, save_for_backward: bool = False,
                      workspace: Optional[LayerWorkspace] = None, out: Optional[torch.Tensor] = None,
                      state: Optional[dict] = None):
    """The fused layer: router -> permute -> grouped MLP -> combine (+ shared
    expert). Returns `out`, or (out, state) with save_for_backward, where
    state holds the tensors that moe_grouped_mlp_backward needs."""
    _need(logits, torch.float32, "logits")
    for t, n in ((x, "x"), (w_gate_up, "w_gate_up"), (w_down, "w_down")):
        _need(t, torch.bfloat16, n)
    T, H = x.shape
    E, _, I2 = w_gate_up.shape
    I = I2 // 2
    dev = x.device
    has_shared = shared_gate_up is not None
    opts = opts or RouterOpts()
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    if save_for_backward and state is None:
        A = T * k
        state = {
            "topk_idx": torch.empty((T, k), dtype=torch.int32, device=dev),
            "topk_prob": torch.empty((T, k), dtype=torch.float32, device=dev),
            "counts": torch.empty(E, dtype=torch.int32, device=dev),
            "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
            "row_of": torch.empty((T, k), dtype=torch.int32, device=dev),
            "x_perm": torch.empty((A, H), dtype=torch.bfloat16, device=dev),
            "gu": torch.empty((A, 2 * I), dtype=torch.bfloat16, device=dev),
            "h": torch.empty((A, I), dtype=torch.bfloat16, device=dev),
            "y_perm": torch.empty((A, H), dtype=torch.bfloat16, device=dev),
        }
    st = state or {}
    if workspace is None:
        workspace = LayerWorkspace(T, H, I, E, k, has_shared, device=dev)
    oc = opts.c()
    g = st.get
    _check(lib().moe_layer_forward(
        _ptr(logits), _ptr(x), T, H, I, E, k, ctypes.byref(oc), _ptr(w_gate_up), _ptr(w_down),
        _ptr(shared_gate_up), _ptr(shared_down), _ptr(out), _ptr(g("topk_idx")), _ptr(g("topk_prob")),
        _ptr(g("counts")), _ptr(g("offsets")), _ptr(g("row_of")), _ptr(g("x_perm")), _ptr(g("gu")),
        _ptr(g("h")), _ptr(g("y_perm")), _ptr(workspace.fwd), workspace.fwd.numel(), _stream()),
        "moe_layer_forward")
    return (out, state) if save_for_backward else out


def moe_grouped_mlp_backward(dout: torch.Tensor, state: dict, w_gate_up: torch.Tensor,
                             w_down: torch.Tensor, workspace: Optional[LayerWorkspace] = None,
                             grads: Optional[dict] = None) -> dict:
    """Gradients of the layer with respect to x, w_gate_up, w_down and the
    routing weights, from the state saved by moe_layer_forward."""
    _need(dout, torch.bfloat16, "dout")
    T, H = dout.shape
    E, _, I2 = w_gate_up.shape
    I = I2 // 2
    k = state["row_of"].shape[1]
    dev = dout.device
    if grads is None:
        grads = {
            "dx": torch.empty((T, H), dtype=torch.bfloat16, device=dev),
            "dw_gate_up": torch.empty_like(w_gate_up),
            "dw_down": torch.empty_like(w_down),
            "dprob": torch.empty((T, k), dtype=torch.float32, device=dev),
        }
    if workspace is None or workspace.bwd is None:
        ws = _workspace(lib().moe_grouped_mlp_backward_workspace_size(T, H, I, E, k), dev)
    else:
        ws = workspace.bwd
    s = state
    _check(lib().moe_grouped_mlp_backward(
        _ptr(dout), T, H, I, E, k, _ptr(w_gate_up), _ptr(w_down), _ptr(s["row_of"]),
        _ptr(s["topk_prob"]), _ptr(s["offsets"]), _ptr(s["x_perm"]), _ptr(s["gu"]), _ptr(s["h"]),
        _ptr(s["y_perm"]), _ptr(grads["dx"]), _ptr(grads["dw_gate_up"]), _ptr(grads["dw_down"]),
        _ptr(grads["dprob"]), _ptr(ws), ws.numel(), _stream()), "moe_grouped_mlp_backward")
    return grads


def moe_grouped_mlp_scaled_backward(dout: torch.Tensor, row_of: torch.Tensor, sorted_token: torch.Tensor,
                                    row_scale: torch.Tensor, offsets: torch.Tensor, x_perm: torch.Tensor,
                                    gu: torch.Tensor, h: torch.Tensor, w_gate_up: torch.Tensor,
                                    w_down: torch.Tensor, grads: Optional[dict] = None,
                                    workspace: Optional[torch.Tensor] = None) -> dict:
    """Gradients of the ScaledSwiGLU layer (moe_grouped_mlp_scaled, then an
    unweighted combine) with respect to x, w_gate_up, w_down and the routing
    weights, from the forward's rows: x_perm, gu and h [A, ...] with their
    sorted_token [A], row_scale [A] and offsets [E+1] (a padded dispatch's or
    not), and row_of [T, k]."""
    _need(dout, torch.bfloat16, "dout")
    _need(row_of, torch.int32, "row_of")
    _need(sorted_token, torch.int32, "sorted_token")
    _need(row_scale, torch.float32, "row_scale")
    _need(offsets, torch.int32, "offsets")
    for t, n in ((x_perm, "x_perm"), (gu, "gu"), (h, "h"), (w_gate_up, "w_gate_up"), (w_down, "w_down")):
        _need(t, torch.bfloat16, n)
    T, H = dout.shape
    E, _, I2 = w_gate_up.shape
    I = I2 // 2
    k = row_of.shape[1]
    A = x_perm.shape[0]
    dev = dout.device
    if grads is None:
        grads = {
            "dx": torch.empty((T, H), dtype=torch.bfloat16, device=dev),
            "dw_gate_up": torch.empty_like(w_gate_up),
            "dw_down": torch.empty_like(w_down),
            "dprob": torch.empty((T, k), dtype=torch.float32, device=dev),
        }
    ws = workspace
    if ws is None:
        ws = _workspace(lib().moe_grouped_mlp_scaled_backward_workspace_size(A, H, I), dev)
    _check(lib().moe_grouped_mlp_scaled_backward(
        _ptr(dout), T, H, I, E, k, _ptr(w_gate_up), _ptr(w_down), _ptr(row_of), _ptr(sorted_token),
        _ptr(row_scale), _ptr(offsets), A, _ptr(x_perm), _ptr(gu), _ptr(h), _ptr(grads["dx"]),
        _ptr(grads["dw_gate_up"]), _ptr(grads["dw_down"]), _ptr(grads["dprob"]), _ptr(ws), ws.numel(),
        _stream()), "moe_grouped_mlp_scaled_backward")
    return grads
