"""CPU oracle of the MoE layer. TEST INFRASTRUCTURE ONLY.

Only tests/, the package's smoke check and the benchmark's CPU-baseline leg
import this module. The product path (the CUDA library and its binding) never
imports it. The arithmetic lives in moe_oracle.c (plain C, explicit loops).
This file compiles that source with gcc and marshals numpy arrays to it.

Every function returns numpy arrays and takes host arrays only:
  bf16 tensors as uint16 bit patterns, fp32 as float32, indices as int32.
ctypes releases the GIL during each call, so `moe_forward_tokens` can spread
per-token work over host threads. Each token is independent, so the results
do not depend on the thread count.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into oracle/_build/libmoe_oracle.so (gcc, -O2,
    no fast-math, no FMA contraction)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
            lib.oracle_round_bf16.argtypes = [ctypes.c_double]
            lib.oracle_round_bf16.restype = ctypes.c_uint16
            lib.oracle_round_bf16_array.argtypes = [P, i64, P]
            lib.oracle_round_bf16_array.restype = None
            lib.oracle_router_topk.argtypes = [P, i64, i32, i32, i32, i32, f32, P, P, P, P, P, P]
            lib.oracle_router_topk.restype = i32
            lib.oracle_router_backward.argtypes = [P, i64, i32, i32, i32, i32, f32, P, P, P]
            lib.oracle_router_backward.restype = i32
            lib.oracle_expert_bias_update.argtypes = [P, i32, f32, P]
            lib.oracle_expert_bias_update.restype = None
            f64 = ctypes.c_double
            lib.oracle_aux_scores.argtypes = [P, i64, i32, i32, P]
            lib.oracle_aux_scores.restype = None
            lib.oracle_aux_loss.argtypes = [P, P, i64, i32, i32, f64]
            lib.oracle_aux_loss.restype = f64
            lib.oracle_aux_loss_backward.argtypes = [P, P, i64, i32, i32, i32, f64, f64, P]
            lib.oracle_aux_loss_backward.restype = None
            lib.oracle_dispatch.argtypes = [P, i64, i32, i32, P, P, P]
            lib.oracle_dispatch.restype = i32
            lib.oracle_dispatch_padded.argtypes = [P, i64, i32, i32, P, i32, P, P, P]
            lib.oracle_dispatch_padded.restype = i32
            lib.oracle_gather_rows.argtypes = [P, i32, P, i64, P]
            lib.oracle_gather_rows.restype = None
            lib.oracle_expert_mlp.argtypes = [P, i64, i32, i32, P, P, i32, P, P, P, P]
            lib.oracle_expert_mlp.restype = None
            lib.oracle_grouped_mlp.argtypes = [P, P, i32, i32, i32, P, P, i32, P]
            lib.oracle_grouped_mlp.restype = None
            lib.oracle_combine.argtypes = [P, P, P, i64, i32, i32, P, P]
            lib.oracle_combine.restype = None
            lib.oracle_moe_forward_tokens.argtypes = [P, P, i32, i32, i32, i32, i32, i32, f32, P,
                                                      P, P, P, P, i32, P, i64, P]
            lib.oracle_moe_forward_tokens.restype = i32
            lib.oracle_moe_backward.argtypes = [P, i64, i32, i32, i32, i32, P, P, P, P, P, i32,
                                                i32, P, i64, P, P, P, P]
            lib.oracle_moe_backward.restype = i32
            lib.oracle_moe_backward_state.argtypes = [P, i64, i32, i32, i32, i32, P, P, P, P, P, i32,
                                                      i32, P, i64, P, P, P, P, P, P, P, P]
            lib.oracle_moe_backward_state.restype = i32
            lib.oracle_moe_backward_scaled.argtypes = [P, i64, i32, i32, i32, i32, P, P, P, P, P, i32,
                                                       i32, P, i64, P, P, P, P, P, P, P]
            lib.oracle_moe_backward_scaled.restype = i32
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def bf16_bits(t) -> np.ndarray:
    """A torch bf16 tensor (any device) -> uint16 numpy array of its bits."""
    import torch
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_float(b: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 values."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(v: float) -> int:
    return int(_load().oracle_round_bf16(float(v)))


def round_bf16_array(v) -> np.ndarray:
    """float64 array -> uint16 bf16 bit patterns (nearest, ties to even)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.zeros(v.shape, np.uint16)
    _load().oracle_round_bf16_array(_p(v), v.size, _p(out))
    return out


def router_topk(logits, k, score=0, renormalize=True, scaling=1.0, expert_bias=None,
                with_map=True):
    lib = _load()
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.zeros((T, k), np.int32)
    prob = np.zeros((T, k), np.float32)
    rmap = np.zeros((T, E), np.uint8) if with_map else None
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    rc = lib.oracle_router_topk(_p(logits), T, E, k, score, int(renormalize), scaling,
                                _p(_c(expert_bias, np.float32)), _p(idx), _p(prob), _p(rmap),
                                _p(counts), _p(offsets))
    if rc:
        raise ValueError(f"oracle_router_topk rejected its arguments ({rc})")
    return dict(topk_idx=idx, topk_prob=prob, routing_map=rmap, counts=counts, offsets=offsets)


def router_backward(logits, topk_idx, dprob, score=0, renormalize=True, scaling=1.0):
    """dL/dlogits [T,E] (fp32) from dL/dtopk_prob, for the experts in topk_idx
    (oracle_router_backward; fp64 inside)."""
    lib = _load()
    logits = _c(logits, np.float32)
    topk_idx = _c(topk_idx, np.int32)
    dprob = _c(dprob, np.float32)
    T, E = logits.shape
    k = topk_idx.shape[1]
    dl = np.zeros((T, E), np.float32)
    rc = lib.oracle_router_backward(_p(logits), T, E, k, score, int(renormalize), scaling, _p(topk_idx),
                                    _p(dprob), _p(dl))
    if rc:
        raise ValueError(f"oracle_router_backward: invalid index ({rc})")
    return dl


def expert_bias_update(counts, bias, coeff):
    """The expert bias after one load-balancing update (returns a new array)."""
    lib = _load()
    counts = _c(counts, np.int32)
    out = np.array(bias, np.float32, copy=True)
    lib.oracle_expert_bias_update(_p(counts), len(counts), coeff, _p(out))
    return out


def aux_scores(logits, score=0):
    """Dense scores [T,E] (float64) for the auxiliary loss: softmax over all
    experts (score 0) or the sigmoid of each logit (score 1)."""
    lib = _load()
    logits = _c(logits, np.float32)
    T, E = logits.shape
    out = np.zeros((T, E), np.float64)
    lib.oracle_aux_scores(_p(logits), T, E, int(score), _p(out))
    return out


def aux_loss(logits, counts, k, coeff, score=0):
    """The load-balancing loss (float) from the logits and per-expert counts
    (oracle_aux_loss on oracle_aux_scores)."""
    lib = _load()
    s = aux_scores(logits, score)
    counts = _c(counts, np.int32)
    T, E = s.shape
    return float(lib.oracle_aux_loss(_p(s), _p(counts), T, E, int(k), float(coeff)))


def aux_loss_backward(logits, counts, k, coeff, score=0, grad_loss=1.0):
    """d(grad_loss * loss)/dlogits [T,E] (float64), counts held fixed."""
    lib = _load()
    logits = _c(logits, np.float32)
    counts = _c(counts, np.int32)
    T, E = logits.shape
    out = np.zeros((T, E), np.float64)
    lib.oracle_aux_loss_backward(_p(logits), _p(counts), T, E, int(k), int(score), float(coeff),
                                 float(grad_loss), _p(out))
    return out


def dispatch(topk_idx, offsets, E):
    lib = _load()
    topk_idx = _c(topk_idx, np.int32)
    offsets = _c(offsets, np.int32)
    T, k = topk_idx.shape
    A = int(offsets[E])
    sorted_token = np.full(A, -1, np.int32)
    row_of = np.full((T, k), -1, np.int32)
    rc = lib.oracle_dispatch(_p(topk_idx), T, k, E, _p(offsets), _p(sorted_token), _p(row_of))
    if rc:
        raise ValueError(f"oracle_dispatch: invalid routing ({rc})")
    return sorted_token, row_of


def dispatch_padded(topk_idx, offsets, E, align):
    """Padded dispatch: (padded_offsets [E+1], sorted_token [padded total] with
    -1 in the pad rows, row_of [T,k]) (oracle_dispatch_padded)."""
    lib = _load()
    topk_idx = _c(topk_idx, np.int32)
    offsets = _c(offsets, np.int32)
    T, k = topk_idx.shape
    counts = np.diff(offsets.astype(np.int64))
    total = int(sum(-(-c // align) * align for c in counts)) if align >= 1 else 0
    padded = np.zeros(E + 1, np.int32)
    sorted_token = np.full(max(total, 1), -1, np.int32)
    row_of = np.full((T, k), -1, np.int32)
    rc = lib.oracle_dispatch_padded(_p(topk_idx), T, k, E, _p(offsets), int(align), _p(padded),
                                    _p(sorted_token), _p(row_of))
    if rc:
        raise ValueError(f"oracle_dispatch_padded: invalid routing ({rc})")
    return padded, sorted_token[:total], row_of


def gather_rows(x_bits, sorted_token):
    lib = _load()
    x_bits = _c(x_bits, np.uint16)
    sorted_token = _c(sorted_token, np.int32)
    H = x_bits.shape[1]
    out = np.zeros((sorted_token.shape[0], H), np.uint16)
    lib.oracle_gather_rows(_p(x_bits), H, _p(sorted_token), sorted_token.shape[0], _p(out))
    return out


def expert_mlp(x_bits, w_gu_bits, w_d_bits, round_bf16=True, want_intermediates=False):
    """One expert on rows x_bits [n,H]; w_gu_bits [H,2I], w_d_bits [I,H]."""
    lib = _load()
    x_bits = _c(x_bits, np.uint16)
    w_gu_bits = _c(w_gu_bits, np.uint16)
    w_d_bits = _c(w_d_bits, np.uint16)
    n, H = x_bits.shape
    I = w_d_bits.shape[0]
    y = np.zeros((n, H), np.float64)
    g = u = h = None
    if want_intermediates:
        g, u, h = (np.zeros((n, I), np.float64) for _ in range(3))
    lib.oracle_expert_mlp(_p(x_bits), n, H, I, _p(w_gu_bits), _p(w_d_bits), int(round_bf16),
                          _p(y), _p(g), _p(u), _p(h))
    return (y, g, u, h) if want_intermediates else y


def grouped_mlp(x_perm_bits, offsets, w_gu_bits, w_d_bits, round_bf16=True):
    lib = _load()
    x_perm_bits = _c(x_perm_bits, np.uint16)
    offsets = _c(offsets, np.int32)
    w_gu_bits = _c(w_gu_bits, np.uint16)
    w_d_bits = _c(w_d_bits, np.uint16)
    E, H, I2 = w_gu_bits.shape
    y = np.zeros((x_perm_bits.shape[0], H), np.float64)
    lib.oracle_grouped_mlp(_p(x_perm_bits), _p(offsets), E, H, I2 // 2, _p(w_gu_bits),
                           _p(w_d_bits), int(round_bf16), _p(y))
    return y


def combine(y_perm, row_of, probs=None, shared=None):
    lib = _load()
    y_perm = _c(y_perm, np.float64)
    row_of = _c(row_of, np.int32)
    T, k = row_of.shape
    H = y_perm.shape[1]
    out = np.zeros((T, H), np.float64)
    lib.oracle_combine(_p(y_perm), _p(row_of), _p(_c(probs, np.float32)), T, k, H,
                       _p(_c(shared, np.float64)), _p(out))
    return out


def _chunks(tokens, threads):
    tokens = np.asarray(tokens, np.int64)
    n = max(1, min(threads, len(tokens)))
    return [c for c in np.array_split(tokens, n) if len(c)]


def moe_forward_tokens(x_bits, logits, w_gu_bits, w_d_bits, k, tokens=None, score=0,
                       renormalize=True, scaling=1.0, expert_bias=None, shared_gu_bits=None,
                       shared_d_bits=None, round_bf16=True, threads=None):
    """The layer by its plain definition for the listed tokens (default: all);
    rows of the result are in list order (float64 [n, H])."""
    lib = _load()
    x_bits = _c(x_bits, np.uint16)
    logits = _c(logits, np.float32)
    w_gu_bits = _c(w_gu_bits, np.uint16)
    w_d_bits = _c(w_d_bits, np.uint16)
    shared_gu_bits = _c(shared_gu_bits, np.uint16)
    shared_d_bits = _c(shared_d_bits, np.uint16)
    expert_bias = _c(expert_bias, np.float32)
    T, H = x_bits.shape
    E, _, I2 = w_gu_bits.shape
    if tokens is None:
        tokens = np.arange(T, dtype=np.int64)
    tokens = np.asarray(tokens, np.int64)
    out = np.zeros((len(tokens), H), np.float64)
    threads = threads or os.cpu_count() or 1

    def run(chunk_and_start):
        chunk, start = chunk_and_start
        o = np.zeros((len(chunk), H), np.float64)
        rc = lib.oracle_moe_forward_tokens(_p(x_bits), _p(logits), H, I2 // 2, E, k, score,
                                           int(renormalize), scaling, _p(expert_bias),
                                           _p(w_gu_bits), _p(w_d_bits), _p(shared_gu_bits),
                                           _p(shared_d_bits), int(round_bf16), _p(chunk), len(chunk),
                                           _p(o))
        if rc:
            raise ValueError(f"oracle_moe_forward_tokens failed ({rc})")
        out[start:start + len(chunk)] = o

    chunks = _chunks(tokens, threads)
    starts = np.cumsum([0] + [len(c) for c in chunks[:-1]])
    with ThreadPoolExecutor(max_workers=len(chunks)) as ex:
        list(ex.map(run, zip(chunks, starts)))
    return out


def moe_backward(x_bits, topk_idx, topk_prob, w_gu_bits, w_d_bits, dout_bits, round_bf16=True,
                 only_expert=-1, tokens=None, want=("dx", "dw_gate_up", "dw_down", "dprob"),
                 threads=None, state=None, scaled=False):
    """Gradients of the layer for a given routing (see moe_oracle.c).

    scaled: the ScaledSwiGLU layer, with the routing weight applied to the
    SwiGLU output before FC2 and an unweighted combine
    (oracle_moe_backward_scaled); its saved state needs no y.

    state: None (the forward values are recomputed), or a saved forward state
    dict(row_of [T,k] int32, gu [rows,2I], h [rows,I], y [rows,H] as bf16 bit
    patterns) whose rows the chain rule reads instead
    (oracle_moe_backward_state).

    With a token list and only per-token outputs wanted (dx, dprob), the list
    is split over `threads` host threads (default: all cores); each token's
    rows are independent of the others, so the split changes nothing."""
    if tokens is not None and not ({"dw_gate_up", "dw_down"} & set(want)):
        tl = np.asarray(tokens, np.int64)
        chunks = _chunks(tl, threads or os.cpu_count() or 1)
        if len(chunks) > 1:
            def one(c):
                return moe_backward(x_bits, topk_idx, topk_prob, w_gu_bits, w_d_bits, dout_bits,
                                    round_bf16, only_expert, c, want, threads=1, state=state, scaled=scaled)
            with ThreadPoolExecutor(max_workers=len(chunks)) as ex:
                parts = list(ex.map(one, chunks))
            return {key: (None if parts[0][key] is None else np.concatenate([q[key] for q in parts]))
                    for key in ("dx", "dw_gate_up", "dw_down", "dprob")}
    lib = _load()
    x_bits = _c(x_bits, np.uint16)
    topk_idx = _c(topk_idx, np.int32)
    topk_prob = _c(topk_prob, np.float32)
    w_gu_bits = _c(w_gu_bits, np.uint16)
    w_d_bits = _c(w_d_bits, np.uint16)
    dout_bits = _c(dout_bits, np.uint16)
    T, H = x_bits.shape
    E, _, I2 = w_gu_bits.shape
    I = I2 // 2
    k = topk_idx.shape[1]
    tl = None if tokens is None else np.asarray(tokens, np.int64)
    nt = T if tl is None else len(tl)
    dx = np.zeros((nt, H)) if "dx" in want else None
    ne = 1 if only_expert >= 0 else E
    dwgu = np.zeros((ne, H, I2)) if "dw_gate_up" in want else None
    dwd = np.zeros((ne, I, H)) if "dw_down" in want else None
    dprob = np.zeros((nt, k)) if "dprob" in want else None
    st = [None] * 4
    if state is not None:
        st = [_c(state["row_of"], np.int32), _c(state["gu"], np.uint16), _c(state["h"], np.uint16),
              None if scaled else _c(state["y"], np.uint16)]
        rows = st[1].shape[0]
        if st[0].shape != (T, k) or st[2].shape != (rows, I) or (not scaled and st[3].shape != (rows, H)) or \
                st[1].shape != (rows, 2 * I) or (st[0].size and (st[0].min() < 0 or st[0].max() >= rows)):
            raise ValueError("moe_backward: state shapes do not match")
    if scaled:
        rc = lib.oracle_moe_backward_scaled(_p(x_bits), T, H, I, E, k, _p(topk_idx), _p(topk_prob),
                                            _p(w_gu_bits), _p(w_d_bits), _p(dout_bits), int(round_bf16),
                                            only_expert, _p(tl), 0 if tl is None else len(tl),
                                            _p(st[0]), _p(st[1]), _p(st[2]),
                                            _p(dx), _p(dwgu), _p(dwd), _p(dprob))
        if rc:
            raise ValueError(f"oracle_moe_backward_scaled failed ({rc})")
        return dict(dx=dx, dw_gate_up=dwgu, dw_down=dwd, dprob=dprob)
    rc = lib.oracle_moe_backward_state(_p(x_bits), T, H, I, E, k, _p(topk_idx), _p(topk_prob),
                                       _p(w_gu_bits), _p(w_d_bits), _p(dout_bits), int(round_bf16),
                                       only_expert, _p(tl), 0 if tl is None else len(tl),
                                       _p(st[0]), _p(st[1]), _p(st[2]), _p(st[3]),
                                       _p(dx), _p(dwgu), _p(dwd), _p(dprob))
    if rc:
        raise ValueError(f"oracle_moe_backward failed ({rc})")
    return dict(dx=dx, dw_gate_up=dwgu, dw_down=dwd, dprob=dprob)
