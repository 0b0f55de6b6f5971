"""Python binding of libswitchmoe.so (the C ABI in include/switch_moe.h).

Argument marshalling only: every function here turns torch tensors into
device pointers, the current CUDA stream into a handle, and a non-OK status
into a SwitchError.  All arithmetic of the layer runs in the CUDA library;
there is no CPU or PyTorch fallback, and importing this module fails loudly
when the library is missing.
"""
import ctypes
import os
from ctypes import POINTER, c_double, c_float, c_int32, c_int64, c_size_t, c_void_p, c_char_p

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libswitchmoe.so")

SWITCH_OK = 0
STATUS_NAMES = {0: "SWITCH_OK", 1: "SWITCH_ERR_INVALID_ARG", 2: "SWITCH_ERR_UNSUPPORTED",
                3: "SWITCH_ERR_WORKSPACE_TOO_SMALL", 4: "SWITCH_ERR_CUDA",
                5: "SWITCH_ERR_TIMEOUT", 6: "SWITCH_ERR_DEVICE_BOUNDS"}
SWITCH_F32, SWITCH_BF16 = 0, 1
FLAG_ROUTER_SIMT = 1
FLAG_ROUTER_3TERM = 2
FLAG_UNFUSED_COMBINE = 4
FLAG_GATHER_IN_GEMM = 8
FLAG_NO_RESIDUAL = 16
FLAG_GEMM_1SM = 32
FLAG_GEMM_PAIRS = 64
FLAG_ROWS_DISPATCHED = 128
FLAG_TOP2 = 512
FLAG_TRAINING = 1024
FLAG_GEMM1_ROWS_PAIRS = 2048


class SwitchConfig(ctypes.Structure):
    _fields_ = [("T", c_int64), ("d_model", c_int32), ("d_ff", c_int32),
                ("n_experts", c_int32), ("dtype", c_int32),
                ("capacity_factor", c_double), ("alpha", c_float), ("flags", c_int32),
                ("spin_limit", c_int64)]


class SwitchEp(ctypes.Structure):
    """Expert-parallel group: world_size ranks, this one `rank`."""
    _fields_ = [("world_size", c_int32), ("rank", c_int32)]


class SwitchError(RuntimeError):
    def __init__(self, status, where=None):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{where or 'switch'}: {name}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m sparse_mixture_experts_switch_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    cfgp = POINTER(SwitchConfig)
    sig = {
        "switch_capacity": (c_int64, [c_int64, c_int32, c_double]),
        "switch_workspace_size": (c_int32, [cfgp, POINTER(c_size_t)]),
        "switch_router": (c_int32, [cfgp, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_void_p, c_size_t, c_void_p]),
        "switch_dispatch": (c_int32, [cfgp, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                      c_void_p]),
        "switch_dispatch_noalloc": (c_int32, [cfgp, c_void_p, c_void_p, c_void_p, c_void_p,
                                              c_void_p, c_void_p, c_void_p]),
        "switch_expert_ffn": (c_int32, [cfgp, c_void_p, c_void_p, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
        "switch_combine": (c_int32, [cfgp, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_void_p]),
        "switch_aux_loss": (c_int32, [cfgp, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_size_t, c_void_p]),
        "switch_layer_forward": (c_int32, [cfgp, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_void_p, c_void_p, c_size_t, c_void_p]),
        "switch_layer_backward": (c_int32, [cfgp, c_void_p, c_void_p, c_void_p, c_void_p,
                                            c_void_p, c_void_p, c_float, c_void_p, c_void_p,
                                            c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                            c_size_t, c_void_p]),
        "switch_backward_workspace_size": (c_int32, [cfgp, POINTER(c_size_t)]),
        "switch_get_device_error": (c_int32, [c_void_p, c_void_p, POINTER(c_int32),
                                              POINTER(c_int64)]),
        "switch_status_string": (c_char_p, [c_int32]),
        "switch_ep_sizes": (c_int32, [cfgp, POINTER(SwitchEp), POINTER(c_size_t),
                                      POINTER(c_size_t), POINTER(c_size_t)]),
        "switch_ep_route": (c_int32, [cfgp, POINTER(SwitchEp), c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                      c_void_p]),
        "switch_ep_dispatch": (c_int32, [cfgp, POINTER(SwitchEp), c_void_p, c_void_p,
                                         POINTER(c_void_p), c_void_p, c_void_p, c_void_p,
                                         c_void_p, c_size_t, c_void_p]),
        "switch_ep_experts": (c_int32, [cfgp, POINTER(SwitchEp), c_void_p, c_void_p, c_void_p,
                                        POINTER(c_void_p), c_void_p, c_size_t, c_void_p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


# ------------------------------------------------------------- marshalling

def _p(t):
    """Device pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensors only: the library reads device memory")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status, where):
    if status != SWITCH_OK:
        raise SwitchError(status, where)


def config(T, d_model, d_ff, n_experts, capacity_factor, dtype="bf16", alpha=0.01,
           flags=0, spin_limit=0):
    dt = {"bf16": SWITCH_BF16, "f32": SWITCH_F32}[dtype] if isinstance(dtype, str) else dtype
    return SwitchConfig(T, d_model, d_ff, n_experts, dt, float(capacity_factor),
                        float(alpha), flags, spin_limit)


def switch_capacity(T, n_experts, capacity_factor):
    return _lib.switch_capacity(T, n_experts, float(capacity_factor))


def switch_workspace_size(cfg):
    n = c_size_t(0)
    _check(_lib.switch_workspace_size(ctypes.byref(cfg), ctypes.byref(n)),
           "switch_workspace_size")
    return n.value


def workspace(cfg, device="cuda"):
    """A zero-filled device workspace of switch_workspace_size(cfg) bytes."""
    return torch.zeros(max(switch_workspace_size(cfg), 1), dtype=torch.uint8, device=device)


def switch_router(cfg, x, w_r, b_r, idx, gate, probs, ws, stream=None):
    _check(_lib.switch_router(ctypes.byref(cfg), _p(x), _p(w_r), _p(b_r), _p(idx), _p(gate),
                              _p(probs), _p(ws), ws.numel(), _stream(stream)), "switch_router")


def switch_dispatch(cfg, idx, probs, rank, drop, counts, slot_token, x, x_disp, ws,
                    stream=None):
    _check(_lib.switch_dispatch(ctypes.byref(cfg), _p(idx), _p(probs), _p(rank), _p(drop),
                                _p(counts), _p(slot_token), _p(x), _p(x_disp), _p(ws),
                                ws.numel(), _stream(stream)), "switch_dispatch")


def switch_dispatch_noalloc(cfg, idx, probs, rank, drop, counts, slot_token, stream=None):
    """switch_dispatch without a workspace, for callers that cannot allocate
    device memory (scratch lives in a fixed array inside the library)."""
    _check(_lib.switch_dispatch_noalloc(ctypes.byref(cfg), _p(idx), _p(probs), _p(rank),
                                        _p(drop), _p(counts), _p(slot_token), _stream(stream)),
           "switch_dispatch_noalloc")


def switch_expert_ffn(cfg, x, slot_token, counts, w1, w2, y, ws, stream=None):
    _check(_lib.switch_expert_ffn(ctypes.byref(cfg), _p(x), _p(slot_token), _p(counts),
                                  _p(w1), _p(w2), _p(y), _p(ws), ws.numel(),
                                  _stream(stream)), "switch_expert_ffn")


def switch_combine(cfg, x_residual, idx, rank, drop, gate, y, out, stream=None):
    _check(_lib.switch_combine(ctypes.byref(cfg), _p(x_residual), _p(idx), _p(rank), _p(drop),
                               _p(gate), _p(y), _p(out), _stream(stream)), "switch_combine")


def switch_aux_loss(cfg, counts, probs, loss, f, P, ws, stream=None):
    _check(_lib.switch_aux_loss(ctypes.byref(cfg), _p(counts), _p(probs), _p(loss), _p(f),
                                _p(P), _p(ws), ws.numel(), _stream(stream)),
           "switch_aux_loss")


def switch_layer_forward(cfg, x, w_r, b_r, w1, w2, out, idx, gate, counts, loss, ws,
                         stream=None):
    _check(_lib.switch_layer_forward(ctypes.byref(cfg), _p(x), _p(w_r), _p(b_r), _p(w1),
                                     _p(w2), _p(out), _p(idx), _p(gate), _p(counts),
                                     _p(loss), _p(ws), ws.numel(), _stream(stream)),
           "switch_layer_forward")


def switch_backward_workspace_size(cfg):
    n = c_size_t(0)
    _check(_lib.switch_backward_workspace_size(ctypes.byref(cfg), ctypes.byref(n)),
           "switch_backward_workspace_size")
    return n.value


def backward_workspace(cfg, device="cuda"):
    """A zero-filled device workspace of switch_backward_workspace_size(cfg)
    bytes (every entry point accepts it)."""
    return torch.zeros(max(switch_backward_workspace_size(cfg), 1), dtype=torch.uint8,
                       device=device)


def switch_layer_backward(cfg, x, w_r, b_r, w1, w2, dout, dloss, dx, dw_r, db_r, dw1, dw2,
                          dgate, ws, stream=None):
    _check(_lib.switch_layer_backward(ctypes.byref(cfg), _p(x), _p(w_r), _p(b_r), _p(w1),
                                      _p(w2), _p(dout), float(dloss), _p(dx), _p(dw_r),
                                      _p(db_r), _p(dw1), _p(dw2), _p(dgate), _p(ws),
                                      ws.numel(), _stream(stream)), "switch_layer_backward")


# ----------------------------------------------------- expert parallelism

def ep(world_size, rank):
    return SwitchEp(world_size, rank)


def switch_ep_sizes(cfg, ep_):
    """(workspace bytes, exchange-record bytes, receive-buffer bytes)."""
    a, b, c = c_size_t(0), c_size_t(0), c_size_t(0)
    _check(_lib.switch_ep_sizes(ctypes.byref(cfg), ctypes.byref(ep_), ctypes.byref(a),
                                ctypes.byref(b), ctypes.byref(c)), "switch_ep_sizes")
    return a.value, b.value, c.value


def _ptr_array(ptrs):
    arr = (c_void_p * len(ptrs))()
    for i, v in enumerate(ptrs):
        arr[i] = v if isinstance(v, int) else _p(v)
    return arr


def switch_ep_route(cfg, ep_, x, w_r, b_r, idx, gate, record, ws, stream=None):
    _check(_lib.switch_ep_route(ctypes.byref(cfg), ctypes.byref(ep_), _p(x), _p(w_r), _p(b_r),
                                _p(idx), _p(gate), _p(record), _p(ws), ws.numel(),
                                _stream(stream)), "switch_ep_route")


def switch_ep_dispatch(cfg, ep_, x, records, recv_peers, out, counts, loss, ws, stream=None):
    """recv_peers: the G ranks' receive buffers (tensors, or device addresses
    as ints for buffers mapped from other processes)."""
    _check(_lib.switch_ep_dispatch(ctypes.byref(cfg), ctypes.byref(ep_), _p(x), _p(records),
                                   _ptr_array(recv_peers), _p(out), _p(counts), _p(loss),
                                   _p(ws), ws.numel(), _stream(stream)), "switch_ep_dispatch")


def switch_ep_experts(cfg, ep_, w1_local, w2_local, recv, out_peers, ws, stream=None):
    """out_peers: the G ranks' outputs (tensors or device addresses)."""
    _check(_lib.switch_ep_experts(ctypes.byref(cfg), ctypes.byref(ep_), _p(w1_local),
                                  _p(w2_local), _p(recv), _ptr_array(out_peers), _p(ws),
                                  ws.numel(), _stream(stream)), "switch_ep_experts")


def switch_get_device_error(ws, stream=None):
    """(status, where, info); synchronises the stream and clears the word."""
    where = c_int32(0)
    info = c_int64(0)
    st = _lib.switch_get_device_error(_p(ws), _stream(stream), ctypes.byref(where),
                                      ctypes.byref(info))
    return st, where.value, info.value


def switch_status_string(status):
    return _lib.switch_status_string(status).decode()
