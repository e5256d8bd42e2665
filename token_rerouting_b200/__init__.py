"""Python binding of libue, the sm_100a exact-load rebalancing hot path.

Argument marshalling only: every step of the path runs in the CUDA kernels
behind include/ue.h. PyTorch is used by callers for device memory and
streams; tensors are passed by ``data_ptr()``. There is no CPU fallback: if
``libue.so`` is missing the import of the library fails loudly (build it with
``python -m token_rerouting_b200.build``).

The functions carry the C names: ``ue_init``, ``ue_gate_topk``, ``ue_count``,
``ue_plan``, ``ue_reroute``, ``ue_permute``, ``ue_combine``, ``ue_get_error``,
``ue_destroy``, the planner variants ``ue_plan_ex``, ``ue_reroute_ex``,
``ue_locality_split``, ``ue_reroute_local``, and the rows beside the forward
path (see include/ue.h for the contract of each).
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libue.so")

STATUS = {
    0: "UE_OK",
    1: "UE_ERR_INVALID_ARG",
    2: "UE_ERR_CUDA",
    3: "UE_ERR_NOMEM",
    4: "UE_ERR_DEVICE_BOUNDS",
    5: "UE_ERR_TIMEOUT",
    6: "UE_ERR_UNSUPPORTED",
}
UE_OK, UE_ERR_INVALID_ARG, UE_ERR_CUDA, UE_ERR_NOMEM = 0, 1, 2, 3
UE_ERR_DEVICE_BOUNDS, UE_ERR_TIMEOUT, UE_ERR_UNSUPPORTED = 4, 5, 6

# every symbol include/ue.h declares
EXPORTS = ("ue_init", "ue_destroy", "ue_get_error", "ue_gate_topk", "ue_count", "ue_gate_count",
           "ue_plan", "ue_plan_ex", "ue_reroute", "ue_plan_reroute", "ue_reroute_ex",
           "ue_locality_split",
           "ue_reroute_local", "ue_permute", "ue_combine", "ue_combine_backward",
           "ue_permute_backward", "ue_weight_sync", "ue_grad_reduce", "ue_reroute_noalloc",
           "ue_debug_set_lookback_limit", "ue_debug_drop_first_publish")


class UEError(RuntimeError):
    def __init__(self, call: str, code: int):
        super().__init__(f"{call} returned {STATUS.get(code, code)}")
        self.code = code


class ue_config(ctypes.Structure):
    _fields_ = [("R", ctypes.c_int32), ("T", ctypes.c_int32), ("E", ctypes.c_int32),
                ("K", ctypes.c_int32), ("S", ctypes.c_int32), ("d", ctypes.c_int32)]


class ue_placement(ctypes.Structure):
    _fields_ = [("slot_expert", ctypes.c_void_p), ("n_copies", ctypes.c_void_p),
                ("slot_quota", ctypes.c_void_p), ("slot_offset", ctypes.c_void_p),
                ("rank_load", ctypes.c_void_p), ("stats", ctypes.c_void_p)]


UE_SOLVER_GREEDY, UE_SOLVER_BISECT = 0, 1
UE_ORDER_PREFIX, UE_ORDER_INTERLEAVE = 0, 1


class ue_plan_opts(ctypes.Structure):
    _fields_ = [("solver", ctypes.c_int32), ("min_tokens", ctypes.c_int32),
                ("eps_inv", ctypes.c_int32), ("threshold", ctypes.c_int32),
                ("allow_zero_master", ctypes.c_int32)]


def plan_opts(solver: int = UE_SOLVER_GREEDY, min_tokens: int | None = None, eps_inv: int = 100,
              threshold: int | None = None, allow_zero_master: bool = False) -> ue_plan_opts:
    """Planner options; the defaults are the pages' (minimum 1024 pairs per
    replica and eps 0.01, early stop at 1.0, for the bisection; no minimum for
    the greedy)."""
    if min_tokens is None:
        min_tokens = 1024 if solver == UE_SOLVER_BISECT else 0
    return ue_plan_opts(solver, min_tokens, eps_inv,
                        eps_inv if threshold is None else threshold, int(bool(allow_zero_master)))


_lib = None


def load_library(path: str | None = None):
    """Load libue.so (once). Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"libue.so not found at {p}; build it with `python -m token_rerouting_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.ue_init.argtypes = [ctypes.POINTER(ue_config), i32, ctypes.POINTER(vp)]
    lib.ue_destroy.argtypes = [vp]
    lib.ue_get_error.argtypes = [vp, vp]
    lib.ue_gate_topk.argtypes = [vp, vp, vp, vp, vp]
    lib.ue_gate_count.argtypes = [vp, vp, vp, vp, vp, vp, vp]
    lib.ue_count.argtypes = [vp, vp, vp, vp, vp]
    lib.ue_plan.argtypes = [vp, vp, ctypes.POINTER(ue_placement), vp]
    lib.ue_plan_ex.argtypes = [vp, vp, ctypes.POINTER(ue_plan_opts), ctypes.POINTER(ue_placement),
                               vp]
    lib.ue_reroute.argtypes = [vp, vp, ctypes.POINTER(ue_placement), vp, vp, vp]
    lib.ue_plan_reroute.argtypes = [vp, vp, vp, ctypes.POINTER(ue_placement), vp, vp, vp]
    lib.ue_reroute_ex.argtypes = [vp, vp, ctypes.POINTER(ue_placement), i32, vp, vp, vp]
    lib.ue_locality_split.argtypes = [vp, vp, ctypes.POINTER(ue_placement), vp, vp, vp]
    lib.ue_reroute_local.argtypes = [vp, vp, vp, ctypes.POINTER(ue_placement), vp, vp, vp, vp,
                                     vp]
    lib.ue_permute.argtypes = [vp, vp, vp, vp, vp]
    lib.ue_combine.argtypes = [vp, vp, vp, vp, vp, vp]
    lib.ue_combine_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
    lib.ue_permute_backward.argtypes = [vp, vp, vp, vp, vp]
    lib.ue_weight_sync.argtypes = [vp, ctypes.POINTER(ue_placement), vp, vp, i64, vp]
    lib.ue_grad_reduce.argtypes = [vp, ctypes.POINTER(ue_placement), vp, vp, i64, vp]
    lib.ue_reroute_noalloc.argtypes = [ctypes.POINTER(ue_config), vp,
                                       ctypes.POINTER(ue_placement), vp, vp, vp, vp]
    lib.ue_debug_set_lookback_limit.argtypes = [vp, i64]
    lib.ue_debug_drop_first_publish.argtypes = [vp, i32]
    for name in EXPORTS:
        getattr(lib, name).restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def _ptr(x):
    """Device (or host) address of a tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ok(call, rc):
    if rc != UE_OK:
        raise UEError(call, rc)


def make_config(R, T, E, K, S, d) -> ue_config:
    return ue_config(R, T, E, K, S, d)


def ue_init(cfg: ue_config, device: int = 0):
    """Create a context (opaque handle) for one simulated EP group."""
    lib = load_library()
    h = ctypes.c_void_p()
    _ok("ue_init", lib.ue_init(ctypes.byref(cfg), device, ctypes.byref(h)))
    return h


def ue_destroy(ctx):
    _ok("ue_destroy", load_library().ue_destroy(ctx))


def ue_get_error(ctx, stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error code."""
    return load_library().ue_get_error(ctx, _stream(stream))


def ue_gate_topk(ctx, logits, idx, w, stream=None):
    _ok("ue_gate_topk", load_library().ue_gate_topk(ctx, _ptr(logits), _ptr(idx), _ptr(w),
                                                    _stream(stream)))


def ue_gate_count(ctx, logits, idx, w, load_re, load_e, stream=None):
    _ok("ue_gate_count", load_library().ue_gate_count(ctx, _ptr(logits), _ptr(idx), _ptr(w),
                                                      _ptr(load_re), _ptr(load_e),
                                                      _stream(stream)))


def ue_count(ctx, idx, load_re, load_e, stream=None):
    _ok("ue_count", load_library().ue_count(ctx, _ptr(idx), _ptr(load_re), _ptr(load_e),
                                            _stream(stream)))


def placement(slot_expert, n_copies, slot_quota, slot_offset, rank_load, stats) -> ue_placement:
    """ue_placement from six int32 device tensors (slot_expert may be None)."""
    return ue_placement(_ptr(slot_expert), _ptr(n_copies), _ptr(slot_quota),
                        _ptr(slot_offset), _ptr(rank_load), _ptr(stats))


def ue_plan(ctx, load_e, plan: ue_placement, stream=None):
    _ok("ue_plan", load_library().ue_plan(ctx, _ptr(load_e), ctypes.byref(plan),
                                          _stream(stream)))


def ue_plan_ex(ctx, load_e, opts: ue_plan_opts, plan: ue_placement, stream=None):
    _ok("ue_plan_ex", load_library().ue_plan_ex(ctx, _ptr(load_e), ctypes.byref(opts),
                                                ctypes.byref(plan), _stream(stream)))


def ue_reroute_ex(ctx, idx, plan: ue_placement, order: int, phys_slot, dest_row, stream=None):
    _ok("ue_reroute_ex", load_library().ue_reroute_ex(ctx, _ptr(idx), ctypes.byref(plan), order,
                                                      _ptr(phys_slot), _ptr(dest_row),
                                                      _stream(stream)))


def ue_locality_split(ctx, load_re, plan: ue_placement, src_quota, src_offset, stream=None):
    _ok("ue_locality_split",
        load_library().ue_locality_split(ctx, _ptr(load_re), ctypes.byref(plan), _ptr(src_quota),
                                         _ptr(src_offset), _stream(stream)))


def ue_reroute_local(ctx, idx, load_re, plan: ue_placement, src_quota, src_offset, phys_slot,
                     dest_row, stream=None):
    _ok("ue_reroute_local",
        load_library().ue_reroute_local(ctx, _ptr(idx), _ptr(load_re), ctypes.byref(plan),
                                        _ptr(src_quota), _ptr(src_offset), _ptr(phys_slot),
                                        _ptr(dest_row), _stream(stream)))


def ue_reroute(ctx, idx, plan: ue_placement, phys_slot, dest_row, stream=None):
    _ok("ue_reroute", load_library().ue_reroute(ctx, _ptr(idx), ctypes.byref(plan),
                                                _ptr(phys_slot), _ptr(dest_row),
                                                _stream(stream)))


def ue_plan_reroute(ctx, load_e, idx, plan: ue_placement, phys_slot, dest_row, stream=None):
    _ok("ue_plan_reroute",
        load_library().ue_plan_reroute(ctx, _ptr(load_e), _ptr(idx), ctypes.byref(plan),
                                       _ptr(phys_slot), _ptr(dest_row), _stream(stream)))


def ue_permute(ctx, hidden, dest_row, dispatch, stream=None):
    _ok("ue_permute", load_library().ue_permute(ctx, _ptr(hidden), _ptr(dest_row),
                                                _ptr(dispatch), _stream(stream)))


def ue_combine(ctx, y, dest_row, w, out, stream=None):
    _ok("ue_combine", load_library().ue_combine(ctx, _ptr(y), _ptr(dest_row), _ptr(w),
                                                _ptr(out), _stream(stream)))


def ue_combine_backward(ctx, dout, y, dest_row, w, dy, dw, stream=None):
    _ok("ue_combine_backward",
        load_library().ue_combine_backward(ctx, _ptr(dout), _ptr(y), _ptr(dest_row), _ptr(w),
                                           _ptr(dy), _ptr(dw), _stream(stream)))


def ue_permute_backward(ctx, ddispatch, dest_row, dhidden, stream=None):
    _ok("ue_permute_backward",
        load_library().ue_permute_backward(ctx, _ptr(ddispatch), _ptr(dest_row), _ptr(dhidden),
                                           _stream(stream)))


def ue_weight_sync(ctx, plan: ue_placement, master, replicas, bytes_per_expert: int,
                   stream=None):
    _ok("ue_weight_sync",
        load_library().ue_weight_sync(ctx, ctypes.byref(plan), _ptr(master), _ptr(replicas),
                                      bytes_per_expert, _stream(stream)))


def ue_grad_reduce(ctx, plan: ue_placement, replica_grads, master_grads, numel_per_expert: int,
                   stream=None):
    _ok("ue_grad_reduce",
        load_library().ue_grad_reduce(ctx, ctypes.byref(plan), _ptr(replica_grads),
                                      _ptr(master_grads), numel_per_expert, _stream(stream)))


def ue_reroute_noalloc(cfg: ue_config, idx, plan: ue_placement, phys_slot, dest_row,
                       error=None, stream=None):
    """ue_reroute without a context; allocates nothing (see include/ue.h)."""
    _ok("ue_reroute_noalloc",
        load_library().ue_reroute_noalloc(ctypes.byref(cfg), _ptr(idx), ctypes.byref(plan),
                                          _ptr(phys_slot), _ptr(dest_row), _ptr(error),
                                          _stream(stream)))


def ue_debug_set_lookback_limit(ctx, polls: int):
    _ok("ue_debug_set_lookback_limit",
        load_library().ue_debug_set_lookback_limit(ctx, polls))


def ue_debug_drop_first_publish(ctx, enable: bool):
    _ok("ue_debug_drop_first_publish",
        load_library().ue_debug_drop_first_publish(ctx, 1 if enable else 0))


from .layer import Layer  # noqa: E402  (buffers + one call per step)

__all__ = ["ue_init", "ue_destroy", "ue_get_error", "ue_gate_topk", "ue_count", "ue_gate_count", "ue_plan",
           "ue_plan_ex", "ue_reroute_ex", "ue_locality_split", "ue_reroute_local",
           "ue_plan_opts", "plan_opts", "UE_SOLVER_GREEDY", "UE_SOLVER_BISECT",
           "UE_ORDER_PREFIX", "UE_ORDER_INTERLEAVE",
           "ue_reroute", "ue_plan_reroute", "ue_permute", "ue_combine", "ue_combine_backward",
           "ue_permute_backward", "ue_weight_sync", "ue_grad_reduce", "ue_reroute_noalloc",
           "ue_debug_set_lookback_limit",
           "ue_debug_drop_first_publish", "ue_config", "ue_placement", "make_config",
           "placement", "load_library", "Layer", "UEError", "STATUS", "EXPORTS"]
