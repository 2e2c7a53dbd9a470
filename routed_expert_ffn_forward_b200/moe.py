"""ctypes binding of libmoe.so (include/moe.h), same names as the C ABI.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Pointers are passed as Python ints (``tensor.data_ptr()``) and
streams as ints (``torch.cuda.Stream().cuda_stream``) or None.  A call whose
status is not MOE_OK raises MoEError carrying the status and moe_last_error().
Loading fails loudly if the library has not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LIB_VARIANT=debug loads the bounds-checking build (libmoe_debug.so)
LIB_PATH = os.path.join(_HERE, "libmoe_debug.so" if os.environ.get("MOE_LIB_VARIANT") == "debug" else "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_OOM = -3
MOE_ERR_CUDA = -4
MOE_ERR_CACHE_TOO_SMALL = -5
MOE_ERR_NOT_READY = -6
STATUS_NAMES = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_OOM",
                -4: "MOE_ERR_CUDA", -5: "MOE_ERR_CACHE_TOO_SMALL", -6: "MOE_ERR_NOT_READY"}

MOE_Q8_0 = 8
MOE_Q4_K = 12
MOE_Q5_K = 13
MOE_Q6_K = 14
MOE_MXFP4 = 39
MOE_CACHE_LRU = 0
MOE_CACHE_LFU = 1
MOE_GATE_SOFTMAX_TOPK = 0
MOE_GATE_SIGMOID_RENORM = 1
SIZE_MAX = (1 << 64) - 1

# every entry point declared in include/moe.h
EXPORTS = ("moe_expert_bytes", "moe_layer_create", "moe_layer_create_mixed", "moe_layer_destroy", "moe_set_router",
           "moe_set_experts", "moe_set_cache_bytes", "moe_set_cache_policy", "moe_set_few_row_tiles", "moe_forward", "moe_forward_routed",
           "moe_forward_host", "moe_get_routing", "moe_get_logits", "moe_prefetch",
           "moe_check", "moe_get_stats", "moe_reset_stats", "moe_set_profiling", "moe_get_profile",
           "moe_reset_profile", "moe_route_noalloc", "moe_set_test_hooks", "moe_set_expert_parallel",
           "moe_forward_partial", "moe_combine_partials", "moe_last_error")

KERNELS = ("router", "topk", "permute", "gate_up", "down", "combine", "prep", "small", "forward", "fused",
           "few_gate_up", "few_down")


class moe_stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "forwards", "tokens", "decode_calls", "prefill_calls", "cache_hits", "cache_misses",
        "prefetches", "evictions", "h2d_bytes", "cache_slots", "slot_bytes", "launches")]

    def as_dict(self) -> dict:
        return {n: int(getattr(self, n)) for n, _ in self._fields_}


class moe_profile(ctypes.Structure):
    _fields_ = [("forwards", ctypes.c_uint64), ("ms", ctypes.c_double * len(KERNELS)),
                ("launches", ctypes.c_uint64 * len(KERNELS))]

    def as_dict(self) -> dict:
        return {"forwards": int(self.forwards),
                "ms": {k: float(self.ms[i]) for i, k in enumerate(KERNELS)},
                "launches": {k: int(self.launches[i]) for i, k in enumerate(KERNELS)}}


class MoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int


def lib() -> ctypes.CDLL:
    """Load libmoe.so (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built: run `python -m routed_expert_ffn_forward_b200.build`"
                              + (" --debug-bounds" if LIB_PATH.endswith("_debug.so") else ""))
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "moe_expert_bytes": (ctypes.c_size_t, [_I, _I, _I]),
            "moe_layer_create": (_I, [_I, _I, _I, _I, _I, _I, ctypes.POINTER(_P)]),
            "moe_layer_create_mixed": (_I, [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_P)]),
            "moe_layer_destroy": (_I, [_P]),
            "moe_set_router": (_I, [_P, _P, _P, _I]),
            "moe_set_experts": (_I, [_P, _P, _P, _P]),
            "moe_set_cache_bytes": (_I, [ctypes.c_size_t]),
            "moe_set_cache_policy": (_I, [_I]),
            "moe_set_few_row_tiles": (_I, [_I]),
            "moe_forward": (_I, [_P, _P, _P, _I, _P]),
            "moe_forward_routed": (_I, [_P, _P, _P, _I, _P, _P]),
            "moe_forward_host": (_I, [_P, _P, _P, _I, _P]),
            "moe_get_routing": (_I, [_P, _P, _P, _P]),
            "moe_get_logits": (_I, [_P, _P, _P]),
            "moe_prefetch": (_I, [_P, _P, _I]),
            "moe_check": (_I, [_P]),
            "moe_get_stats": (_I, [ctypes.POINTER(moe_stats)]),
            "moe_reset_stats": (_I, []),
            "moe_set_profiling": (_I, [_I]),
            "moe_get_profile": (_I, [ctypes.POINTER(moe_profile)]),
            "moe_reset_profile": (_I, []),
            "moe_route_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
            "moe_set_test_hooks": (_I, [ctypes.c_uint64, _I]),
            "moe_set_expert_parallel": (_I, [_P, _I, _I]),
            "moe_forward_partial": (_I, [_P, _P, _P, _I, _P]),
            "moe_combine_partials": (_I, [_P, _P, _I, _I, _I, _P]),
            "moe_last_error": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != MOE_OK:
        raise MoEError(status, (lib().moe_last_error() or b"").decode())


def _ptr_array(ptrs) -> ctypes.Array:
    return (_P * len(ptrs))(*[int(p) for p in ptrs])


# ---------------------------------------------------------------- entry points
def moe_expert_bytes(hidden: int, inter: int, quant: int = MOE_Q4_K) -> int:
    return int(lib().moe_expert_bytes(hidden, inter, quant))


def moe_layer_create(hidden: int, inter: int, n_experts: int, top_k: int, n_shared: int,
                     quant: int = MOE_Q4_K) -> int:
    h = _P()
    _check(lib().moe_layer_create(hidden, inter, n_experts, top_k, n_shared, quant, ctypes.byref(h)))
    return int(h.value)


def moe_layer_create_mixed(hidden: int, inter: int, n_experts: int, top_k: int, n_shared: int,
                           quant_gate_up: int, quant_down: int) -> int:
    h = _P()
    _check(lib().moe_layer_create_mixed(hidden, inter, n_experts, top_k, n_shared, quant_gate_up, quant_down,
                                        ctypes.byref(h)))
    return int(h.value)


def moe_layer_destroy(layer: int) -> None:
    _check(lib().moe_layer_destroy(layer))


def moe_set_router(layer: int, W: int, bias: int | None, gating: int) -> None:
    _check(lib().moe_set_router(layer, W, bias or None, gating))


def moe_set_experts(layer: int, gate_ptrs, up_ptrs, down_ptrs) -> None:
    _check(lib().moe_set_experts(layer, _ptr_array(gate_ptrs), _ptr_array(up_ptrs), _ptr_array(down_ptrs)))


def moe_set_cache_bytes(nbytes: int) -> None:
    _check(lib().moe_set_cache_bytes(nbytes))


def moe_set_cache_policy(policy: int) -> None:
    _check(lib().moe_set_cache_policy(policy))


def moe_set_few_row_tiles(max_rows: int) -> None:
    _check(lib().moe_set_few_row_tiles(max_rows))


def moe_forward(layer: int, x: int, out: int, T: int, stream: int | None = None) -> None:
    _check(lib().moe_forward(layer, x, out, T, stream or None))


def moe_forward_routed(layer: int, x: int, out: int, T: int, forced_ids_host: int,
                       stream: int | None = None) -> None:
    _check(lib().moe_forward_routed(layer, x, out, T, forced_ids_host, stream or None))


def moe_forward_host(layer: int, x_host: int, out_host: int, T: int, stream: int | None = None) -> None:
    _check(lib().moe_forward_host(layer, x_host, out_host, T, stream or None))


def moe_get_routing(layer: int, ids: int | None, weights: int | None, stream: int | None = None) -> None:
    _check(lib().moe_get_routing(layer, ids or None, weights or None, stream or None))


def moe_get_logits(layer: int, logits: int, stream: int | None = None) -> None:
    _check(lib().moe_get_logits(layer, logits, stream or None))


def moe_prefetch(layer: int, ids_host: int, n: int) -> None:
    _check(lib().moe_prefetch(layer, ids_host, n))


def moe_check(layer: int) -> None:
    _check(lib().moe_check(layer))


def moe_get_stats() -> dict:
    s = moe_stats()
    _check(lib().moe_get_stats(ctypes.byref(s)))
    return s.as_dict()


def moe_reset_stats() -> None:
    _check(lib().moe_reset_stats())


def moe_set_profiling(enable: bool) -> None:
    _check(lib().moe_set_profiling(1 if enable else 0))


def moe_get_profile() -> dict:
    p = moe_profile()
    _check(lib().moe_get_profile(ctypes.byref(p)))
    return p.as_dict()


def moe_reset_profile() -> None:
    _check(lib().moe_reset_profile())


def moe_route_noalloc(x: int, W: int, bias: int | None, T: int, H: int, E: int, top_k: int, gating: int,
                      ids: int, weights: int, stream: int | None = None) -> None:
    _check(lib().moe_route_noalloc(x, W, bias or None, T, H, E, top_k, gating, ids, weights, stream or None))


def moe_set_expert_parallel(layer: int, rank: int, world: int) -> None:
    _check(lib().moe_set_expert_parallel(layer, rank, world))


def moe_forward_partial(layer: int, x: int, partial: int, T: int, stream: int | None = None) -> None:
    _check(lib().moe_forward_partial(layer, x, partial, T, stream or None))


def moe_combine_partials(partials: int, out: int, T: int, H: int, world: int, stream: int | None = None) -> None:
    _check(lib().moe_combine_partials(partials, out, T, H, world, stream or None))


def moe_set_test_hooks(wait_limit_ns: int, hold_barrier: int) -> None:
    _check(lib().moe_set_test_hooks(wait_limit_ns, hold_barrier))


def moe_last_error() -> str:
    return (lib().moe_last_error() or b"").decode()
