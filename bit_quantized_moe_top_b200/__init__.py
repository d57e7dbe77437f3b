"""Python binding of the B200 quantized MoE expert layer (``libmoeq.so``).

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels of the shared library; torch is used for device memory and streams.
The functions carry the C ABI's names (see ``include/moe_layer.h``); the
``MoELayer`` class is a small convenience wrapper over them. Importing this
package fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoeq.so")

MOE_OK = 0
STATUS_NAMES = ["MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_OOM", "MOE_ERR_NOT_LOADED", "MOE_ERR_UNSUPPORTED",
                "MOE_ERR_BITS_UNAVAILABLE", "MOE_ERR_CUDA", "MOE_ERR_DEVICE_CHECK", "MOE_ERR_TIMEOUT",
                "MOE_ERR_TOO_LARGE"]
FMT_INT_ASYM, FMT_BITPLANE_LUT, FMT_DENSE16 = 0, 1, 2
FLAG_NO_TOPK_RENORM = 1
FLAG_DETERMINISTIC = 2
PATH_AUTO, PATH_DECODE, PATH_PREFILL = 0, 1, 2

# every symbol the header declares
EXPORTS = ["moe_layer_create", "moe_layer_set_expert_weights", "moe_layer_set_bits", "moe_layer_set_comp_top_n",
           "moe_layer_set_path", "moe_layer_set_wait_limit",
           "moe_layer_forward", "moe_layer_forward_host", "moe_layer_get_routing", "moe_layer_debug_unpack",
           "moe_layer_sync_status", "moe_layer_last_launch_count", "moe_layer_set_profiling",
           "moe_layer_kernel_times", "moe_route_topk_noalloc", "moe_plan_reduce", "moe_plan_restore",
           "moe_layer_release_planes", "moe_layer_reload_planes", "moe_layer_page_state",
           "moe_layer_set_tileq", "moe_layer_clear_tileq",
           "moe_status_string", "moe_layer_destroy"]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"{where}: {name} ({_lib().moe_status_string(status).decode()})")


class ExpertDesc(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int * 2), ("format", ctypes.c_int), ("group_size", ctypes.c_int),
                ("rank", ctypes.c_int)]


class PlanBlock(ctypes.Structure):
    _fields_ = [("committed_bits", ctypes.c_int), ("floor_bits", ctypes.c_int), ("max_steps", ctypes.c_int),
                ("plane_bytes", ctypes.c_longlong), ("sensitivity", ctypes.c_float * 5),
                ("routing_mult", ctypes.c_float), ("prompt_factor", ctypes.c_float)]


_LIB = None


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with bit_quantized_moe_top_b200.build.build()")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, U = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
        lib.moe_layer_create.argtypes = [I, I, I, I, I, ctypes.POINTER(ExpertDesc), U, ctypes.POINTER(P)]
        lib.moe_layer_set_expert_weights.argtypes = [P, I, I, P, P, P, P, P, I]
        lib.moe_layer_set_bits.argtypes = [P, I, I, I]
        lib.moe_layer_set_path.argtypes = [P, I]
        lib.moe_layer_set_wait_limit.argtypes = [P, ctypes.c_ulonglong]
        lib.moe_layer_set_comp_top_n.argtypes = [P, I]
        lib.moe_layer_set_tileq.argtypes = [P, I, I, I, I, P, P, P, I]
        lib.moe_layer_clear_tileq.argtypes = [P, I]
        lib.moe_layer_forward.argtypes = [P, P, P, I, I, P, P]
        lib.moe_layer_forward_host.argtypes = [P, P, P, I, I, P, P]
        lib.moe_layer_get_routing.argtypes = [P, P, P, P, P, P, P]
        lib.moe_layer_debug_unpack.argtypes = [P, I, I, P]
        lib.moe_layer_sync_status.argtypes = [P]
        lib.moe_layer_last_launch_count.argtypes = [P]
        lib.moe_layer_set_profiling.argtypes = [P, I]
        lib.moe_layer_kernel_times.argtypes = [P, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float), I]
        lib.moe_route_topk_noalloc.argtypes = [P, I, I, I, U, P, P, P, P, P]
        lib.moe_layer_release_planes.argtypes = [P, I, I, I, P]
        lib.moe_layer_reload_planes.argtypes = [P, I, I, I, P]
        lib.moe_layer_page_state.argtypes = [P, I, I, ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(I)]
        PB = ctypes.POINTER(PlanBlock)
        IP, LP = ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_longlong)
        lib.moe_plan_reduce.argtypes = [PB, I, ctypes.c_longlong, ctypes.c_float, IP, LP]
        lib.moe_plan_restore.argtypes = [PB, I, IP, ctypes.c_longlong, ctypes.c_float, IP, LP]
        lib.moe_status_string.argtypes = [I]
        lib.moe_status_string.restype = ctypes.c_char_p
        lib.moe_layer_destroy.argtypes = [P]
        lib.moe_layer_destroy.restype = None
        for name in EXPORTS:
            if name not in ("moe_status_string", "moe_layer_destroy"):
                getattr(lib, name).restype = I
        _LIB = lib
    return _LIB


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


# ---------------------------------------------------------------------------
# thin functions with the C names
# ---------------------------------------------------------------------------

def moe_layer_create(num_experts: int, d_model: int, d_ff: int, max_tokens: int, max_top_k: int,
                     descs: Sequence[ExpertDesc], flags: int = 0) -> int:
    arr = (ExpertDesc * num_experts)(*descs)
    out = ctypes.c_void_p()
    _check(_lib().moe_layer_create(num_experts, d_model, d_ff, max_tokens, max_top_k, arr, flags, ctypes.byref(out)),
           "moe_layer_create")
    return out.value


def moe_layer_set_expert_weights(layer: int, expert: int, block: int, codes, scales, zeros_or_lut, A, B) -> None:
    kind = 1 if codes.is_cuda else 0
    for t in (codes, scales, zeros_or_lut, A, B):
        if t is not None:
            assert t.is_contiguous() and t.is_cuda == codes.is_cuda
    _check(_lib().moe_layer_set_expert_weights(layer, expert, block, _ptr(codes), _ptr(scales), _ptr(zeros_or_lut),
                                               _ptr(A), _ptr(B), kind), "moe_layer_set_expert_weights")


def moe_layer_set_bits(layer: int, expert: int, block: int, bits: int) -> None:
    _check(_lib().moe_layer_set_bits(layer, expert, block, bits), "moe_layer_set_bits")


def moe_layer_set_comp_top_n(layer: int, n: int) -> None:
    _check(_lib().moe_layer_set_comp_top_n(layer, n), "moe_layer_set_comp_top_n")


def moe_layer_set_tileq(layer: int, block: int, rank: int, tile_m: int, tile_k: int, U, V, cores) -> None:
    """U [M, rank], V [rank, K_in], cores [E, P, Q, rank, rank]: bf16 torch
    tensors, all on the host or all on the device."""
    kind = 1 if U.is_cuda else 0
    for t in (U, V, cores):
        assert t.is_contiguous() and t.is_cuda == U.is_cuda
    _check(_lib().moe_layer_set_tileq(layer, block, rank, tile_m, tile_k, _ptr(U), _ptr(V), _ptr(cores), kind),
           "moe_layer_set_tileq")


def moe_layer_clear_tileq(layer: int, block: int) -> None:
    _check(_lib().moe_layer_clear_tileq(layer, block), "moe_layer_clear_tileq")


def moe_layer_set_path(layer: int, path: int) -> None:
    _check(_lib().moe_layer_set_path(layer, path), "moe_layer_set_path")


def moe_layer_set_wait_limit(layer: int, limit_ns: int) -> None:
    _check(_lib().moe_layer_set_wait_limit(layer, limit_ns), "moe_layer_set_wait_limit")


def moe_layer_forward(layer: int, X, logits, top_k: int, Y, stream: Optional[int] = None) -> None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(X.device).cuda_stream
    _check(_lib().moe_layer_forward(layer, _ptr(X), _ptr(logits), X.shape[0], top_k, _ptr(Y), stream),
           "moe_layer_forward")


def moe_layer_forward_host(layer: int, X_host, logits_host, top_k: int, Y_host, stream: Optional[int] = None) -> None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    _check(_lib().moe_layer_forward_host(layer, _ptr(X_host), _ptr(logits_host), X_host.shape[0], top_k,
                                         _ptr(Y_host), stream), "moe_layer_forward_host")


def moe_layer_get_routing(layer: int, idx=None, w=None, counts=None, offsets=None, perm_token=None,
                          inv_pos=None) -> None:
    _check(_lib().moe_layer_get_routing(layer, _ptr(idx), _ptr(w), _ptr(counts), _ptr(offsets), _ptr(perm_token),
                                        _ptr(inv_pos)), "moe_layer_get_routing")


def moe_layer_debug_unpack(layer: int, expert: int, block: int, out) -> None:
    _check(_lib().moe_layer_debug_unpack(layer, expert, block, _ptr(out)), "moe_layer_debug_unpack")


def moe_layer_sync_status(layer: int) -> int:
    return _lib().moe_layer_sync_status(layer)


def moe_layer_last_launch_count(layer: int) -> int:
    return _lib().moe_layer_last_launch_count(layer)


def moe_layer_set_profiling(layer: int, enable) -> None:
    """enable: False/0 off, True/1 every kernel, 2 the gate/up expert GEMM alone."""
    level = int(enable) if not isinstance(enable, bool) else (1 if enable else 0)
    _check(_lib().moe_layer_set_profiling(layer, level), "moe_layer_set_profiling")


def moe_layer_kernel_times(layer: int, cap: int = 64):
    names = (ctypes.c_char_p * cap)()
    ms = (ctypes.c_float * cap)()
    n = _lib().moe_layer_kernel_times(layer, names, ms, cap)
    if n < 0:
        return []
    return [(names[i].decode(), float(ms[i])) for i in range(min(n, cap))]


def moe_route_topk_noalloc(logits, top_k: int, idx, w, counts, offsets, flags: int = 0,
                           stream: Optional[int] = None) -> None:
    """Top-k routing with no device allocation (scratch lives in the library
    image): for callers that may not allocate device memory themselves."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(logits.device).cuda_stream
    T, E = logits.shape
    _check(_lib().moe_route_topk_noalloc(_ptr(logits), T, E, top_k, flags, _ptr(idx), _ptr(w), _ptr(counts),
                                         _ptr(offsets), stream), "moe_route_topk_noalloc")


def moe_layer_release_planes(layer: int, expert: int, block: int, keep: int, stream: Optional[int] = None) -> None:
    _check(_lib().moe_layer_release_planes(layer, expert, block, keep, _stream(stream)), "moe_layer_release_planes")


def moe_layer_reload_planes(layer: int, expert: int, block: int, planes: int, stream: Optional[int] = None) -> None:
    _check(_lib().moe_layer_reload_planes(layer, expert, block, planes, _stream(stream)), "moe_layer_reload_planes")


def moe_layer_page_state(layer: int, expert: int, block: int):
    """(committed_bits, resident_planes, host_planes) of (expert, block)."""
    c, r, h = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(_lib().moe_layer_page_state(layer, expert, block, ctypes.byref(c), ctypes.byref(r), ctypes.byref(h)),
           "moe_layer_page_state")
    return c.value, r.value, h.value


def _stream(stream):
    if stream is not None:
        return stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _plan_blocks(blocks):
    arr = (PlanBlock * len(blocks))()
    for i, b in enumerate(blocks):
        arr[i].committed_bits = b["committed_bits"]
        arr[i].floor_bits = b["floor_bits"]
        arr[i].max_steps = b["max_steps"]
        arr[i].plane_bytes = b["plane_bytes"]
        for j, g in b["sensitivity"].items():
            arr[i].sensitivity[j] = g
        arr[i].routing_mult = b["routing_mult"]
        arr[i].prompt_factor = b["prompt_factor"]
    return arr


def moe_plan_reduce(blocks, bytes_target: int, eps: float):
    """Greedy reduction plan. ``blocks``: dicts with the moe_plan_block_t
    fields (``sensitivity`` maps a bitwidth b to g of b -> b-1). Returns
    (status, new_bits, bytes_released); status MOE_OK or MOE_ERR_TOO_LARGE."""
    n = len(blocks)
    out = (ctypes.c_int * max(n, 1))()
    rel = ctypes.c_longlong(0)
    st = _lib().moe_plan_reduce(_plan_blocks(blocks), n, bytes_target, eps, out, ctypes.byref(rel))
    if st not in (MOE_OK, 9):
        raise MoEError(st, "moe_plan_reduce")
    return st, [out[i] for i in range(n)], rel.value


def moe_plan_restore(blocks, max_bits, bytes_budget: int, eps: float):
    """Greedy restore plan; returns (new_bits, bytes_used)."""
    n = len(blocks)
    out = (ctypes.c_int * max(n, 1))()
    mb = (ctypes.c_int * max(n, 1))(*max_bits)
    used = ctypes.c_longlong(0)
    _check(_lib().moe_plan_restore(_plan_blocks(blocks), n, mb, bytes_budget, eps, out, ctypes.byref(used)),
           "moe_plan_restore")
    return [out[i] for i in range(n)], used.value


def moe_status_string(status: int) -> str:
    return _lib().moe_status_string(status).decode()


def moe_layer_destroy(layer: int) -> None:
    _lib().moe_layer_destroy(layer)


# ---------------------------------------------------------------------------
# convenience wrapper
# ---------------------------------------------------------------------------

class MoELayer:
    """Owns one ``moe_layer_t``; tensors are torch tensors."""

    def __init__(self, num_experts, d_model, d_ff, max_tokens, max_top_k, descs, flags=0):
        self.E, self.K, self.N = num_experts, d_model, d_ff
        self.max_tokens, self.max_top_k = max_tokens, max_top_k
        ds = [d if isinstance(d, ExpertDesc) else ExpertDesc((ctypes.c_int * 2)(*d["bits"]), d["format"],
                                                            d.get("group_size", 0), d.get("rank", 0))
              for d in descs]
        self.handle = moe_layer_create(num_experts, d_model, d_ff, max_tokens, max_top_k, ds, flags)

    def set_expert_weights(self, expert, block, codes, scales=None, zeros_or_lut=None, A=None, B=None):
        moe_layer_set_expert_weights(self.handle, expert, block, codes, scales, zeros_or_lut, A, B)

    def set_bits(self, expert, block, bits):
        moe_layer_set_bits(self.handle, expert, block, bits)

    def release_planes(self, expert, block, keep, stream=None):
        moe_layer_release_planes(self.handle, expert, block, keep, stream)

    def reload_planes(self, expert, block, planes, stream=None):
        moe_layer_reload_planes(self.handle, expert, block, planes, stream)

    def page_state(self, expert, block):
        return moe_layer_page_state(self.handle, expert, block)

    def set_comp_top_n(self, n):
        moe_layer_set_comp_top_n(self.handle, n)

    def set_tileq(self, block, rank, tile_m, tile_k, U, V, cores):
        moe_layer_set_tileq(self.handle, block, rank, tile_m, tile_k, U, V, cores)

    def clear_tileq(self, block):
        moe_layer_clear_tileq(self.handle, block)

    def set_path(self, path):
        moe_layer_set_path(self.handle, path)

    def set_wait_limit(self, limit_ns):
        moe_layer_set_wait_limit(self.handle, limit_ns)

    def forward(self, X, logits, top_k, Y=None, stream=None):
        import torch
        if Y is None:
            Y = torch.empty_like(X)
        moe_layer_forward(self.handle, X, logits, top_k, Y, stream)
        return Y

    def forward_host(self, X_host, logits_host, top_k, Y_host=None, stream=None):
        import torch
        if Y_host is None:
            Y_host = torch.empty_like(X_host)
        moe_layer_forward_host(self.handle, X_host, logits_host, top_k, Y_host, stream)
        return Y_host

    def routing(self, T, top_k, device="cuda"):
        import torch
        r = {"idx": torch.empty(T, top_k, dtype=torch.int32, device=device),
             "w": torch.empty(T, top_k, dtype=torch.float32, device=device),
             "counts": torch.empty(self.E, dtype=torch.int32, device=device),
             "offsets": torch.empty(self.E + 1, dtype=torch.int32, device=device),
             "perm_token": torch.empty(T * top_k, dtype=torch.int32, device=device),
             "inv_pos": torch.empty(T, top_k, dtype=torch.int32, device=device)}
        moe_layer_get_routing(self.handle, r["idx"], r["w"], r["counts"], r["offsets"], r["perm_token"], r["inv_pos"])
        return r

    def debug_unpack(self, expert, block, device="cuda"):
        import torch
        M, K = (2 * self.N, self.K) if block == 0 else (self.K, self.N)
        out = torch.empty(M, K, dtype=torch.uint8, device=device)
        moe_layer_debug_unpack(self.handle, expert, block, out)
        return out

    def sync_status(self) -> int:
        return moe_layer_sync_status(self.handle)

    def last_launch_count(self) -> int:
        return moe_layer_last_launch_count(self.handle)

    def set_profiling(self, enable=True):
        moe_layer_set_profiling(self.handle, enable)

    def kernel_times(self):
        return moe_layer_kernel_times(self.handle)

    def close(self):
        if getattr(self, "handle", None):
            moe_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
