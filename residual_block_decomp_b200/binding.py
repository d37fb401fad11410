"""Python binding of the C ABI in include/bitstack.h (argument marshalling only).

Every function here has the name of the C entry point it calls and does nothing but
turn Python / torch arguments into pointers and sizes; every step of the hot path
runs in the CUDA library.  A non-OK status raises ``BsError`` (``.status`` holds the
code).  The library is loaded from the package directory; if it is missing, import
fails loudly: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
# BITSTACK_LIB may name another build of the same ABI (e.g. a profiling build).
LIB_PATH = os.environ.get("BITSTACK_LIB") or os.path.join(_PKG, "libbitstack_b200.so")

BS_OK = 0
BS_ERR_INVALID_ARG = 1
BS_ERR_UNSUPPORTED_SHAPE = 2
BS_ERR_ALIGNMENT = 3
BS_ERR_CAPACITY = 4
BS_ERR_RANGE = 5
BS_ERR_CUDA = 6
BS_ERR_TIMEOUT = 7
BS_ERR_NO_DEVICE = 8

BS_F16 = 0
BS_BF16 = 1
BS_F32 = 2

BS_ORDER_AVERAGE = 0
BS_ORDER_GREEDY = 1
BS_ORDER_RANDOM = 2

EXPORTS = (
    "bs_block_bytes", "bs_stack_device_bytes", "bs_workspace_bytes", "bs_pack_record",
    "bs_stack_create", "bs_stack_destroy", "bs_stack_num_blocks", "bs_append_block",
    "bs_drop_block", "bs_linear", "bs_reconstruct", "bs_unpack_signs",
    "bs_get_device_error", "bs_status_string", "bs_debug_set_wait", "bs_linear_no_alloc",
    "bs_plan_order", "bs_plan_budget", "bs_plain_rank", "bs_plain_block_bytes", "bs_plain_stack_device_bytes",
    "bs_plain_workspace_bytes", "bs_plain_stack_create", "bs_group_workspace_bytes", "bs_linear_group",
    "bs_decompose_workspace_bytes", "bs_decompose",
)


class BsError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {bs_status_string(status)} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m residual_block_decomp_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong
    sig = {
        "bs_block_bytes": (Z, [I, I, I]),
        "bs_stack_device_bytes": (Z, [I, I, I, I]),
        "bs_workspace_bytes": (Z, [I, I, I, I, I]),
        "bs_pack_record": (I, [I, I, I, P, P, P, P]),
        "bs_stack_create": (I, [I, I, I, I, P, Z, P, P, ctypes.POINTER(P)]),
        "bs_stack_destroy": (I, [P]),
        "bs_stack_num_blocks": (I, [P, ctypes.POINTER(I)]),
        "bs_append_block": (I, [P, P, P]),
        "bs_drop_block": (I, [P]),
        "bs_linear": (I, [P, P, I, I, I, P, P, Z, P]),
        "bs_reconstruct": (I, [P, I, P, I, P]),
        "bs_unpack_signs": (I, [P, I, P, P]),
        "bs_get_device_error": (I, [P]),
        "bs_status_string": (ctypes.c_char_p, [I]),
        "bs_debug_set_wait": (I, [P, LL, I]),
        "bs_linear_no_alloc": (I, [P, P, I, I, I, P, P]),
        "bs_plan_order": (I, [I, P, P, I, I, P, P, P]),
        "bs_plan_budget": (I, [LL, P, I, P, ctypes.c_ulonglong, P]),
        "bs_plain_rank": (I, [I, I, I]),
        "bs_plain_block_bytes": (Z, [I, I, I]),
        "bs_plain_stack_device_bytes": (Z, [I, I, I, I]),
        "bs_plain_workspace_bytes": (Z, [I, I, I, I, I]),
        "bs_plain_stack_create": (I, [I, I, I, I, P, Z, P, P, ctypes.POINTER(P)]),
        "bs_group_workspace_bytes": (Z, [I, P, P, I]),
        "bs_linear_group": (I, [I, P, P, P, P, I, I, P, Z, P]),
        "bs_decompose_workspace_bytes": (Z, [I, I, I]),
        "bs_decompose": (I, [I, I, I, I, P, P, ctypes.c_ulonglong, I, P, Z, P, P, Z, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _check(status: int, where: str) -> None:
    if status != BS_OK:
        raise BsError(status, where)


def _stream(stream) -> int | None:
    """A cudaStream_t as an int: a torch stream, a raw handle, or None (current stream)."""
    if stream is None:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream or None
        return None
    if hasattr(stream, "cuda_stream"):
        return stream.cuda_stream or None
    return int(stream) or None


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _dtype_code(t) -> int:
    import torch
    return {torch.float16: BS_F16, torch.bfloat16: BS_BF16, torch.float32: BS_F32}[t.dtype]


# ------------------------------------------------------------------ sizes ----------
def bs_block_bytes(m: int, d: int, k: int) -> int:
    return int(lib.bs_block_bytes(m, d, k))


def bs_stack_device_bytes(m: int, d: int, k: int, capacity: int) -> int:
    return int(lib.bs_stack_device_bytes(m, d, k, capacity))


def bs_workspace_bytes(m: int, d: int, k: int, n_loaded: int, batch: int) -> int:
    return int(lib.bs_workspace_bytes(m, d, k, n_loaded, batch))


def bs_status_string(status: int) -> str:
    return lib.bs_status_string(int(status)).decode()


# ------------------------------------------------------------------ packing ---------
def bs_pack_record(m: int, d: int, k: int, neg_bits: np.ndarray, U: np.ndarray, V: np.ndarray,
                   out: np.ndarray | None = None) -> np.ndarray:
    """neg_bits: uint8 m x d/8 canonical bits; U, V: fp16.  Returns the uint8 record."""
    neg_bits = np.ascontiguousarray(neg_bits, dtype=np.uint8)
    U = np.ascontiguousarray(U, dtype=np.float16)
    V = np.ascontiguousarray(V, dtype=np.float16)
    if out is None:
        out = np.empty(bs_block_bytes(m, d, k), dtype=np.uint8)
    _check(lib.bs_pack_record(m, d, k, _ptr(neg_bits), _ptr(U), _ptr(V), _ptr(out)), "bs_pack_record")
    return out


# ---------------------------------------------------------------- stack life -------
def bs_stack_create(m: int, d: int, k: int, capacity: int, dev_blocks, inv_scale, stream=None) -> int:
    h = ctypes.c_void_p()
    st = lib.bs_stack_create(m, d, k, capacity, _ptr(dev_blocks), dev_blocks.numel() * dev_blocks.element_size(),
                             _ptr(inv_scale), _stream(stream), ctypes.byref(h))
    _check(st, "bs_stack_create")
    return h.value


def bs_plain_rank(m: int, d: int, k: int) -> int:
    return int(lib.bs_plain_rank(m, d, k))


def bs_plain_block_bytes(m: int, d: int, k_prime: int) -> int:
    return int(lib.bs_plain_block_bytes(m, d, k_prime))


def bs_plain_stack_device_bytes(m: int, d: int, k_prime: int, capacity: int) -> int:
    return int(lib.bs_plain_stack_device_bytes(m, d, k_prime, capacity))


def bs_plain_workspace_bytes(m: int, d: int, k_prime: int, n_loaded: int, batch: int) -> int:
    return int(lib.bs_plain_workspace_bytes(m, d, k_prime, n_loaded, batch))


def bs_plain_stack_create(m: int, d: int, k_prime: int, capacity: int, dev_blocks, inv_scale, stream=None) -> int:
    h = ctypes.c_void_p()
    st = lib.bs_plain_stack_create(m, d, k_prime, capacity, _ptr(dev_blocks),
                                   dev_blocks.numel() * dev_blocks.element_size(), _ptr(inv_scale), _stream(stream),
                                   ctypes.byref(h))
    _check(st, "bs_plain_stack_create")
    return h.value


def bs_stack_destroy(handle: int) -> None:
    _check(lib.bs_stack_destroy(handle), "bs_stack_destroy")


def bs_stack_num_blocks(handle: int) -> int:
    n = ctypes.c_int()
    _check(lib.bs_stack_num_blocks(handle, ctypes.byref(n)), "bs_stack_num_blocks")
    return n.value


def bs_append_block(handle: int, host_record, stream=None) -> None:
    _check(lib.bs_append_block(handle, _ptr(host_record), _stream(stream)), "bs_append_block")


def bs_drop_block(handle: int) -> None:
    _check(lib.bs_drop_block(handle), "bs_drop_block")


# ------------------------------------------------------------------- compute -------
def bs_linear(handle: int, x, n_loaded: int, y, workspace=None, stream=None) -> None:
    """y[batch, m] = x[batch, d] W_hat_n^T; x and y are CUDA tensors of one dtype."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.bs_linear(handle, _ptr(x), x.shape[0], _dtype_code(x), n_loaded, _ptr(y), _ptr(workspace), ws_bytes,
                       _stream(stream))
    _check(st, "bs_linear")


def bs_linear_no_alloc(handle: int, x, n_loaded: int, y, stream=None) -> None:
    """bs_linear for batch <= 4 with the library's own fixed scratch array: for
    callers that cannot allocate a workspace (see include/bitstack.h)."""
    st = lib.bs_linear_no_alloc(handle, _ptr(x), x.shape[0], _dtype_code(x), n_loaded, _ptr(y), _stream(stream))
    _check(st, "bs_linear_no_alloc")


def bs_reconstruct(handle: int, n: int, W_out, stream=None) -> None:
    _check(lib.bs_reconstruct(handle, n, _ptr(W_out), _dtype_code(W_out), _stream(stream)), "bs_reconstruct")


def bs_unpack_signs(handle: int, block: int, out, stream=None) -> None:
    _check(lib.bs_unpack_signs(handle, block, _ptr(out), _stream(stream)), "bs_unpack_signs")


def bs_get_device_error(handle: int) -> int:
    return int(lib.bs_get_device_error(handle))


def bs_debug_set_wait(handle: int, timeout_ns: int, unreachable_flag: bool = False) -> None:
    _check(lib.bs_debug_set_wait(handle, int(timeout_ns), 1 if unreachable_flag else 0), "bs_debug_set_wait")


def bs_plan_order(n_blocks, kind: int, scores=None, draws=None):
    """Global load order of all blocks: two int32 arrays (weight, block) of
    sum(n_blocks) entries.  ``scores`` is a (n_weights, >= max n_blocks) float64
    array (GREEDY), ``draws`` sum(n_blocks) float64 numbers in [0, 1) (RANDOM)."""
    counts = np.ascontiguousarray(n_blocks, dtype=np.int32)
    total = int(counts.sum()) if counts.size else 0
    out_w = np.zeros(max(total, 1), dtype=np.int32)
    out_b = np.zeros(max(total, 1), dtype=np.int32)
    sc = None if scores is None else np.ascontiguousarray(scores, dtype=np.float64)
    dr = None if draws is None else np.ascontiguousarray(draws, dtype=np.float64)
    stride = 0 if sc is None else (sc.shape[1] if sc.ndim == 2 else 0)
    _check(lib.bs_plan_order(counts.size, _ptr(counts), _ptr(sc), stride, int(kind), _ptr(dr), _ptr(out_w),
                             _ptr(out_b)), "bs_plan_order")
    return out_w[:total], out_b[:total]


def bs_plan_budget(order_weight, block_bytes, budget_bytes: int):
    """Blocks per weight that the longest fitting prefix of ``order_weight`` loads."""
    order = np.ascontiguousarray(order_weight, dtype=np.int32)
    sizes = np.ascontiguousarray(block_bytes, dtype=np.uint64)
    out = np.zeros(max(sizes.size, 1), dtype=np.int32)
    _check(lib.bs_plan_budget(order.size, _ptr(order) if order.size else None, sizes.size, _ptr(sizes),
                              int(budget_bytes), _ptr(out)), "bs_plan_budget")
    return out[:sizes.size]


def _handles(handles):
    return (ctypes.c_void_p * len(handles))(*[int(h) for h in handles])


def bs_group_workspace_bytes(handles, n_loaded, batch: int) -> int:
    counts = np.ascontiguousarray(n_loaded, dtype=np.int32)
    return int(lib.bs_group_workspace_bytes(len(handles), _handles(handles), _ptr(counts), batch))


def bs_linear_group(handles, xs, n_loaded, ys, workspace, stream=None) -> None:
    """One decode launch over many stacks: ys[l] = xs[l] W_hat_{n_loaded[l]}^T (CUDA
    tensors, one dtype, batch 1..4)."""
    nl = len(handles)
    counts = np.ascontiguousarray(n_loaded, dtype=np.int32)
    xp = (ctypes.c_void_p * nl)(*[_ptr(t) for t in xs])
    yp = (ctypes.c_void_p * nl)(*[_ptr(t) for t in ys])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.bs_linear_group(nl, _handles(handles), xp, yp, _ptr(counts), xs[0].shape[0], _dtype_code(xs[0]),
                             _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "bs_linear_group")


def bs_decompose_workspace_bytes(m: int, d: int, k: int = 16) -> int:
    return int(lib.bs_decompose_workspace_bytes(m, d, k))


def bs_decompose(W, s, n_blocks: int, records, res_norms_sq, workspace, seed: int = 0, power_iters: int = 6,
                 k: int = 16, stream=None) -> None:
    """GPU decomposition of W (m x d fp32 CUDA tensor) with scale s (d fp32) into
    n_blocks records (uint8 CUDA tensor) and the squared residual norms (n_blocks + 1
    float64 CUDA tensor)."""
    m, d = W.shape
    st = lib.bs_decompose(m, d, k, n_blocks, _ptr(W), _ptr(s), int(seed), int(power_iters), _ptr(records),
                          records.numel() * records.element_size(), _ptr(res_norms_sq), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "bs_decompose")
