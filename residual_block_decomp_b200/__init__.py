"""B200-native BitStack residual-block linear.

The C ABI (include/bitstack.h) is implemented by libbitstack_b200.so, built from
csrc/ for sm_100a by ``residual_block_decomp_b200.build``; ``binding`` exposes it
under the same names and ``layer`` wraps a stack in torch-allocated device memory.
Attributes are resolved on first use, so the builder can run before the library
exists; using any binding name without the library fails loudly.
"""
import importlib

_BINDING_NAMES = (
    "BS_BF16", "BS_ERR_ALIGNMENT", "BS_ERR_CAPACITY", "BS_ERR_CUDA", "BS_ERR_INVALID_ARG", "BS_ERR_NO_DEVICE",
    "BS_ERR_RANGE", "BS_ERR_TIMEOUT", "BS_ERR_UNSUPPORTED_SHAPE", "BS_F16", "BS_F32", "BS_OK", "BS_ORDER_AVERAGE",
    "BS_ORDER_GREEDY", "BS_ORDER_RANDOM", "EXPORTS",
    "LIB_PATH", "BsError", "bs_append_block", "bs_block_bytes", "bs_decompose", "bs_decompose_workspace_bytes", "bs_debug_set_wait", "bs_drop_block",
    "bs_get_device_error", "bs_group_workspace_bytes", "bs_linear", "bs_linear_group", "bs_linear_no_alloc", "bs_pack_record", "bs_plain_block_bytes",
    "bs_plain_rank", "bs_plain_stack_create", "bs_plain_stack_device_bytes", "bs_plain_workspace_bytes",
    "bs_plan_budget", "bs_plan_order", "bs_reconstruct",
    "bs_stack_create", "bs_stack_destroy", "bs_stack_device_bytes", "bs_stack_num_blocks", "bs_status_string",
    "bs_unpack_signs", "bs_workspace_bytes", "lib",
)
__all__ = list(_BINDING_NAMES) + ["BitStackLinear"]


def __getattr__(name):
    if name in _BINDING_NAMES:
        return getattr(importlib.import_module(".binding", __name__), name)
    if name == "BitStackLinear":
        return importlib.import_module(".layer", __name__).BitStackLinear
    raise AttributeError(name)
