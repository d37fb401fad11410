"""CPU tests of the C-ABI library: it loads, exports every declared entry point, and
its host-side logic (sizes, packing, argument validation) behaves as specified.
No GPU is needed; no compute call is made."""
import ctypes
import os
import re

import numpy as np
import pytest

import residual_block_decomp_b200 as R
import workloads as wl
from oracle import pack

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "bitstack.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bs_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 15
    for name in names:
        assert hasattr(R.lib, name), name
    assert set(names) == set(R.EXPORTS)


def test_library_is_the_in_tree_build():
    assert os.path.dirname(R.LIB_PATH) == os.path.dirname(os.path.abspath(R.__file__))
    assert os.path.exists(R.LIB_PATH)


def test_block_bytes_formula():
    for (m, d, k) in [(4096, 4096, 16), (14336, 4096, 16), (512, 512, 16), (128, 256, 3)]:
        assert R.bs_block_bytes(m, d, k) == pack.block_bytes(m, d, k)
    assert R.bs_block_bytes(14336, 4096, 16) == 7_929_856
    assert R.bs_block_bytes(0, 4096, 16) == 0
    assert R.bs_block_bytes(128, 12, 16) == 0


def test_device_and_workspace_sizes():
    bb = R.bs_block_bytes(4096, 4096, 16)
    dev = R.bs_stack_device_bytes(4096, 4096, 16, 8)
    assert dev >= 8 * bb and dev % 256 == 0
    assert R.bs_stack_device_bytes(100, 4096, 16, 8) == 0     # m % 128
    assert R.bs_stack_device_bytes(4096, 4096, 8, 8) == 0     # k != 16 on the GPU path
    ws = R.bs_workspace_bytes(4096, 4096, 16, 8, 1)
    # one fp32 partial per 128-row tile x 4-chunk group x block and row, + row-tile counters
    assert ws == 32 * (16 // 4) * 8 * 128 * 4 + 256
    assert R.bs_workspace_bytes(4096, 4096, 16, 8, 4) > ws
    assert R.bs_workspace_bytes(4096, 4096, 16, 0, 1) == 0    # n = 0 needs none
    # prefill: a grid that fills the SMs needs none; 64 tokens (32 CTAs) split K in 4
    # (148 SMs assumed without a device): 256 bytes of counters, then 4 partial tiles
    # of 128 rows x 64 tokens per row tile
    assert R.bs_workspace_bytes(4096, 4096, 16, 8, 4096) == 0
    assert R.bs_workspace_bytes(4096, 4096, 16, 8, 64) == 256 + 4 * 32 * 128 * 64 * 4
    # 16 tokens of the 4096 x 14336 MLP weight: 4 splits of 112 K-tiles, 32-token tiles
    assert R.bs_workspace_bytes(4096, 14336, 16, 8, 16) == 256 + 4 * 32 * 128 * 32 * 4
    # 14336 rows: 112 CTAs already fill the SMs' one wave (148 // 112 = 1 split): none
    assert R.bs_workspace_bytes(14336, 4096, 16, 8, 16) == 0
    # one row tile, 600 tokens of 2560 columns: 5 token tiles of 128 in clusters of 4
    # (8 CTAs with the padding) -> min(148 // 8, 80 // 8) = 10 splits of 8 K-tiles;
    # counters for 1 x 5 tiles, then 10 partial tiles of 128 x 128 per token tile
    assert R.bs_workspace_bytes(128, 2560, 16, 5, 600) == 256 + 10 * 5 * 128 * 128 * 4
    # 16 loaded blocks fit the prefill's shared memory at 64 tokens; 40 do not (U, V and
    # one sign group alone pass 227 KB)
    assert R.bs_workspace_bytes(128, 4096, 16, 16, 64) > 0
    assert R.bs_workspace_bytes(128, 4096, 16, 40, 64) == 0


@pytest.mark.parametrize("m,d,seed", [(128, 256, 0), (256, 512, 1), (384, 768, 2), (512, 512, 3)])
def test_host_packer_matches_oracle_bit_exactly(m, d, seed):
    gen = np.random.default_rng(seed)
    neg, U, V = wl.synthetic_block(m, d, 16, gen)
    rec = R.bs_pack_record(m, d, 16, pack.pack_canonical(neg), U, V)
    assert np.array_equal(rec, pack.make_record(neg, U, V))


def test_host_packer_rejects_bad_arguments():
    bits = np.zeros((128, 32), np.uint8)
    U = np.zeros((128, 16), np.float16)
    V = np.zeros((256, 16), np.float16)
    out = np.zeros(R.bs_block_bytes(128, 256, 16), np.uint8)
    null = ctypes.c_void_p(None)
    assert R.lib.bs_pack_record(128, 256, 16, null, U.ctypes.data, V.ctypes.data, out.ctypes.data) == R.BS_ERR_INVALID_ARG
    assert R.lib.bs_pack_record(100, 256, 16, bits.ctypes.data, U.ctypes.data, V.ctypes.data,
                                out.ctypes.data) == R.BS_ERR_UNSUPPORTED_SHAPE
    assert R.lib.bs_pack_record(128, 200, 16, bits.ctypes.data, U.ctypes.data, V.ctypes.data,
                                out.ctypes.data) == R.BS_ERR_UNSUPPORTED_SHAPE


def test_stack_create_validates_before_touching_a_device():
    h = ctypes.c_void_p()
    fake_dev, fake_s = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 21)
    big = R.bs_stack_device_bytes(4096, 4096, 16, 8)
    create = R.lib.bs_stack_create
    assert create(4096, 4096, 16, 8, None, big, fake_s, None, ctypes.byref(h)) == R.BS_ERR_INVALID_ARG
    assert create(4096, 4096, 16, 0, fake_dev, big, fake_s, None, ctypes.byref(h)) == R.BS_ERR_INVALID_ARG
    assert create(4000, 4096, 16, 8, fake_dev, big, fake_s, None, ctypes.byref(h)) == R.BS_ERR_UNSUPPORTED_SHAPE
    assert create(4096, 4096, 12, 8, fake_dev, big, fake_s, None, ctypes.byref(h)) == R.BS_ERR_UNSUPPORTED_SHAPE
    assert create(4096, 4096, 16, 8, ctypes.c_void_p((1 << 20) + 64), big, fake_s, None,
                  ctypes.byref(h)) == R.BS_ERR_ALIGNMENT
    assert create(4096, 4096, 16, 8, fake_dev, big, ctypes.c_void_p((1 << 21) + 4), None,
                  ctypes.byref(h)) == R.BS_ERR_ALIGNMENT
    assert create(4096, 4096, 16, 8, fake_dev, big - 1, fake_s, None, ctypes.byref(h)) == R.BS_ERR_CAPACITY
    # valid arguments on a machine without an sm_100 device
    import torch
    if not torch.cuda.is_available():
        assert create(4096, 4096, 16, 8, fake_dev, big, fake_s, None, ctypes.byref(h)) == R.BS_ERR_NO_DEVICE
        assert h.value is None


def test_null_handles_are_rejected():
    assert R.lib.bs_stack_destroy(None) == R.BS_ERR_INVALID_ARG
    assert R.lib.bs_drop_block(None) == R.BS_ERR_INVALID_ARG
    assert R.lib.bs_append_block(None, None, None) == R.BS_ERR_INVALID_ARG
    assert R.lib.bs_linear(None, None, 1, 0, 0, None, None, 0, None) == R.BS_ERR_INVALID_ARG
    assert R.lib.bs_reconstruct(None, 0, None, 0, None) == R.BS_ERR_INVALID_ARG
    assert R.lib.bs_get_device_error(None) == R.BS_ERR_INVALID_ARG
    assert R.lib.bs_debug_set_wait(None, 1000, 0) == R.BS_ERR_INVALID_ARG


def test_status_strings():
    for code in range(9):
        s = R.bs_status_string(code)
        assert s and s != "unknown status"
    assert R.bs_status_string(99) == "unknown status"


def test_no_alloc_capacity_figures_in_the_header():
    """The header's worked example of the no-alloc scratch limit: 4096 x 4096 fits
    n = 64 at batch 1 (the decode path's block limit), 31 at batch 2, 21 at batch 3 and
    15 at batch 4 in 8 MiB, and one block more does not."""
    import residual_block_decomp_b200 as R
    cap = 8 << 20
    for b, n_max in ((1, 64), (2, 31), (3, 21), (4, 15)):
        assert R.bs_workspace_bytes(4096, 4096, 16, n_max, b) <= cap
        if n_max < 64:
            assert R.bs_workspace_bytes(4096, 4096, 16, n_max + 1, b) > cap
    assert R.bs_workspace_bytes(4096, 4096, 16, 8, 1) == 256 + 8 * 65536   # 0.5 MiB
