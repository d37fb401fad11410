"""A BitStack linear layer over torch-allocated device memory.

Plumbing around the C ABI: torch allocates the device buffers (block records, 1/s,
workspace, outputs) and pinned host memory for the records, which stand in for the
storage device the blocks are loaded from and offloaded to (review page "BitStack:
Fine-Grained Size Control...", Fig. 2: blocks move between storage and memory as the
budget changes).  Every computation is a call into the CUDA library.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B


class BitStackLinear:
    """One weight's block stack on one GPU.

    Parameters
    ----------
    m, d : out_features, in_features (m % 128 == 0, d % 256 == 0 for BitStack blocks)
    capacity : the most blocks the device area holds
    inv_scale : length-d float32 1/s of the activation-aware scaling
    k : singular vectors per block (16 on the GPU path; k' for plain blocks)
    plain : the blocks are "w/o AVD" rank-k' factor pairs (vanilla SVD, no signs)
    """

    def __init__(self, m: int, d: int, capacity: int, inv_scale, k: int = 16, device: str | int = "cuda",
                 stream=None, plain: bool = False):
        self.m, self.d, self.k, self.capacity = int(m), int(d), int(k), int(capacity)
        self.plain = bool(plain)
        self.device = torch.device(device)
        nbytes = (B.bs_plain_stack_device_bytes if plain else B.bs_stack_device_bytes)(m, d, k, capacity)
        if nbytes == 0:
            raise B.BsError(B.BS_ERR_UNSUPPORTED_SHAPE, "BitStackLinear")
        self.dev_blocks = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.inv_scale = torch.as_tensor(np.asarray(inv_scale, dtype=np.float32)).to(self.device).contiguous()
        self.block_bytes = (B.bs_plain_block_bytes if plain else B.bs_block_bytes)(m, d, k)
        create = B.bs_plain_stack_create if plain else B.bs_stack_create
        self.handle = create(m, d, k, capacity, self.dev_blocks, self.inv_scale, stream)
        self.host_records: list[torch.Tensor] = []   # the storage copy of every block, pinned
        self._inflight: list[torch.Tensor] = []
        self._ws: torch.Tensor | None = None

    # ----------------------------------------------------------- storage side ----
    def add_record(self, record) -> int:
        """Keeps a block record (uint8, bs_block_bytes long) in pinned host memory."""
        rec = torch.as_tensor(np.ascontiguousarray(record, dtype=np.uint8))
        if rec.numel() != self.block_bytes:
            raise ValueError("record has the wrong size")
        pinned = torch.empty(self.block_bytes, dtype=torch.uint8, pin_memory=True)
        pinned.copy_(rec)
        self.host_records.append(pinned)
        return len(self.host_records) - 1

    def add_pinned_record(self, pinned: torch.Tensor) -> int:
        """Keeps an already pinned record (uint8, bs_block_bytes long) without copying
        it; several stacks may share one storage copy."""
        if pinned.numel() != self.block_bytes or not pinned.is_pinned():
            raise ValueError("need a pinned record of the stack's block size")
        self.host_records.append(pinned)
        return len(self.host_records) - 1

    # ----------------------------------------------------------- memory side -----
    @property
    def n_blocks(self) -> int:
        return B.bs_stack_num_blocks(self.handle)

    def append(self, stream=None) -> None:
        """Loads the next stored block onto the GPU (one async copy)."""
        n = self.n_blocks
        if n >= len(self.host_records):
            raise IndexError("no stored block left to load")
        B.bs_append_block(self.handle, self.host_records[n], stream)

    def drop(self) -> None:
        """Offloads the last loaded block (no transfer)."""
        B.bs_drop_block(self.handle)

    def set_loaded(self, n: int, stream=None) -> None:
        """Appends or drops blocks until n are loaded."""
        while self.n_blocks < n:
            self.append(stream)
        while self.n_blocks > n:
            self.drop()

    def workspace(self, n_loaded: int, batch: int) -> torch.Tensor | None:
        need = (B.bs_plain_workspace_bytes if self.plain else B.bs_workspace_bytes)(self.m, self.d, self.k,
                                                                                     n_loaded, batch)
        if need == 0:
            return None
        if self._ws is None or self._ws.numel() < need:
            # zeroed once: completed calls leave it consistent (device_error re-zeroes it)
            self._ws = torch.zeros(need, dtype=torch.uint8, device=self.device)
        return self._ws

    def forward(self, x: torch.Tensor, n_loaded: int | None = None, out: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        n = self.n_blocks if n_loaded is None else int(n_loaded)
        x = x.contiguous()
        if out is None:
            out = torch.empty((x.shape[0], self.m), dtype=x.dtype, device=self.device)
        ws = workspace if workspace is not None else self.workspace(n, x.shape[0])
        B.bs_linear(self.handle, x, n, out, ws, stream)
        return out

    __call__ = forward

    def reconstruct(self, n: int | None = None, dtype=torch.float32, stream=None) -> torch.Tensor:
        n = self.n_blocks if n is None else int(n)
        W = torch.empty((self.m, self.d), dtype=dtype, device=self.device)
        B.bs_reconstruct(self.handle, n, W, stream)
        return W

    def unpack_signs(self, block: int, stream=None) -> torch.Tensor:
        out = torch.empty((self.m, self.d), dtype=torch.int8, device=self.device)
        B.bs_unpack_signs(self.handle, block, out, stream)
        return out

    def device_record(self, block: int) -> torch.Tensor:
        """A view of block `block`'s record bytes on the device."""
        off = block * self.block_bytes
        return self.dev_blocks[off:off + self.block_bytes]

    def device_error(self) -> int:
        """Reads and clears the stack's sticky device error word.  After an error the
        workspace's counters may be stale, so the layer's own workspace is zeroed."""
        status = B.bs_get_device_error(self.handle)
        if status != B.BS_OK and self._ws is not None:
            self._ws.zero_()
        return status

    def close(self) -> None:
        if self.handle:
            B.bs_stack_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def record_from_parts(sign_words: np.ndarray, U: np.ndarray, V: np.ndarray) -> np.ndarray:
    """A block record from sign words already in the device tile order (uint32) and
    fp16 factors U (m x k) and V (d x k): the three parts laid end to end."""
    return np.concatenate([np.ascontiguousarray(sign_words, dtype="<u4").view(np.uint8),
                           np.ascontiguousarray(U, dtype=np.float16).view(np.uint8).reshape(-1),
                           np.ascontiguousarray(V, dtype=np.float16).view(np.uint8).reshape(-1)])
