"""CPU oracle for the BitStack residual-block linear (test infrastructure).

This package is the parity authority for the CUDA path.  It is a plain, slow,
obviously-correct NumPy implementation in float64 of what the hot path computes:

* activation-aware scaling of the weight per input channel (``decompose``),
* iterative absolute-value decomposition into residual blocks (``decompose``),
* sign packing, canonical and in the device tile order, and the block record
  (``pack``),
* weight reconstruction and the linear layer in explicit and factored form
  (``linear``),
* the global block order and greedy memory-budget fill (``budget``).

It is test infrastructure: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.  It
shares no code with ``residual_block_decomp_b200`` and never imports it; the only
module both sides use is ``workloads`` (seeded random draws, no arithmetic of the
method).

Citations name the page and the figure / section they follow:

* README   -- "BitStack: Any-Size Compression of Large Language Models in Variable
              Memory Environments", the project README (GitHub).
* Review   -- "BitStack: Fine-Grained Size Control for Compressed Large Language
              Models in Variable Memory Environments", the paper-review page
              (figure and table captions).
* Abstract -- the abstract on the code-index page.
* Rebuttal -- the OpenReview discussion page (author replies A1-A3 and the weight
              restoration snippet).

Parity status of each function is stated in its docstring; "parity unpinned" marks
a function no test pins to something other than itself.
"""
from . import budget, decompose, linear, pack  # noqa: F401
