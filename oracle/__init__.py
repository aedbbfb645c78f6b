"""CPU oracle for per-frame paged-KV prefill attention.

TEST INFRASTRUCTURE ONLY. Nothing in the library package imports, calls or
links anything here. The only callers are the tests, `__graft_entry__.smoke()`
and the `cpu_baseline` / reference leg of `bench.py`. The oracle and the CUDA
path share no code: the only common module is `workload`, which draws the
seeded inputs and holds none of the method's arithmetic.

The oracle is plain Python + numpy in float64. It restates what the pages say
the method computes:

  [P1] "How the Paged KV Cache Attention Mechanism Enables Long Sequence
       Inference in LingBot-Map"
  [P2] "KV Cache Mechanism in LingBot-Map for Streaming Inference: A Deep Dive"
  [P3] "FlashInfer Paged KV Cache Performance Benefits in LingBot-Map:
       Technical Implementation and Benchmarks"
  [P4] "How LingBot-Map Achieves ~20 FPS Inference with Its KV Cache"

Modules:
  frames    -- brute-force frame-list simulator: which frames and special
               tokens are visible after any sequence of cache operations.
  pages     -- page-level model: free list, scale/window pages, special
               stream packing, visible page table, last_page_len, and the
               expected pool image after each append.
  attention -- dense fp64 attention over the visible tokens, a brute-force
               loop version, chunked partials and their log-sum-exp merge.
  stream    -- drives a whole stream of frames through `frames` and gives
               the expected attention output of any frame step.

Every function is pinned by tests in `tests/test_oracle_*.py` against values
the pages print, closed forms, a library routine (PyTorch SDPA in float64) or
brute force. No function here is "parity unpinned".
"""
from .frames import FrameListSim
from .pages import PageModel, PoolImage, OracleError, SharedPatchPool
from . import attention

__all__ = ["FrameListSim", "PageModel", "PoolImage", "OracleError", "SharedPatchPool", "attention"]
