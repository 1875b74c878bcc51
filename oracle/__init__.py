"""Oracle: a plain, slow CPU definition of paged decode attention and the
cache operations around it, in float64.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
CPU-baseline leg may import this package.  The CUDA library never calls it,
shares no code with it, and has no CPU fallback to it.

What each function follows (page titles as printed on the pages):

* ``attention.paged_decode`` -- "PagedAttention 与 vLLM 推理加速" §2.3
  (the kernel reads every K in the sequence's blocks through the block
  table, Q x K gives the attention scores) and §1 (each new token attends
  over every earlier token's K/V, itself included); the softmax and the
  weighted sum of V are the standard scaled-dot-product attention.
* ``attention.paged_multi`` -- several query tokens per sequence (the
  verification pass of speculative decoding, "PagedAttention 与 vLLM 推理
  加速" §6; prefill chunks in mixed batches, "LLM Systems 24 ..."
  §2.2.1.3), each attending causally over its sequence's tokens.
* ``cache.RefCache.append`` -- "vLLM + PagedAttention：打造高并发LLM推理引擎",
  "它是怎么工作的": the page table records which block token n lives in;
  a new token is written into its slot, old tokens are never moved.
* ``cache.RefCache.copy_blocks`` and ``allocator.RefAllocator`` --
  "PagedAttention 与 vLLM 推理加速" §3.2(3) (shared blocks are only copied
  when a writer appends) and "LLM Systems 24 ..." §3 (reference counts and
  copy-on-write share KV blocks across samples).
* ``RefAllocator.swap_out`` / ``swap_in`` and ``cache.swap_blocks`` --
  "LLM Systems 24 ..." §3, conclusion (a request preempted for lack of KV
  blocks is swapped out and later swapped back in); the policy details are
  readings stated in ``allocator``.
* ``fp8`` and ``RefCache.append_fp8`` -- an FP8 E4M3 KV cache with one
  scale for K and one for V (the pages name FP8 only for TensorRT-LLM's
  low-precision operators; the format and the scaling are readings stated
  in ``fp8``).
* ``brute.contiguous_decode`` -- the contiguous-cache baseline the pages
  contrast paging with ("PagedAttention 与 vLLM 推理加速" §2.2), in pure
  Python, used only to pin ``paged_decode`` on tiny inputs.

Every function is pinned by tests that do not retype its formula: brute
force on tiny inputs, invariance under block relabelling, shared-prefix
versus private-copy layouts, closed forms, and the pages' worked examples.
"""

from .storage import widen, nan_fill  # noqa: F401
from .attention import paged_decode, paged_multi, decode_head  # noqa: F401
from .cache import RefCache, swap_blocks  # noqa: F401
from .allocator import RefAllocator, RefAllocError  # noqa: F401
from .brute import contiguous_decode  # noqa: F401
from .replay import replay  # noqa: F401
from . import fp8  # noqa: F401
