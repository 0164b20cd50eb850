"""CPU oracle for the routed-expert MoE layer (test infrastructure).

A plain, slow, readable restatement of what the layer computes, in float64
unless a step's decision has to be taken in the kernel's fp32.  Only the test
suite, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import it; the library never calls it and shares no code,
tables or constants with it.

Sources (titles of the pages the method is described on):
  * explainx.ai, "FreeToken 753B local MoE single-GPU hardware guide",
    section "Decode: decide whether to move an expert or compute where it lives"
    -- per-token expert choice, GPU/CPU split of misses, exact merge.
  * ainewsfeed.tech, "FreeToken Runs 753B GLM-5.2 on a Single Workstation GPU",
    third paragraph -- q* split, exact merge without router modification,
    shared LRU expert cache.
  * futuresignalnews.com, "Unlocking Frontier LLMs", mechanism 1 -- q* =
    number of experts to fill into the GPU cache.
  * freetoken.wiki, "FreeToken 753b model", mechanism table -- global LRU cache.

Parity status per function is stated in each module header.
"""
from . import formats, moe, lru  # noqa: F401
