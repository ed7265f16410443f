"""Plain CPU oracle for paged decode attention and its companion operations.

TEST INFRASTRUCTURE, NOT THE PRODUCT.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
package.  The CUDA library never imports, links or calls anything here, and
nothing here imports the CUDA library: the two sides share only the seeded
input generator in ``workloads.py``.

Everything is written to be checked by eye against the pages it follows:

* ``fp``            exact decoding of fp16 / bf16 storage bits to float64.
* ``attention``     gather a sequence's logical K/V through its block table,
                    then softmax(q K^T * scale) V in float64; the split-context
                    partial/merge algebra; the causal multi-token form
                    of a chunked prefill.
* ``cache_ops``     reshape_and_cache (scatter of new K/V into their slots) and
                    copy_blocks (copy-on-write block copies), on raw bits.
* ``block_manager`` free list, reference counts, fork, copy-on-write and
                    prefix caching across requests.
* ``utilisation``   KV memory accounting: paged blocks versus contiguous
                    max-length reservation.

Sources, cited by page title and section:
  [P1] "Why OS Virtual Memory Paging Saved LLM Inference: The vLLM Breakthrough"
  [P2] "vLLM & PagedAttention: Operating Systems Ideas for LLM Serving"
  [P3] "Can OS paging techniques reduce LLM serving memory waste?"

Parity status: every function here is pinned by tests/test_oracle_*.py against
closed forms, special cases that reduce to a library routine, invariants the
pages state, or brute force on tiny inputs.
"""
