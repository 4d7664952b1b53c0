"""fp64 CPU oracle for packed-sequence (THD) causal attention under load-balanced
KV-all-gather context parallelism.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call, link or
execute anything in this package; only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` use it.  It shares no code with
the CUDA library: it is a plain, slow, obviously correct restatement of what the
method computes, written from the MindSpeed pull request #3820 ("feat: kvallgather
cp thd load balance"):

  * section "What this PR does / why we need it?": load-balanced KV-all-gather
    context parallelism for the THD format, EOD-aware symmetric sequence
    partitioning, direct rank-major K/V indexing, metadata caching, and MHA / GQA
    / expanded MLA head layouts;
  * section "Does this PR introduce any user-facing change?": causal attention
    with EOD attention-mask reset over THD packed sequences, each packed
    subsequence length divisible by 2 * context_parallel_size.

Modules:
  partition  -- validation, the symmetric two-chunk partition, load-balance counts
  tiles      -- the cached per-tile metadata table, built by brute-force enumeration
  attention  -- fp64 forward / backward, full and sampled, plus brute-force forms
"""
from . import partition, tiles, attention  # noqa: F401
