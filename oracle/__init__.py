"""Float64 CPU oracle for paged attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
(``paged_kv_cache_483_b200``) never imports it, and this package imports
nothing from the product: the two share no code.  It is deliberately plain
and slow; every function names the page passage it restates.

Pages this oracle follows (cited by title and section):
  * "abhik.ai examples/pagedattention.py" -- ``KVPool``: physical pool,
    allocation order, append, fork, copy-on-write, release, gather, Eq. 3.
  * "vladkulikov.com modern-llms module 9 notebook" -- ``PagedKVPool``:
    multi-token append with preflight, share_prefix, fill accounting,
    snapshot, validate.
  * "docs.rs ferrum-kv 0.4.0 src/attention.rs" -- ``paged_attention``: GQA
    grouping, the causal rule max_visible = kv_len - q_tokens + qt, softmax.
  * "semidirectx cmu11-667 lecture19 infer_world.py", section 3 (online
    softmax and tiled attention) -- the (m, l, acc) recurrence.
  * "vladkulikov.com modern-llms module 9 notebook", prefix-hash trace --
    ``PrefixCache``: content-keyed identity of full blocks.
  * "vladkulikov.com modern-llms module 9 notebook", KV quantisation --
    ``quantize_rows``: per-row absmax integer codes; ``quantize_rows_fp8``:
    the same per-row absmax recipe on the E4M3 grid of the OCP 8-bit
    floating point specification (a reading: the pages quantise to integers).
  * "vladkulikov.com modern-llms module 9 notebook", streaming and
    sliding-window caches -- ``visible_positions``: sink + recent window.

Parity status: every function is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_pins.py`` and its neighbours (page-printed traces, closed forms, brute force
in 40-digit decimal arithmetic, invariants).  No function is unpinned.
"""

from .kv_pool import KVPool, PoolError, PoolExhausted  # noqa: F401
from .prefix_cache import PrefixCache, prefix_key, run_prefix_trace, trace_tokens  # noqa: F401
from .quant import quantize_rows, dequantize_rows, fake_quantize_rows, stored_rows  # noqa: F401
from .quant import (  # noqa: F401
    E4M3_MAX, e4m3_values, e4m3_round, quantize_rows_fp8, dequantize_rows_fp8, stored_rows_fp8,
)
from .attention import (  # noqa: F401
    attention_two_pass, paged_attention, attention_tiled, partition_stats,
    combine_partitions, attention_split_kv, online_softmax_stats,
    visible_positions, attention_window,
)
