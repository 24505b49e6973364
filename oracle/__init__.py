"""CPU fp64 oracle of the Ulysses sequence-parallel hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run anything under
``oracle/``.  The product path (the CUDA library and its Python binding) never
does, and the oracle imports nothing from it.

Pages followed (cited by title and section):
  [TF-ALST]  Transformers docs, "Ulysses sequence parallelism" (the DeepSpeed
             ALST page): the seq-sharded -> head-sharded -> seq-sharded figure;
             "Configuration" (head count divisible by sp_size, padding to a
             multiple of sp_size, position_ids instead of a 4D mask).
  [ACC-SP]   Accelerate concept guide, "Sequence parallelism": "How Ulysses SP
             differs from FSDP CP"; "ALST/Ulysses SP backend configuration"
             (packed samples must not attend across sample boundaries).
  [BLOG]     "Ulysses Sequence Parallelism: Training with Million-Token
             Contexts": "How Ulysses works" steps 1-6 (sharding, all-to-all,
             local attention, inverse all-to-all; heads are independent);
             "Communication complexity"; the position_ids masking paragraph;
             "Loss aggregation".
  [ACC-SP] also: the custom training loop's weighted per-rank loss
             aggregation (labels -100 excluded, zero-token ranks skipped,
             division by max(total, 1)).

Every function here is pinned by ``tests/test_oracle_*.py`` against something
other than itself (brute force, closed forms, a library routine, finite
differences, the figure's worked layout).  Nothing here is "parity unpinned".
"""
from .ulysses_oracle import *  # noqa: F401,F403
from .ulysses_oracle import __all__  # noqa: F401
