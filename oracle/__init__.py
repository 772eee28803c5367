"""CPU oracle for the Ulysses sequence-parallel attention block.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call, link
or execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference arm use it. The product path is the
CUDA library; it has no CPU fallback.

The oracle is a plain, slow, obviously correct restatement of what the block
computes, written from these pages:

* "mstar.model.components.distributed.sequence_parallel" (API documentation:
  ``sp_seq_split``, ``scatter_sequence``, ``gather_sequence``,
  ``sp_head_slice``, ``sp_head_gather``, ``ulysses_attention``);
* "h3_blackwell_runtime/distributed.py -- Ragged Ulysses sequence-parallel
  transport" (``balanced_ranges``, ``SequenceParallelContext.seq_to_heads`` /
  ``heads_to_seq``);
* "maxdiffusion PR #428: experimental two-phase (head-chunked) Ulysses
  all-to-all" (``ulysses_attention_chunks``);
* "deepspeed/sequence/autosp_vit.py" (``UlyssesSPViTAttention``: replicated
  cls token, non-causal attention).

Every virtual rank is a separate numpy array. Floating-point attention runs in
float64 on the exact upcast of the inputs. Layout operations copy values
without touching them, so they are exercised on raw bit patterns too.

Modules:

* :mod:`oracle.partition` -- balanced ranges, per-rank token counts, head-chunk
  ranges.
* :mod:`oracle.layout` -- scatter/gather of the sequence, head slice/gather,
  seq->head and head->seq exchanges.
* :mod:`oracle.attention` -- float64 softmax attention and the Ulysses block.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against worked examples, closed forms, invariants, a library routine (float64
scaled-dot-product attention) or brute force. No function is "parity
unpinned".
"""

from . import attention, layout, partition  # noqa: F401
