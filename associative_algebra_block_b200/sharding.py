"""Token sharding of the row-typed projections across ranks.

A token's row type comes from its absolute position inside its sequence
(agihunt.info digest, paragraph on the Transformer mapping), so a shard
must not cut a sequence: rank r takes whole packed sequences and keeps the
position rule (sequence length, offset) unchanged.  The forward pass needs no
exchange between ranks (every output row depends on its own input row only);
the backward's weight gradient is a sum over tokens, so the ranks' dW add up
(one all-reduce).
"""
from __future__ import annotations


def token_shard(rows: int, seq_len: int, world: int, rank: int) -> tuple[int, int]:
    """Row range [r0, r1) of ``rank`` when ``rows`` tokens packed as
    sequences of ``seq_len`` are split over ``world`` ranks by whole
    sequences (the last sequence may be short).  Sequences are dealt as
    evenly as possible: the first ``n_seq % world`` ranks take one more."""
    if seq_len <= 0 or world <= 0 or not 0 <= rank < world or rows < 0:
        raise ValueError("bad shard request")
    n_seq = -(-rows // seq_len)
    base, extra = divmod(n_seq, world)
    s0 = rank * base + min(rank, extra)
    s1 = s0 + base + (1 if rank < extra else 0)
    return min(rows, s0 * seq_len), min(rows, s1 * seq_len)
