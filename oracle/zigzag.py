"""Zigzag pairing of causal prefill shards across cards (plain Python; test infrastructure).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``.  It restates the assignment rule of
"Day 0 Inference Adaptation and Performance Optimization for Hybrid Sparse Attention LLMs",
section 5.2, and of "Rapid Adaptation and Inference Optimization" (Zigzag load balancing). The
sequence is cut into S = 2N contiguous shards. Card i of N takes shard i and shard S-1-i, so
each card pairs an early, cheap shard with a late, expensive one under the causal index. The
per-card results are put back in the original shard order afterwards.
"""
from __future__ import annotations


def assignment(n_cards: int) -> list:
    """[[i, 2N-1-i] for each card i]: the shard indices each card computes."""
    if n_cards < 1:
        raise ValueError("at least one card")
    s = 2 * n_cards
    return [[i, s - 1 - i] for i in range(n_cards)]


def shard_ranges(tokens: int, n_shards: int) -> list:
    """Contiguous [start, end) token ranges of n_shards near-equal shards (the first
    tokens % n_shards shards take one token more)."""
    if n_shards < 1 or tokens < 0:
        raise ValueError("bad split")
    base, extra = divmod(tokens, n_shards)
    out, start = [], 0
    for i in range(n_shards):
        end = start + base + (1 if i < extra else 0)
        out.append((start, end))
        start = end
    return out


def card_positions(tokens: int, n_cards: int) -> list:
    """Token positions each card computes, in the order the card holds them."""
    ranges = shard_ranges(tokens, 2 * n_cards)
    return [[t for sh in pair for t in range(*ranges[sh])] for pair in assignment(n_cards)]


def causal_load(positions) -> int:
    """Index work of a set of query positions under the causal mask: position t scores t + 1
    history positions."""
    return sum(t + 1 for t in positions)


def restore(per_card: list, tokens: int, n_cards: int) -> list:
    """Put per-card results (one item per position, in card_positions order) back in the
    original position order."""
    out = [None] * tokens
    for pos, vals in zip(card_positions(tokens, n_cards), per_card):
        if len(pos) != len(vals):
            raise ValueError("a card returned the wrong number of results")
        for t, v in zip(pos, vals):
            out[t] = v
    return out
