"""Plain restatement of the weight-page bitwidth planner (test infrastructure).

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` alone; the library's planner
never calls it and shares no code with it.

PagedWeight: Efficient MoE LLM Serving with Dynamic Quality-Aware Weight
Quantization, "What carries the argument": under memory pressure the planner
lowers bitwidths of weight pages (expert linear blocks) by taking the actions
with the lowest predicted damage per released byte until the byte target is
met; the predicted damage of an action is d = max{eps, mu * g * eta} with g the
offline sensitivity of the block's bitwidth transition, mu the routing-bucket
multiplier and eta the exponentiated prompt residual. Figure 4: pages are
restored before a higher bitwidth is committed (the restore plan below undoes
reductions, the most damage removed per byte first).

Readings where the pages are silent: one action drops or
restores one bit-plane of one block; a block's floor bitwidth and per-plan
depth cap bound its actions ("bitwidth floor stages", "depth caps"); equal
damage per byte goes to the lower block index; a block's next action is a
candidate only once its previous action was taken; in a restore plan an
action that no longer fits the byte budget ends that block's restores.

The steps are written as a plain scan over all blocks at every step (no
heap): slow and obviously in the order the definition gives.
"""
from __future__ import annotations


def damage(block: dict, b: int, eps: float) -> float:
    """Predicted damage of the transition b -> b-1 of ``block``."""
    return max(eps, block["routing_mult"] * block["sensitivity"][b] * block["prompt_factor"])


def plan_reduce(blocks: list, bytes_target: int, eps: float):
    """Returns (target_met, new_bits, bytes_released)."""
    bits = [b["committed_bits"] for b in blocks]
    lowest = [max(b["floor_bits"], b["committed_bits"] - b["max_steps"]) for b in blocks]
    released = 0
    while released < bytes_target:
        best = None
        for i, blk in enumerate(blocks):
            if bits[i] <= lowest[i]:
                continue
            per_byte = damage(blk, bits[i], eps) / blk["plane_bytes"]
            if best is None or per_byte < best[0]:
                best = (per_byte, i)
        if best is None:
            break
        i = best[1]
        bits[i] -= 1
        released += blocks[i]["plane_bytes"]
    return released >= bytes_target, bits, released


def plan_restore(blocks: list, max_bits: list, bytes_budget: int, eps: float):
    """Returns (new_bits, bytes_used)."""
    bits = [b["committed_bits"] for b in blocks]
    highest = [min(m, b["committed_bits"] + b["max_steps"]) for m, b in zip(max_bits, blocks)]
    stopped = [False] * len(blocks)
    used = 0
    while True:
        best = None
        for i, blk in enumerate(blocks):
            if stopped[i] or bits[i] >= highest[i]:
                continue
            per_byte = damage(blk, bits[i] + 1, eps) / blk["plane_bytes"]
            if best is None or per_byte > best[0]:
                best = (per_byte, i)
        if best is None:
            break
        i = best[1]
        if used + blocks[i]["plane_bytes"] > bytes_budget:
            stopped[i] = True
            continue
        bits[i] += 1
        used += blocks[i]["plane_bytes"]
    return bits, used
