"""Runs the oracle's per-expert work in a pool of spawned processes.

Test infrastructure: the arithmetic is the oracle's own (``dequant_block``,
``expert_job``, ``routed_jobs``, ``combine``); this module only distributes
the experts of one forward over processes so that full-size layers (hundreds
of experts, each dequantised to fp64) are checked in seconds. It imports
numpy and the oracle only, so that a spawned worker starts quickly, and it is
started with ``spawn`` (a pool forked after the parent touched the GPU would
hang).
"""
from __future__ import annotations

import multiprocessing as mp
import os
from typing import Dict, Optional, Sequence

import numpy as np

import oracle as orc


def _expert_worker(job):
    e, blocks, N, xs, comp, plain = job
    ex = {}
    for b, nm in ((0, "1"), (1, "2")):
        ex["W" + nm] = orc.dequant_block(blocks[b]["blk"])
        if blocks[b].get("A") is not None:
            ex["A" + nm] = blocks[b]["A"]
            ex["B" + nm] = blocks[b]["B"]
    rows = list(comp) + list(plain)
    local = np.zeros(max(rows) + 1, np.int64)
    for i, p in enumerate(rows):
        local[p] = i
    return orc.expert_job(xs, local, ex, N, comp, plain)


def forward(X: np.ndarray, logits: np.ndarray, top_k: int, block_of, N: int, renorm: bool = True,
            rows: Optional[Sequence[int]] = None, comp_top_n: int = 0, procs: Optional[int] = None) -> Dict:
    """The oracle's forward pass with the per-expert jobs in a process pool.

    ``block_of(e)`` returns ``{0: {"blk": <dequant_block dict>, "A": .., "B": ..},
    1: {...}}`` in numpy (A and B fp64 or None)."""
    X64 = np.asarray(X, np.float64)
    E = np.asarray(logits).shape[1]
    r = orc.routed_jobs(X64, logits, top_k, E, renorm, rows, comp_top_n)
    perm = r["perm_token"]
    jobs = []
    for e, comp, plain in r["jobs"]:
        ps = list(comp) + list(plain)
        jobs.append((e, block_of(e), N, X64[perm[ps]], comp, plain))
    n = procs or max(1, min(len(jobs), (os.cpu_count() or 2) - 1, 32))
    O = {}
    if n == 1 or len(jobs) <= 1:
        for j in jobs:
            O.update(_expert_worker(j))
    else:
        with mp.get_context("spawn").Pool(n) as pool:
            for part in pool.imap_unordered(_expert_worker, jobs, chunksize=1):
                O.update(part)
    Y = orc.combine(r["want"], r["w"], r["inv_pos"], O, X64.shape[1])
    return {"Y": Y, "idx": r["idx"], "w": r["w"], "counts": r["counts"], "offsets": r["offsets"],
            "perm_token": perm, "inv_pos": r["inv_pos"]}
