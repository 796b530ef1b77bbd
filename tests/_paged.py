"""Test-side helpers: build tiny paged pools from logical rows, and glue that runs either the
oracle's or the library's host steps over a synthetic workload. No attention arithmetic."""
from __future__ import annotations

import numpy as np

import synth


def scatter_rows(rows_per_head, page, page_order, D, num_pages=None, fill=0):
    """Place logical token rows into pages.

    rows_per_head: list over heads of uint16[n_h, D] (bf16 bits) in logical order.
    page_order: physical page ids handed out in order (head by head, page by page).
    Returns (pool uint16[P, page, D], page_ids flat, head_count int32[len]).
    """
    counts = [-(-r.shape[0] // page) for r in rows_per_head]
    need = sum(counts)
    P = num_pages if num_pages is not None else max(int(np.max(page_order[:need])) + 1 if need else 1, 1)
    pool = np.full((P, page, D), fill, dtype=np.uint16)
    ids = []
    k = 0
    for r, c in zip(rows_per_head, counts):
        for p in range(c):
            pid = int(page_order[k]); k += 1
            ids.append(pid)
            chunk = r[p * page:(p + 1) * page]
            pool[pid, :chunk.shape[0]] = chunk
    return pool, np.asarray(ids, dtype=np.int32), np.asarray(counts, dtype=np.int32)


def flat_table(ids, counts):
    """One dense row per head laid end to end (a single group whose rows are exactly the
    heads' page lists): returns (table, head_off)."""
    off = np.zeros(len(counts), dtype=np.int64)
    off[1:] = np.cumsum(counts)[:-1]
    return np.asarray(ids, dtype=np.int32), off


def bf16(x):
    return synth.f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def widen(bits):
    return synth.bf16_to_f64(np.asarray(bits))
