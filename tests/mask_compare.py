"""Mask and output comparison between the CUDA path and the oracle.

A GPU/oracle mask difference is excused only for blocks the oracle marks as
near-threshold (running mass within 1e-4 of tau) or as near-ties at the cut;
every other difference is a failure.  Excused blocks are counted and reported.
"""
from __future__ import annotations

import numpy as np

import oracle


def dense_from_lists(count: np.ndarray, idx: np.ndarray) -> np.ndarray:
    H, Nb = count.shape
    cols = np.arange(Nb)[None, None, :]
    valid = cols < count[:, :, None]
    dense = np.zeros((H, Nb, Nb), dtype=bool)
    hh, II, tt = np.nonzero(valid)
    dense[hh, II, idx[hh, II, tt]] = True
    return dense


def check_mask_format(count: np.ndarray, idx: np.ndarray):
    """rr.h mask format: count in [1, I+1], idx strictly ascending within [0, I],
    the last row dense."""
    H, Nb = count.shape
    I = np.arange(Nb)[None, :]
    assert np.all(count >= 1) and np.all(count <= I + 1), "count out of range"
    assert np.all(count[:, -1] == Nb), "last query block not dense"
    cols = np.arange(Nb)[None, None, :]
    valid = cols < count[:, :, None]
    assert np.all(np.where(valid, (idx >= 0) & (idx <= I[:, :, None]), True)), "idx out of range"
    inc = np.diff(idx, axis=2) > 0
    both = valid[:, :, 1:]
    assert np.all(np.where(both, inc, True)), "idx not strictly ascending"


def compare_masks(count_g, idx_g, count_o, idx_o, m_o, tau, band=1e-4, tie=1e-6):
    """Returns a dict of counts: rows, rows_differing, blocks_band, blocks_tie, blocks_fail."""
    dg = dense_from_lists(count_g, idx_g)
    do = dense_from_lists(count_o, idx_o)
    diff = dg != do
    rows = np.argwhere(diff.any(axis=2))
    stats = {"rows": int(count_o.size), "rows_differing": int(len(rows)), "blocks_band": 0,
             "blocks_tie": 0, "blocks_fail": 0, "fail_examples": []}
    for h, I in rows:
        near, ties = oracle.band_blocks(m_o[h, I], int(I), tau, band, tie)
        for J in np.nonzero(diff[h, I])[0]:
            J = int(J)
            if J in near:
                stats["blocks_band"] += 1
            elif J in ties:
                stats["blocks_tie"] += 1
            else:
                stats["blocks_fail"] += 1
                if len(stats["fail_examples"]) < 5:
                    stats["fail_examples"].append((int(h), int(I), J))
    return stats


def output_errors(o_gpu: np.ndarray, o_ref: np.ndarray):
    """max and mean |o_gpu - o_ref| over the rows o_ref holds (NaN rows skipped)."""
    ok = ~np.isnan(o_ref)
    err = np.abs(o_gpu.astype(np.float64)[ok] - o_ref[ok])
    return float(err.max()), float(err.mean())
