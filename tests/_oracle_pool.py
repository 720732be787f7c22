"""Runs the fp64 oracle over the heads of a large prefill in worker
processes (spawned, never forked: the parent holds a CUDA context).  Each
worker evaluates one query head with the oracle's `attention` on that head's
slices; the head map (query head h reads key/value head h // (Hq // Hkv)) is
applied here, when the slices are cut.  Imports numpy and the oracle only."""

from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np


def _one_head(args):
    from threadpoolctl import threadpool_limits

    from oracle import fp64_attention as orc
    qh, kh, vh, scale, causal = args
    with threadpool_limits(1):  # one core per worker
        O, L = orc.attention(qh[:, :, None], kh[:, :, None], vh[:, :, None], scale, causal)
    return O[:, :, 0], L[:, 0]


def attention_by_head(q, k, v, scale, causal, workers=None):
    """q [B, T, Hq, d], k/v [B, S, Hkv, d] float64 -> O [B, T, Hq, d], LSE [B, Hq, T]."""
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    group = Hq // Hkv
    jobs = [(np.ascontiguousarray(q[:, :, h]), np.ascontiguousarray(k[:, :, h // group]),
             np.ascontiguousarray(v[:, :, h // group]), scale, causal) for h in range(Hq)]
    workers = workers or min(Hq, os.cpu_count() or 1)
    O = np.zeros((B, T, Hq, d))
    L = np.full((B, Hq, T), -np.inf)
    with ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
        for h, (oh, lh) in enumerate(ex.map(_one_head, jobs)):
            O[:, :, h] = oh
            L[:, h] = lh
    return O, L
