"""Parallel fp64 oracle for the large parity cases (test infrastructure).

The expert FFN of a whole prefill chunk is ~1.8 TFLOP of fp64 work plus the
closed-form dequantisation of every chosen expert; this runs the oracle's
own functions (oracle.ExpertSource, oracle.expert_ffn) expert by expert in
a pool of worker processes.  Workers are started with the "spawn" method
(never forked from a process that holds a CUDA context) and import only
numpy, the oracle and the seeded input generator.  Nothing is reordered
inside an expert: each worker computes exactly what oracle.moe_layer
computes for that expert's rows.
"""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor
from typing import Optional

import numpy as np

_STATE = {}


def _init(shape, seed: int, layer: int, x_bits: np.ndarray, k: int) -> None:
    from threadpoolctl import threadpool_limits
    threadpool_limits(1)
    import oracle as o
    import synth
    _STATE["src"] = o.ExpertSource(
        shape.H, shape.F, shape.fmt_up_gate, shape.fmt_down,
        lambda e: synth.gen_expert_blob(shape, seed, layer, e))
    _STATE["x"] = x_bits
    _STATE["k"] = k


def _expert_rows(e: int, pairs: np.ndarray):
    import oracle as o
    src = _STATE["src"]
    x = o.bf16_to_f64(_STATE["x"][pairs // _STATE["k"]])
    _, y = o.expert_ffn(x, *src.weights(int(e)))
    src.cache.clear()
    return pairs, y


def expert_outputs(shape, seed: int, layer: int, x_bits: np.ndarray,
                   topk_idx: np.ndarray, workers: Optional[int] = None
                   ) -> np.ndarray:
    """y_pairs [T*k, H] in float64 for the routing topk_idx [T, k]: every
    pair through the oracle's dense FFN on its expert's dequantised
    weights (oracle.group_pairs gives the pairs of each expert)."""
    import oracle as o
    T, k = topk_idx.shape
    off, pairs, act = o.group_pairs(topk_idx, shape.E)
    y = np.empty((T * k, shape.H))
    n = workers or max(1, min(32, (os.cpu_count() or 2) - 1))
    ctx = mp.get_context("spawn")
    # largest experts first, so the pool drains evenly
    order = sorted(act, key=lambda e: -(off[e + 1] - off[e]))
    with ProcessPoolExecutor(n, mp_context=ctx, initializer=_init,
                             initargs=(shape, seed, layer, x_bits, k)) as ex:
        futs = [ex.submit(_expert_rows, int(e),
                          pairs[off[e]:off[e + 1]].astype(np.int64))
                for e in order]
        for f in futs:
            pp, yy = f.result()
            y[pp] = yy
    return y
