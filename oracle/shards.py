"""The oracle on row shards in worker processes -- TEST INFRASTRUCTURE ONLY (tests and the
benchmark's CPU-baseline leg).  Rows are independent once S is fixed, so a tensor's oracle
result is the concatenation of its shards' results at the whole tensor's S.  Workers are
started with the spawn method (never forked from a process that has touched the GPU)."""
from __future__ import annotations

import os

import numpy as np


def shard_job(args):
    """One shard: (x rows float32, kind, S or None, importance or None) -> dict of arrays.
    kind: "nvfp4:<objective>", "nvfp4_had:<objective>", "if4", "if4_sweep", "if4_had",
    "mxfp4", "mxfp4_had", "mxfp4:mx_sweep", "mxfp4_had:mx_sweep"."""
    import oracle as O
    x, kind, S, imp = args
    base, _, obj = kind.partition(":")
    if base.startswith("nvfp4"):
        r = O.nvfp4_quantize(x, obj, importance=imp, S=S, hadamard16=base.endswith("_had"))
        return {"codes": r["codes"], "scales": r["scales"], "gap": r["gap"], "tie": r["tie"], "p": r["p"],
                "p2": r["p2"], "status": r["status"]}
    if base.startswith("if4"):
        sweep = "sweep" if (obj == "if4_sweep" or base == "if4_sweep") else "absmax"
        r = O.if4_quantize(x, S=S, hadamard16=base.endswith("_had"), sweep=sweep)
        return {"codes": r["codes"], "scales": r["scales"], "gap": r["gap"], "tie": r["tie"], "status": r["status"]}
    r = O.mxfp4_quantize(x, hadamard=base.endswith("_had"), sweep="sweep" if obj == "mx_sweep" else "rule")
    return {"codes": r["codes"], "scales": r["scales"], "gap": r["gap"], "tie": r["tie"], "status": r["status"]}


def workers() -> int:
    return max(1, min(64, len(os.sched_getaffinity(0))))


def run_sharded(x, kind, S=None, importance=None, pool=None, shards=None):
    """The oracle on the whole float32 tensor x, split by rows over a spawn-started process pool
    (one shard per worker unless `shards` says otherwise); returns the concatenated arrays."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    import oracle as O
    O.lib()   # built once here, so the workers only load it
    rows = x.shape[0]
    n = shards or workers()
    step = -(-rows // n)
    jobs = [(np.ascontiguousarray(x[a:a + step]), kind, S, importance) for a in range(0, rows, step)]
    own = pool is None
    if own:
        pool = ProcessPoolExecutor(max_workers=min(n, len(jobs)), mp_context=mp.get_context("spawn"))
    try:
        parts = list(pool.map(shard_job, jobs))
    finally:
        if own:
            pool.shutdown()
    out = {k: np.concatenate([p[k] for p in parts]) for k in parts[0] if k != "status"}
    out["status"] = max(p["status"] for p in parts)
    return out
