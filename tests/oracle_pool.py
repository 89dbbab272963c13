"""The oracle's containers of many streams, computed in parallel processes.

The pool is started with "spawn", never "fork": the calling test process
already holds a CUDA context, and a process forked after that hangs.  Each
worker imports only the oracle (plain C through ctypes) and returns the
sha256 of each container, so that large containers do not travel back.
"""
import hashlib
import multiprocessing as mp
import os


def _digest(x):
    import oracle
    return hashlib.sha256(oracle.encode(x)).hexdigest()


def oracle_digests(streams, workers=None):
    """sha256 hex digest of oracle.encode(x) for every x in streams, in order."""
    if workers is None:
        workers = max(1, min(8, os.cpu_count() or 1))
    with mp.get_context("spawn").Pool(workers) as pool:
        return pool.map(_digest, streams, chunksize=4)
