"""The oracle's containers of many streams, computed in parallel processes.

The pool is started with "spawn", never "fork": the calling test process
already holds a CUDA context, and a process forked after that hangs.  Each
worker imports only the oracle (plain C through ctypes) and the input
generators, and returns the sha256 of each container (and, on request, the
exponent histogram), so that large containers do not travel back.
"""
import hashlib
import multiprocessing as mp
import os


def _digest(x):
    import oracle
    return hashlib.sha256(oracle.encode(x)).hexdigest()


def _digest_hist_of(job):
    import oracle
    gen, args = job
    x = gen(*args)
    return hashlib.sha256(oracle.encode(x)).hexdigest(), [int(v) for v in oracle.histogram(x)]


def _workers(workers):
    return workers if workers else max(1, min(8, os.cpu_count() or 1))


def oracle_digests(streams, workers=None):
    """sha256 hex digest of oracle.encode(x) for every x in streams, in order."""
    with mp.get_context("spawn").Pool(_workers(workers)) as pool:
        return pool.map(_digest, streams, chunksize=4)


def oracle_digests_and_histograms(gen, arg_list, workers=None):
    """For every args in arg_list: x = gen(*args) generated in a worker
    (gen: a module-level function, e.g. kvgen.contiguous_tensor), and
    (sha256 of oracle.encode(x), oracle.histogram(x) as 256 ints)."""
    with mp.get_context("spawn").Pool(_workers(workers)) as pool:
        return pool.map(_digest_hist_of, [(gen, tuple(a)) for a in arg_list], chunksize=1)
