"""The compressed transfer protocol between two ranks, on CPU with gloo.

Rank 0 encodes chunks of streams and sends, per chunk, a fixed-size header
(segment count and container sizes) and the packed containers; rank 1
receives and decodes.  The GPU codec needs a GPU, so a codec backed by the
CPU oracle stands in for it here: what is checked is the protocol -- chunk
order, ragged last chunk, empty streams, sizes and offsets of the packed
containers, buffer reuse across overlapping sends."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from lossless_bf16_kv_splitzip_b200.transfer import chunk_ranges, pack_offsets


def test_chunk_ranges_and_offsets():
    assert chunk_ranges(7, 3) == [(0, 3), (3, 6), (6, 7)]
    assert chunk_ranges(0, 4) == []
    with pytest.raises(ValueError):
        chunk_ranges(3, 0)
    offs, total = pack_offsets([5, 0, 7])
    assert list(offs) == [0, 5, 5] and total == 12


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _streams():
    import kvgen
    lens = [3000, 0, 17, 65536 + 9, 2048, 1, 40000]
    return [kvgen.mixed_small(n, seed=900 + i) for i, n in enumerate(lens)]


class OracleChunks:
    """CPU stand-in for the GPU codec, with the same encode/decode interface."""

    def __init__(self, streams, per_chunk):
        import oracle
        oracle.build()
        self.oracle = oracle
        self.streams = streams
        self.chunks = chunk_ranges(len(streams), per_chunk)
        self.out = {}

    def encode(self, c):
        import torch
        a, b = self.chunks[c]
        blobs = [self.oracle.encode(self.streams[i]) for i in range(a, b)]
        payload = torch.from_numpy(np.frombuffer(b"".join(blobs), np.uint8).copy())
        return payload, [len(x) for x in blobs]

    def decode(self, c, payload, sizes):
        a, b = self.chunks[c]
        offs, _ = pack_offsets(sizes)
        raw = payload.numpy().tobytes()
        for k, i in enumerate(range(a, b)):
            blob = raw[int(offs[k]): int(offs[k]) + sizes[k]]
            self.out[i] = (blob, self.oracle.decode(blob, self.streams[i].size))


def _worker(rank, world, port, per_chunk, result_dir):
    import torch
    import torch.distributed as dist

    from lossless_bf16_kv_splitzip_b200.transfer import recv_chunks, send_chunks

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    streams = _streams()
    codec = OracleChunks(streams, per_chunk)
    n_chunks = len(codec.chunks)
    if rank == 0:
        send_chunks(codec, n_chunks, per_chunk, dst=1)
    else:
        recv_chunks(codec, n_chunks, per_chunk, src=0, device=torch.device("cpu"))
        ok = sorted(codec.out) == list(range(len(streams)))
        for i, x in enumerate(streams):
            blob, y = codec.out[i]
            ok = ok and blob == codec.oracle.encode(x) and np.array_equal(y, x)
        with open(os.path.join(result_dir, "ok"), "w") as f:
            f.write("1" if ok else "0")
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("per_chunk", [1, 3])
def test_send_recv_two_ranks(tmp_path, per_chunk):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, per_chunk, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    assert (tmp_path / "ok").read_text() == "1"
