"""Compressed KV transfer: chunked encode -> send -> receive -> decode.

The explainer's setting (section 1 "Le probleme": a prefill server hands
the KV cache of a request to a decode server; "Les Resultats": the transfer
gets faster by the compression ratio when the codec outruns the link).  The
cache is cut into chunks of whole tensors (or requests); chunk c+1 is
encoded while chunk c crosses the link and chunk c-1 is decoded, so the
codec's time hides behind the link's.

Two forms:

* ``host_transfer`` -- one GPU: the link is PCIe through pinned host memory
  (device-to-host copy, then host-to-device copy into the receiving
  buffers), both directions running at once on their own streams.  This is
  what a KV hand-off staged through host memory (an RDMA NIC's bounce
  buffer) costs, and the only link one GPU has.
* ``send_chunks`` / ``recv_chunks`` -- two ranks of a ``torch.distributed``
  group (NCCL between GPUs): per chunk, the container sizes, then the packed
  containers, sent with non-blocking point-to-point calls so that the next
  chunk is encoded while the previous one is in flight.

The codec is an object with ``encode(c) -> (payload uint8 tensor, sizes
list)`` and ``decode(c, payload, sizes)``; ``SplitZipChunks`` is the one
backed by the library's batched calls.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def chunk_ranges(n_units: int, per_chunk: int):
    """[(first, end)) unit ranges of at most per_chunk units, in order."""
    if per_chunk < 1:
        raise ValueError("per_chunk must be >= 1")
    return [(i, min(i + per_chunk, n_units)) for i in range(0, n_units, per_chunk)]


def pack_offsets(sizes):
    """Byte offsets of containers laid end to end, and the total."""
    off = np.zeros(len(sizes) + 1, dtype=np.int64)
    np.cumsum(np.asarray(sizes, dtype=np.int64), out=off[1:])
    return off[:-1], int(off[-1])


kBuffers = 3  # payload buffers per side: chunk c uses c % kBuffers


class SplitZipChunks:
    """The library's codec over a contiguous [S, n] cache of 16-bit tensors
    cut into chunks of ``per_chunk`` tensors (one codebook per tensor).

    encode(c): the chunk's containers packed end to end (device uint8) and
    their sizes; decode(c, payload, sizes): unpacks into the receiving
    plan's container buffer and decodes into ``out``.  The sizes of chunk c
    reach pinned host memory on the encode's own stream, so the host can
    read them after waiting for that stream alone."""

    def __init__(self, src, out, per_chunk: int, device):
        import torch

        from . import BatchPlan
        S, n = src.shape
        self.n = n
        self.chunks = chunk_ranges(S, per_chunk)
        self.src, self.out = src, out
        self.tx, self.rx, self.in_ptrs, self.out_ptrs, self.host_sizes = [], [], [], [], []
        for a, b in self.chunks:
            self.tx.append(BatchPlan([n] * (b - a), n, device=device))
            self.rx.append(BatchPlan([n] * (b - a), n, device=device))
            self.in_ptrs.append(torch.tensor([src.data_ptr() + 2 * n * k for k in range(a, b)],
                                             dtype=torch.int64, device=device))
            self.out_ptrs.append(torch.tensor([out.data_ptr() + 2 * n * k for k in range(a, b)],
                                              dtype=torch.int64, device=device))
            self.host_sizes.append(torch.zeros(b - a, dtype=torch.int64, pin_memory=True))
        cap = max(int(p.container.numel()) for p in self.tx)
        self.payload = [torch.empty(cap, dtype=torch.uint8, device=device) for _ in range(kBuffers)]
        self.rx_payload = [torch.empty(cap, dtype=torch.uint8, device=device) for _ in range(kBuffers)]

    def encode_async(self, c, stream):
        """Encode chunk c on ``stream``; its sizes follow to pinned memory."""
        import torch
        self.tx[c].encode(self.in_ptrs[c], stream)
        with torch.cuda.stream(stream):
            self.host_sizes[c].copy_(self.tx[c].sizes[: self.tx[c].n_segs], non_blocking=True)

    def sizes(self, c):
        """Chunk c's container sizes; the encode's stream must have reached them."""
        return [int(v) for v in self.host_sizes[c].numpy()]

    def pack(self, c, sizes):
        """The chunk's containers end to end in payload buffer c % kBuffers."""
        plan = self.tx[c]
        buf = self.payload[c % kBuffers]
        offs, total = pack_offsets(sizes)
        for k, z in enumerate(sizes):
            o = int(plan.out_offset[k])
            buf[int(offs[k]): int(offs[k]) + z].copy_(plan.container[o: o + z], non_blocking=True)
        return buf[:total]

    def encode(self, c):
        import torch
        st = torch.cuda.current_stream(self.src.device)
        self.encode_async(c, st)
        st.synchronize()
        sizes = self.sizes(c)
        return self.pack(c, sizes), sizes

    def unpack(self, c, payload, sizes):
        plan = self.rx[c]
        offs, _ = pack_offsets(sizes)
        for k, z in enumerate(sizes):
            o = int(plan.out_offset[k])
            plan.container[o: o + z].copy_(payload[int(offs[k]): int(offs[k]) + z], non_blocking=True)

    def decode(self, c, payload, sizes, stream=None):
        self.unpack(c, payload, sizes)
        self.rx[c].decode(self.out_ptrs[c], stream)

    def statuses_ok(self):
        return all(int(p.enc_status.abs().sum()) == 0 for p in self.tx) and \
            all(int(p.dec_status.abs().sum()) == 0 for p in self.rx)


@dataclass
class TransferResult:
    seconds: float      # first encode (or copy) to the last decode (or copy), device time
    link_bytes: int     # bytes that crossed the link (each direction)
    chunks: int
    placed: list        # (staging offset, bytes) of every chunk


def host_transfer(codec: SplitZipChunks | None, src, out, per_chunk: int, staging, align: int = 4096):
    """One GPU: move the [S, n] cache ``src`` into ``out`` through the pinned
    host buffer ``staging``, chunk by chunk: one device-to-host copy and one
    host-to-device copy per chunk, each on its own stream, so that chunk c+1
    goes out while chunk c comes in.  With a codec the chunk's containers
    cross: encoded, then packed end to end on a stream of their own (the
    copy streams only copy), and on the other side unpacked into the
    receiving plan and decoded; three payload buffers per side rotate.
    Without a codec the raw 16-bit values cross.  Chunks start at
    ``align``-byte offsets of ``staging``.  Returns device time, bytes that
    crossed, and where each chunk was staged."""
    import torch
    dev = src.device
    S, n = src.shape
    chunks = chunk_ranges(S, per_chunk) if codec is None else codec.chunks
    s_enc, s_pack, s_d2h, s_h2d, s_dec = (torch.cuda.Stream(dev) for _ in range(5))
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)

    def events():
        return [torch.cuda.Event() for _ in chunks]
    enc_done, pack_done, d2h_done, h2d_done, unpacked = events(), events(), events(), events(), events()
    cur = torch.cuda.current_stream(dev)
    cur.synchronize()
    start.record(s_enc)
    for st in (s_pack, s_d2h, s_h2d, s_dec):
        st.wait_event(start)
    if codec is not None:  # all encodes go ahead on their own stream
        for c in range(len(chunks)):
            codec.encode_async(c, s_enc)
            enc_done[c].record(s_enc)
    src_u8 = src.view(torch.uint8).view(S, 2 * n)
    out_u8 = out.view(torch.uint8).view(S, 2 * n)
    pos = 0
    moved = 0
    placed = []
    for c, (a, b) in enumerate(chunks):
        if codec is not None:
            enc_done[c].synchronize()  # the host needs the sizes to size the copies
            sizes = codec.sizes(c)
            nb = pack_offsets(sizes)[1]
        else:
            nb = (b - a) * 2 * n
        if pos + nb > staging.numel():
            raise ValueError("staging buffer too small: %d bytes needed" % (pos + nb))
        if codec is not None:
            with torch.cuda.stream(s_pack):
                s_pack.wait_event(enc_done[c])
                if c >= kBuffers:  # the buffer's previous chunk has gone out
                    s_pack.wait_event(d2h_done[c - kBuffers])
                payload = codec.pack(c, sizes)
            pack_done[c].record(s_pack)
        with torch.cuda.stream(s_d2h):
            if codec is not None:
                s_d2h.wait_event(pack_done[c])
                staging[pos: pos + nb].copy_(payload, non_blocking=True)
            else:
                staging[pos: pos + nb].copy_(src_u8[a:b].reshape(-1), non_blocking=True)
        d2h_done[c].record(s_d2h)
        with torch.cuda.stream(s_h2d):
            s_h2d.wait_event(d2h_done[c])
            if codec is not None:
                if c >= kBuffers:  # the buffer's previous chunk has been unpacked
                    s_h2d.wait_event(unpacked[c - kBuffers])
                land = codec.rx_payload[c % kBuffers][:nb]
                land.copy_(staging[pos: pos + nb], non_blocking=True)
            else:
                out_u8[a:b].reshape(-1).copy_(staging[pos: pos + nb], non_blocking=True)
        h2d_done[c].record(s_h2d)
        if codec is not None:
            with torch.cuda.stream(s_dec):
                s_dec.wait_event(h2d_done[c])
                codec.unpack(c, land, sizes)
                unpacked[c].record(s_dec)
                codec.rx[c].decode(codec.out_ptrs[c], s_dec)
        placed.append((pos, nb))
        pos += (nb + align - 1) // align * align
        moved += nb
    for st in (s_pack, s_d2h, s_h2d, s_enc):
        s_dec.wait_stream(st)
    end.record(s_dec)
    end.synchronize()
    cur.wait_stream(s_dec)
    return TransferResult(start.elapsed_time(end) / 1e3, moved, len(chunks), placed)


# ------------------------------------------------------------- two ranks
def send_chunks(codec, n_chunks: int, max_segs: int, dst: int, group=None):
    """Sender side: per chunk, encode, then send a fixed-size header (the
    chunk's segment count and sizes, int64[max_segs + 1]) and the packed
    containers to rank ``dst`` without waiting, so that the next chunk's
    encode overlaps the transfer.  The codec's payload buffers rotate (chunk
    c uses buffer c % kBuffers), so the sends of a chunk are waited for before
    its buffer is reused."""
    import torch
    import torch.distributed as dist
    pending = [None] * kBuffers
    for c in range(n_chunks):
        if pending[c % kBuffers] is not None:
            for w in pending[c % kBuffers][0]:
                w.wait()
        payload, sizes = codec.encode(c)
        if len(sizes) > max_segs:
            raise ValueError("chunk %d has %d segments, more than max_segs=%d" % (c, len(sizes), max_segs))
        meta = torch.zeros(max_segs + 1, dtype=torch.int64, device=payload.device)
        meta[0] = len(sizes)
        if sizes:
            meta[1: 1 + len(sizes)] = torch.tensor(sizes, dtype=torch.int64)
        works = [dist.isend(meta, dst, group=group)]
        if payload.numel():
            works.append(dist.isend(payload, dst, group=group))
        pending[c % kBuffers] = (works, meta, payload)  # buffers stay alive until their sends end
    for p in pending:
        if p is not None:
            for w in p[0]:
                w.wait()


def recv_chunks(codec, n_chunks: int, max_segs: int, src: int, device, group=None):
    """Receiver side: per chunk, the header, then the packed containers,
    then decode."""
    import torch
    import torch.distributed as dist
    for c in range(n_chunks):
        meta = torch.zeros(max_segs + 1, dtype=torch.int64, device=device)
        dist.irecv(meta, src, group=group).wait()
        k = int(meta[0].item())
        if k > max_segs:
            raise ValueError("header of chunk %d names %d segments" % (c, k))
        sizes = [int(v) for v in meta[1: 1 + k].tolist()]
        total = int(sum(sizes))
        payload = torch.empty(total, dtype=torch.uint8, device=device)
        if total:
            dist.irecv(payload, src, group=group).wait()
        codec.decode(c, payload, sizes)


# ------------------------------------------------------- host round trip
def host_round_trip(codec: SplitZipChunks, h_in, h_out, staging, align: int = 4096):
    """One GPU, through the public calls: the pinned host cache ``h_in``
    ([S, n] int16) is uploaded chunk by chunk into the codec's ``src``,
    encoded, its containers packed and downloaded into ``staging``,
    uploaded again, decoded into the codec's ``out`` and downloaded into
    ``h_out``.  Uploads and downloads run on their own streams (input
    uploads apart from container uploads, container downloads apart from
    output downloads), so both directions of the link stay busy while the
    kernels run in between.  Returns (device seconds, bytes uploaded, bytes
    downloaded)."""
    import torch
    src, out = codec.src, codec.out
    dev = src.device
    chunks = codec.chunks
    s_in, s_enc, s_pack, s_cd, s_cu, s_dec, s_out = (torch.cuda.Stream(dev) for _ in range(7))
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)

    def events():
        return [torch.cuda.Event() for _ in chunks]
    up, enc_done, pack_done, down, cup, unpacked, dec_done = (events() for _ in range(7))
    cur = torch.cuda.current_stream(dev)
    cur.synchronize()
    start.record(s_in)
    for st in (s_enc, s_pack, s_cd, s_cu, s_dec, s_out):
        st.wait_event(start)

    def launch_front(c):  # upload chunk c's input and encode it
        a, b = chunks[c]
        with torch.cuda.stream(s_in):
            src[a:b].copy_(h_in[a:b], non_blocking=True)
        up[c].record(s_in)
        s_enc.wait_event(up[c])
        codec.encode_async(c, s_enc)
        enc_done[c].record(s_enc)

    ahead = min(2, len(chunks))
    for c in range(ahead):
        launch_front(c)
    pos = 0
    n_up = n_down = 0
    for c, (a, b) in enumerate(chunks):
        enc_done[c].synchronize()  # the host needs the sizes to size the copies
        sizes = codec.sizes(c)
        nb = pack_offsets(sizes)[1]
        if pos + nb > staging.numel():
            raise ValueError("staging buffer too small: %d bytes needed" % (pos + nb))
        with torch.cuda.stream(s_pack):
            s_pack.wait_event(enc_done[c])
            if c >= kBuffers:
                s_pack.wait_event(down[c - kBuffers])
            payload = codec.pack(c, sizes)
        pack_done[c].record(s_pack)
        with torch.cuda.stream(s_cd):
            s_cd.wait_event(pack_done[c])
            staging[pos: pos + nb].copy_(payload, non_blocking=True)
        down[c].record(s_cd)
        with torch.cuda.stream(s_cu):
            s_cu.wait_event(down[c])
            if c >= kBuffers:
                s_cu.wait_event(unpacked[c - kBuffers])
            land = codec.rx_payload[c % kBuffers][:nb]
            land.copy_(staging[pos: pos + nb], non_blocking=True)
        cup[c].record(s_cu)
        with torch.cuda.stream(s_dec):
            s_dec.wait_event(cup[c])
            codec.unpack(c, land, sizes)
            unpacked[c].record(s_dec)
            codec.rx[c].decode(codec.out_ptrs[c], s_dec)
        dec_done[c].record(s_dec)
        with torch.cuda.stream(s_out):
            s_out.wait_event(dec_done[c])
            h_out[a:b].copy_(out[a:b], non_blocking=True)
        if c + ahead < len(chunks):
            launch_front(c + ahead)
        pos += (nb + align - 1) // align * align
        n_up += 2 * (b - a) * src.shape[1] + nb
        n_down += nb + 2 * (b - a) * src.shape[1]
    for st in (s_in, s_enc, s_pack, s_cd, s_cu, s_dec):
        s_out.wait_stream(st)
    end.record(s_out)
    end.synchronize()
    cur.wait_stream(s_out)
    return start.elapsed_time(end) / 1e3, n_up, n_down
