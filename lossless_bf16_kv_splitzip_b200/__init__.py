"""SplitZip lossless BF16 KV-cache codec for NVIDIA B200 -- Python binding.

The codec itself is the CUDA library ``libsplitzip.so`` (C ABI in
``include/splitzip.h``).  The functions named ``sz_*`` below map one to one
onto its entry points and only marshal arguments: device pointers are taken
from torch tensors (or plain ints), the stream from torch's current stream.
Every step of encode and decode runs in the library's kernels; there is no
CPU or PyTorch fallback, and a missing or unbuildable library raises.

The helpers at the end (``encode``, ``decode``, ``BatchPlan``) only allocate
buffers with torch and call the ``sz_*`` functions.

Method: "SplitZip: Ultra Fast Lossless KV Compression for Disaggregated LLM
Serving" (gist.science explainer), sections 1-4.
"""
from __future__ import annotations

import ctypes
import re

import numpy as np

from ._build import LIB_PATH, build, is_stale

__all__ = [
    "SzError", "sz_segment", "sz_plan", "sz_histogram_codebook", "sz_encode", "sz_compress", "sz_decode",
    "sz_plan_batched", "sz_histogram_codebook_batched", "sz_encode_batched", "sz_decode_batched",
    "sz_encode_static", "sz_plan_one_pass", "sz_encode_one_pass", "sz_workspace_one_pass_batched",
    "sz_encode_one_pass_batched", "sz_histogram_accumulate", "sz_histogram_accumulate_batched",
    "sz_select_codebook", "sz_select_codebook_batched", "select_codebooks", "sz_set_wait_limit_ns", "sz_debug_set_flags", "sz_tile_elems",
    "sz_version", "encode", "compress", "encode_one_pass", "decode", "BatchPlan", "lib",
    "HEADER_BYTES", "max_bytes", "STATUS",
]

HEADER_BYTES = 48
STATUS = {
    0: "SZ_OK", -1: "SZ_ERR_NULL", -2: "SZ_ERR_TOO_LARGE", -3: "SZ_ERR_CAPACITY",
    -4: "SZ_ERR_ALIGN", -5: "SZ_ERR_CORRUPT", -6: "SZ_ERR_CUDA", -7: "SZ_ERR_DEVICE_TIMEOUT",
    -8: "SZ_ERR_INVALID", -9: "SZ_ERR_WORKSPACE",
}
for _code, _name in STATUS.items():
    globals()[_name] = _code


class SzError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (%d)" % (where, STATUS.get(status, "?"), status))


class sz_segment(ctypes.Structure):
    _fields_ = [("n_elems", ctypes.c_uint64), ("page_begin", ctypes.c_uint64),
                ("out_offset", ctypes.c_uint64), ("tile_begin", ctypes.c_uint64)]


_lib = None


def lib():
    """The loaded libsplitzip.so (built in-tree on first use if missing)."""
    global _lib
    if _lib is None:
        if is_stale():
            build()
        L = ctypes.CDLL(LIB_PATH)
        u64, u32, i32, vp = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int32, ctypes.c_void_p
        pu64 = ctypes.POINTER(ctypes.c_uint64)
        sig = {
            "sz_plan": [u64, pu64, pu64],
            "sz_histogram_codebook": [vp, u64, vp, vp, vp, u64, vp],
            "sz_encode": [vp, u64, vp, vp, u64, vp, vp, vp, u64, vp],
            "sz_decode": [vp, u64, vp, u64, vp, vp, u64, vp],
            "sz_plan_batched": [u32, vp, u64, vp, pu64, pu64, pu64, pu64],
            "sz_histogram_codebook_batched": [u32, vp, u64, vp, u64, vp, vp, vp, u64, vp],
            "sz_encode_batched": [u32, vp, u64, vp, u64, vp, u64, vp, vp, vp, u64, vp],
            "sz_decode_batched": [u32, vp, u64, vp, u64, vp, u64, vp, vp, u64, vp],
            "sz_encode_static": [vp, u64, vp, u64, vp, vp, vp, vp],
            "sz_compress": [vp, u64, vp, u64, vp, vp, vp, vp, u64, vp],
            "sz_plan_one_pass": [u64, pu64, pu64],
            "sz_encode_one_pass": [vp, u64, vp, vp, u64, vp, vp, vp, u64, vp],
            "sz_workspace_one_pass_batched": [u32, u64, pu64],
            "sz_encode_one_pass_batched": [u32, vp, u64, vp, u64, vp, vp, u64, vp, vp, vp, u64, vp],
            "sz_histogram_accumulate": [vp, u64, vp, vp],
            "sz_histogram_accumulate_batched": [u32, vp, u64, vp, u64, vp, vp, vp, vp],
            "sz_select_codebook": [vp, vp, vp, vp],
            "sz_select_codebook_batched": [u32, vp, vp, vp, vp],
            "sz_set_wait_limit_ns": [u64],
            "sz_debug_set_flags": [u32],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = i32
        L.sz_tile_elems.argtypes = []
        L.sz_tile_elems.restype = u64
        L.sz_version.argtypes = []
        L.sz_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def header_symbols(header_text: str):
    """Entry points declared in include/splitzip.h."""
    return sorted(set(re.findall(r"^\s*(?:sz_status|uint64_t|const char \*)\s*(sz_\w+)\(", header_text,
                                 flags=re.M)))


# ------------------------------------------------------------ marshalling
def _p(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    raise TypeError("expected a tensor, an int address or None, got %r" % type(x))


def _s(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str):
    if st != 0:
        raise SzError(st, where)


# --------------------------------------------------------------- entry points
def sz_plan(n: int):
    """-> (max_compressed_bytes, workspace_bytes)"""
    a, b = ctypes.c_uint64(), ctypes.c_uint64()
    _check(lib().sz_plan(n, ctypes.byref(a), ctypes.byref(b)), "sz_plan")
    return a.value, b.value


def sz_histogram_codebook(d_in, n, d_codebook16, d_hist256=None, d_ws=None, ws_bytes=0, stream=None):
    _check(lib().sz_histogram_codebook(_p(d_in), n, _p(d_codebook16), _p(d_hist256), _p(d_ws), ws_bytes,
                                       _s(stream)), "sz_histogram_codebook")


def sz_encode(d_in, n, d_codebook16, d_out, out_cap, d_out_bytes, d_status, d_ws, ws_bytes, stream=None):
    _check(lib().sz_encode(_p(d_in), n, _p(d_codebook16), _p(d_out), out_cap, _p(d_out_bytes), _p(d_status),
                           _p(d_ws), ws_bytes, _s(stream)), "sz_encode")


def sz_compress(d_in, n, d_out, out_cap, d_out_bytes, d_codebook16, d_status, d_ws, ws_bytes, stream=None):
    _check(lib().sz_compress(_p(d_in), n, _p(d_out), out_cap, _p(d_out_bytes), _p(d_codebook16), _p(d_status),
                             _p(d_ws), ws_bytes, _s(stream)), "sz_compress")


def sz_decode(d_in, in_bytes, d_out, n, d_status, d_ws, ws_bytes, stream=None):
    _check(lib().sz_decode(_p(d_in), in_bytes, _p(d_out), n, _p(d_status), _p(d_ws), ws_bytes, _s(stream)),
           "sz_decode")


def sz_plan_batched(seg_elems, page_elems: int):
    """-> (segs: ctypes array of sz_segment, total_pages, n_tiles, out_bytes, workspace_bytes)"""
    n = len(seg_elems)
    elems = (ctypes.c_uint64 * max(n, 1))(*[int(v) for v in seg_elems])
    segs = (sz_segment * max(n, 1))()
    tp, nt, ob, wb = (ctypes.c_uint64() for _ in range(4))
    _check(lib().sz_plan_batched(n, ctypes.addressof(elems), page_elems, ctypes.addressof(segs),
                                 ctypes.byref(tp), ctypes.byref(nt), ctypes.byref(ob), ctypes.byref(wb)),
           "sz_plan_batched")
    return segs, tp.value, nt.value, ob.value, wb.value


def sz_histogram_codebook_batched(n_segs, d_segs, n_tiles, d_pages, page_elems, d_codebooks, d_status, d_ws,
                                  ws_bytes, stream=None):
    _check(lib().sz_histogram_codebook_batched(n_segs, _p(d_segs), n_tiles, _p(d_pages), page_elems,
                                               _p(d_codebooks), _p(d_status), _p(d_ws), ws_bytes, _s(stream)),
           "sz_histogram_codebook_batched")


def sz_encode_batched(n_segs, d_segs, n_tiles, d_pages, page_elems, d_out, out_cap, d_out_bytes, d_status,
                      d_ws, ws_bytes, stream=None):
    _check(lib().sz_encode_batched(n_segs, _p(d_segs), n_tiles, _p(d_pages), page_elems, _p(d_out), out_cap,
                                   _p(d_out_bytes), _p(d_status), _p(d_ws), ws_bytes, _s(stream)),
           "sz_encode_batched")


def sz_decode_batched(n_segs, d_segs, n_tiles, d_in, in_cap, d_pages, page_elems, d_status, d_ws, ws_bytes,
                      stream=None):
    _check(lib().sz_decode_batched(n_segs, _p(d_segs), n_tiles, _p(d_in), in_cap, _p(d_pages), page_elems,
                                   _p(d_status), _p(d_ws), ws_bytes, _s(stream)), "sz_decode_batched")


def sz_encode_static(d_in, n, d_out, out_cap, d_out_bytes, d_codebook16, d_status, stream=None):
    """Compress one tensor using the library's own device scratch array (no
    workspace argument, nothing allocated); n <= 2^28."""
    _check(lib().sz_encode_static(_p(d_in), n, _p(d_out), out_cap, _p(d_out_bytes), _p(d_codebook16),
                                  _p(d_status), _s(stream)), "sz_encode_static")


def sz_plan_one_pass(n: int):
    """-> (max_compressed_bytes for any codebook, workspace_bytes) of sz_encode_one_pass"""
    a, b = ctypes.c_uint64(), ctypes.c_uint64()
    _check(lib().sz_plan_one_pass(n, ctypes.byref(a), ctypes.byref(b)), "sz_plan_one_pass")
    return a.value, b.value


def sz_encode_one_pass(d_in, n, d_codebook16, d_out, out_cap, d_out_bytes, d_status, d_ws, ws_bytes, stream=None):
    _check(lib().sz_encode_one_pass(_p(d_in), n, _p(d_codebook16), _p(d_out), out_cap, _p(d_out_bytes),
                                    _p(d_status), _p(d_ws), ws_bytes, _s(stream)), "sz_encode_one_pass")


def sz_workspace_one_pass_batched(n_segs: int, n_tiles: int) -> int:
    w = ctypes.c_uint64()
    _check(lib().sz_workspace_one_pass_batched(n_segs, n_tiles, ctypes.byref(w)), "sz_workspace_one_pass_batched")
    return w.value


def sz_encode_one_pass_batched(n_segs, d_segs, n_tiles, d_pages, page_elems, d_codebooks, d_out, out_cap,
                               d_out_bytes, d_status, d_ws, ws_bytes, stream=None):
    _check(lib().sz_encode_one_pass_batched(n_segs, _p(d_segs), n_tiles, _p(d_pages), page_elems, _p(d_codebooks),
                                            _p(d_out), out_cap, _p(d_out_bytes), _p(d_status), _p(d_ws), ws_bytes,
                                            _s(stream)), "sz_encode_one_pass_batched")


def sz_histogram_accumulate(d_in, n, d_hist256, stream=None):
    _check(lib().sz_histogram_accumulate(_p(d_in), n, _p(d_hist256), _s(stream)), "sz_histogram_accumulate")


def sz_histogram_accumulate_batched(n_segs, d_segs, n_tiles, d_pages, page_elems, d_hist_index, d_hists, d_status,
                                    stream=None):
    _check(lib().sz_histogram_accumulate_batched(n_segs, _p(d_segs), n_tiles, _p(d_pages), page_elems,
                                                 _p(d_hist_index), _p(d_hists), _p(d_status), _s(stream)),
           "sz_histogram_accumulate_batched")


def sz_select_codebook(d_hist256, d_codebook16, d_escapes=None, stream=None):
    _check(lib().sz_select_codebook(_p(d_hist256), _p(d_codebook16), _p(d_escapes), _s(stream)),
           "sz_select_codebook")


def sz_select_codebook_batched(n_hists, d_hists, d_codebooks, d_escapes=None, stream=None):
    _check(lib().sz_select_codebook_batched(n_hists, _p(d_hists), _p(d_codebooks), _p(d_escapes), _s(stream)),
           "sz_select_codebook_batched")


def sz_set_wait_limit_ns(limit_ns: int):
    _check(lib().sz_set_wait_limit_ns(limit_ns), "sz_set_wait_limit_ns")


def sz_debug_set_flags(flags: int):
    _check(lib().sz_debug_set_flags(flags), "sz_debug_set_flags")


def sz_tile_elems() -> int:
    return int(lib().sz_tile_elems())


def sz_version() -> str:
    return lib().sz_version().decode()


def max_bytes(n: int) -> int:
    return HEADER_BYTES + n + (n + 1) // 2 + 5 * (n - (n + 15) // 16)


# ------------------------------------------------------------ torch helpers
def _torch():
    import torch
    return torch


def _nbytes(t) -> int:
    """Bytes a contiguous tensor holds: the size the library is told."""
    return t.numel() * t.element_size()


def _workspace(workspace, wsb, dev):
    """The caller's workspace (checked: contiguous, on the device, large
    enough) or a new one of the planned size."""
    torch = _torch()
    if workspace is None:
        return torch.empty(max(wsb, 256), dtype=torch.uint8, device=dev)
    if not workspace.is_contiguous() or workspace.device != dev:
        raise ValueError("workspace must be a contiguous tensor on %s" % dev)
    if _nbytes(workspace) < wsb:
        raise ValueError("workspace holds %d bytes, the call needs %d" % (_nbytes(workspace), wsb))
    return workspace


def _u16_view(x):
    torch = _torch()
    if x.dtype in (torch.bfloat16, torch.float16, torch.int16):
        return x.view(torch.int16)
    if x.dtype == torch.uint16:
        return x
    raise TypeError("expected a 16-bit tensor, got %s" % x.dtype)


def encode(x, stream=None, workspace=None):
    """Encode a contiguous 16-bit CUDA tensor.  Returns (container uint8
    tensor sized for the worst case, size int64 tensor [1], status int32
    tensor [1]) -- all on the device, nothing synchronised."""
    torch = _torch()
    x = _u16_view(x.contiguous())
    n = x.numel()
    cap, wsb = sz_plan(n)
    dev = x.device
    ws = _workspace(workspace, wsb, dev)
    cb = torch.empty(16, dtype=torch.uint8, device=dev)
    out = torch.empty(cap, dtype=torch.uint8, device=dev)
    size = torch.zeros(1, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sz_histogram_codebook(x, n, cb, None, ws, _nbytes(ws), stream)
    sz_encode(x, n, cb, out, cap, size, status, ws, _nbytes(ws), stream)
    return out, size, status


def compress(x, stream=None, workspace=None, codebook=None):
    """Histogram, codebook and container of a contiguous 16-bit CUDA tensor
    in one call (two launches up to 2^21 elements).  Returns (container,
    size int64 tensor [1], status int32 tensor [1])."""
    torch = _torch()
    x = _u16_view(x.contiguous())
    n = x.numel()
    cap, wsb = sz_plan(n)
    dev = x.device
    ws = _workspace(workspace, wsb, dev)
    out = torch.empty(cap, dtype=torch.uint8, device=dev)
    size = torch.zeros(1, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sz_compress(x, n, out, cap, size, codebook, status, ws, _nbytes(ws), stream)
    return out, size, status


def encode_one_pass(x, codebook, stream=None, workspace=None):
    """Encode a contiguous 16-bit CUDA tensor with a given codebook (16
    distinct exponents, uint8 CUDA tensor), reading it once.  Returns
    (container uint8 tensor sized for any codebook, size int64 tensor [1],
    status int32 tensor [1])."""
    torch = _torch()
    x = _u16_view(x.contiguous())
    n = x.numel()
    cap, wsb = sz_plan_one_pass(n)
    dev = x.device
    ws = _workspace(workspace, wsb, dev)
    out = torch.empty(cap, dtype=torch.uint8, device=dev)
    size = torch.zeros(1, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sz_encode_one_pass(x, n, codebook, out, cap, size, status, ws, _nbytes(ws), stream)
    return out, size, status


def select_codebooks(hists, stream=None, escapes=True):
    """Codebooks of caller histograms (uint32/int32 CUDA tensor [rows, 256]
    or [256]).  Returns (codebooks uint8 [rows, 16], escape counts int64
    [rows] or None)."""
    torch = _torch()
    if not hists.is_contiguous() or hists.element_size() != 4 or hists.numel() % 256:
        raise ValueError("hists must be a contiguous 32-bit tensor of rows of 256 counts")
    rows = hists.numel() // 256
    cbs = torch.empty((max(rows, 1), 16), dtype=torch.uint8, device=hists.device)
    esc = torch.empty(max(rows, 1), dtype=torch.int64, device=hists.device) if escapes else None
    sz_select_codebook_batched(rows, hists, cbs, esc, stream)
    return cbs[:rows], (esc[:rows] if esc is not None else None)


def decode(container, n, out=None, stream=None, workspace=None):
    """Decode a container (uint8 CUDA tensor) of n elements into an int16
    tensor (bit patterns).  Returns (out, status int32 tensor [1])."""
    torch = _torch()
    dev = container.device
    if not container.is_contiguous():
        raise ValueError("the container must be a contiguous tensor")
    _, wsb = sz_plan(n)
    ws = _workspace(workspace, wsb, dev)
    if out is None:
        out = torch.empty(n, dtype=torch.int16, device=dev)
    elif not out.is_contiguous() or out.device != dev or _nbytes(out) < 2 * n:
        raise ValueError("out must be a contiguous tensor on %s with room for %d 16-bit values" % (dev, n))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sz_decode(container, _nbytes(container), out, n, status, ws, _nbytes(ws), stream)
    return out, status


class BatchPlan:
    """Buffers of one batched encode/decode: the segment table (host and
    device), container buffer, workspace, per-segment sizes and statuses."""

    def __init__(self, seg_elems, page_elems, device="cuda", buffers=True):
        """buffers=False: only the segment table and the statuses (a plan
        of newly written data for ``accumulate``, which needs no container
        buffer or workspace)."""
        torch = _torch()
        self.device = torch.device(device)
        self.seg_elems = [int(v) for v in seg_elems]
        self.page_elems = int(page_elems)
        segs, self.total_pages, self.n_tiles, self.out_bytes, self.ws_bytes = sz_plan_batched(
            self.seg_elems, self.page_elems)
        self.n_segs = len(self.seg_elems)
        self.h_segs = segs
        raw = np.frombuffer(bytes(segs), dtype=np.uint64).reshape(-1, 4)[: self.n_segs]
        self.out_offset = raw[:, 2].copy()
        self.tile_begin = raw[:, 3].copy()
        self.page_begin = raw[:, 1].copy()
        self.d_segs = torch.from_numpy(raw.copy().view(np.int64)).to(device)
        self.container = self.ws = None
        if buffers:
            self.container = torch.empty(max(self.out_bytes, 16), dtype=torch.uint8, device=device)
            self.ws = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=device)
        self.sizes = torch.zeros(max(self.n_segs, 1), dtype=torch.int64, device=device)
        self.codebooks = torch.zeros((max(self.n_segs, 1), 16), dtype=torch.uint8, device=device)
        self.enc_status = torch.zeros(max(self.n_segs, 1), dtype=torch.int32, device=device)
        self.dec_status = torch.zeros(max(self.n_segs, 1), dtype=torch.int32, device=device)

    def histogram(self, d_page_ptrs, stream=None):
        sz_histogram_codebook_batched(self.n_segs, self.d_segs, self.n_tiles, d_page_ptrs, self.page_elems,
                                      self.codebooks, self.enc_status, self.ws, self.ws.numel(), stream)

    def encode_only(self, d_page_ptrs, stream=None):
        sz_encode_batched(self.n_segs, self.d_segs, self.n_tiles, d_page_ptrs, self.page_elems, self.container,
                          self.container.numel(), self.sizes, self.enc_status, self.ws, self.ws.numel(), stream)

    def encode(self, d_page_ptrs, stream=None):
        self.histogram(d_page_ptrs, stream)
        self.encode_only(d_page_ptrs, stream)

    def encode_one_pass(self, d_page_ptrs, d_codebooks, stream=None):
        """Every segment's container with the caller's codebooks (uint8
        [n_segs][16] on the device), reading the input once; the one-pass
        workspace is allocated on first use."""
        torch = _torch()
        if getattr(self, "ws1", None) is None:
            wb = sz_workspace_one_pass_batched(self.n_segs, self.n_tiles)
            self.ws1 = torch.empty(max(wb, 256), dtype=torch.uint8, device=self.device)
        sz_encode_one_pass_batched(self.n_segs, self.d_segs, self.n_tiles, d_page_ptrs, self.page_elems, d_codebooks,
                                   self.container, self.container.numel(), self.sizes, self.enc_status, self.ws1,
                                   self.ws1.numel(), stream)

    def accumulate(self, d_page_ptrs, d_hists, d_hist_index=None, stream=None):
        """Add every segment's exponent counts (the plan describes newly
        written data) to the caller's histograms d_hists (32-bit [rows, 256]
        on the device), segment k into row d_hist_index[k] (uint32/int32
        [n_segs]) or row k.  Per-segment status in self.acc_status."""
        torch = _torch()
        if getattr(self, "acc_status", None) is None:
            self.acc_status = torch.zeros(max(self.n_segs, 1), dtype=torch.int32, device=self.device)
        if not d_hists.is_contiguous() or d_hists.element_size() != 4:
            raise ValueError("d_hists must be a contiguous 32-bit tensor")
        sz_histogram_accumulate_batched(self.n_segs, self.d_segs, self.n_tiles, d_page_ptrs, self.page_elems,
                                        d_hist_index, d_hists, self.acc_status, stream)

    def decode(self, d_page_ptrs, stream=None, container=None):
        """Decode every segment into the pages d_page_ptrs lists.  container:
        another plan's container buffer for the same segment lengths (its
        offsets are the same), e.g. to decode into another page size."""
        c = self.container if container is None else container
        if not c.is_contiguous():
            raise ValueError("the container must be a contiguous tensor")
        sz_decode_batched(self.n_segs, self.d_segs, self.n_tiles, c, _nbytes(c),
                          d_page_ptrs, self.page_elems, self.dec_status, self.ws, self.ws.numel(), stream)

    def container_bytes(self, k: int, size: int) -> "np.ndarray":
        off = int(self.out_offset[k])
        return self.container[off: off + size].cpu().numpy()
