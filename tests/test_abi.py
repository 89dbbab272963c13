"""The C-ABI library loads, exports every entry point of include/splitzip.h,
and its host-only logic (plans, argument checks) behaves as documented.
No call here reaches the device: every argument error is caught before the
first CUDA call, and sz_plan / sz_plan_batched are host arithmetic."""
import ctypes
import os

import pytest

import lossless_bf16_kv_splitzip_b200 as sz
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "splitzip.h")


def test_library_exports_every_declared_symbol():
    names = sz.header_symbols(open(HEADER).read())
    assert {"sz_plan", "sz_histogram_codebook", "sz_encode", "sz_decode", "sz_plan_batched",
            "sz_histogram_codebook_batched", "sz_encode_batched", "sz_decode_batched"} <= set(names)
    L = ctypes.CDLL(sz.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert sz.sz_version().startswith("splitzip-b200")
    assert sz.sz_tile_elems() == 65536


def test_binding_wraps_every_declared_symbol_by_its_name():
    # the Python layer has one function per C entry point, same name, exported
    names = sz.header_symbols(open(HEADER).read())
    for n in names:
        assert callable(getattr(sz, n, None)), n
        assert n in sz.__all__, n
    for n in sz.__all__:
        assert hasattr(sz, n), n
    # and argument types are declared for every entry point the header names
    L = sz.lib()
    for n in names:
        assert getattr(L, n).argtypes is not None, n


def test_library_is_built_for_sm100a():
    # the cubin is embedded for sm_100a; the host code reports its target
    assert "sm_100a" in sz.sz_version()


@pytest.mark.parametrize("n", [0, 1, 2, 17, 16384, 65536, 65537, 1 << 25, (1 << 27) - 1, 1 << 27, (1 << 32) - 2,
                               (1 << 32) - 1])
def test_plan_worst_case_bound(n):
    cap, ws = sz.sz_plan(n)
    assert cap == 48 + n + (n + 1) // 2 + 5 * (n - (n + 15) // 16)
    # streams below 2^27 elements are cut into 16,384-element tiles (one
    # sub-tile each), longer ones into 65,536-element tiles (four)
    tile = 16384 if n < 1 << 27 else 65536
    tiles = -(-n // tile)
    ranges = min(tiles, 1024)
    # segment histogram, tile count, completion count and record; the first-
    # and last-piece histograms and the record of every range; sub-tile
    # escape starts
    need = 1024 + 4 + 4 + 32 + 2048 * ranges + 16 * ranges + 4 * ((tile // 16384) * tiles + 1)
    assert need <= ws
    if n <= 1 << 20:  # also the one-call compression's scratch: counts of every 4,096-element slice
        nb = max(1, -(-n // 4096))
        small = -(-(-(-(1536 + 4 * nb) // 256) * 256 + 1024 * nb) // 256) * 256
        assert small <= ws <= max(small, need + 6 * 256)
    else:
        assert ws <= need + 6 * 256
    assert ws % 256 == 0


def test_plan_rejects_too_large():
    with pytest.raises(sz.SzError) as e:
        sz.sz_plan(1 << 32)
    assert e.value.status == sz.SZ_ERR_TOO_LARGE


def test_plan_batched_layout():
    elems = [16384 * 3, 0, 16384 * 5 + 64, 100]
    segs, pages, tiles, out, ws = sz.sz_plan_batched(elems, 16384)
    rows = [(s.n_elems, s.page_begin, s.out_offset, s.tile_begin) for s in segs][: len(elems)]
    assert [r[0] for r in rows] == elems
    assert [r[1] for r in rows] == [0, 3, 3, 9]
    assert [r[3] for r in rows] == [0, 3, 3, 9]
    assert pages == 10 and tiles == 10
    off = 0
    for r, n in zip(rows, elems):
        assert r[2] == off and r[2] % 256 == 0
        off += -(-sz.max_bytes(n) // 256) * 256
    assert out == off
    assert ws > 0


def test_plan_batched_tiles_inside_pages():
    # pages of 150016 elements: tiles of 65536, 65536, 18944 per page
    segs, pages, tiles, out, ws = sz.sz_plan_batched([400000], 150016)
    assert pages == 3
    assert tiles == 3 + 3 + 2  # 2 full pages x 3 tiles, last page of 99968: 2 tiles
    segs, pages, tiles, out, ws = sz.sz_plan_batched([100000], 40000)
    assert pages == 3 and tiles == 3  # pages shorter than a tile: one tile each


def test_plan_batched_page_alignment():
    with pytest.raises(sz.SzError) as e:
        sz.sz_plan_batched([1000], 100)  # several pages of 100 elements
    assert e.value.status == sz.SZ_ERR_ALIGN
    sz.sz_plan_batched([50], 100)  # one partial page: fine


# ---- host-side argument errors (fake addresses are never dereferenced)
A = 1 << 40  # a 16-byte aligned fake device address


def _status(f, *args):
    return f(*args)


def test_encode_argument_errors():
    L = sz.lib()
    cap, ws = sz.sz_plan(1000)
    # null output
    assert L.sz_encode(A, 1000, A, None, cap, A, A, A, ws, None) == sz.SZ_ERR_NULL
    # status word required
    assert L.sz_encode(A, 1000, A, A, cap, A, None, A, ws, None) == sz.SZ_ERR_NULL
    # misaligned output
    assert L.sz_encode(A, 1000, A, A + 4, cap, A, A, A, ws, None) == sz.SZ_ERR_ALIGN
    # misaligned input
    assert L.sz_encode(A + 2, 1000, A, A, cap, A, A, A, ws, None) == sz.SZ_ERR_ALIGN
    # capacity below 48 + n + ceil(n/2)
    assert L.sz_encode(A, 1000, A, A, 48 + 1000 + 499, A, A, A, ws, None) == sz.SZ_ERR_CAPACITY
    # workspace too small
    assert L.sz_encode(A, 1000, A, A, cap, A, A, A, ws - 1, None) == sz.SZ_ERR_WORKSPACE
    # too large
    assert L.sz_encode(A, 1 << 32, A, A, cap, A, A, A, ws, None) == sz.SZ_ERR_TOO_LARGE


def test_histogram_and_decode_argument_errors():
    L = sz.lib()
    cap, ws = sz.sz_plan(1000)
    assert L.sz_histogram_codebook(None, 1000, A, None, A, ws, None) == sz.SZ_ERR_NULL
    assert L.sz_histogram_codebook(A, 1000, A, None, A + 8, ws, None) == sz.SZ_ERR_ALIGN
    assert L.sz_histogram_codebook(A, 1000, A, None, A, 16, None) == sz.SZ_ERR_WORKSPACE
    assert L.sz_decode(A, cap, A, 1000, None, A, ws, None) == sz.SZ_ERR_NULL  # status required
    assert L.sz_decode(A + 1, cap, A, 1000, A, A, ws, None) == sz.SZ_ERR_ALIGN
    assert L.sz_decode(A, cap, A, 1000, A, A, 0, None) == sz.SZ_ERR_WORKSPACE


def test_batched_argument_errors():
    L = sz.lib()
    assert L.sz_encode_batched(0, None, 0, None, 16384, None, 0, None, None, None, 0, None) == sz.SZ_OK
    assert L.sz_encode_batched(2, A, 4, A, 16384, A, 1 << 20, A, None, A, 1 << 20, None) == sz.SZ_ERR_NULL
    assert L.sz_encode_batched(2, A, 4, A, 0, A, 1 << 20, A, A, A, 1 << 20, None) == sz.SZ_ERR_INVALID
    assert L.sz_encode_batched(2, A, 4, A, 16384, A + 8, 1 << 20, A, A, A, 1 << 20, None) == sz.SZ_ERR_ALIGN
    assert L.sz_histogram_codebook_batched(2, A, 4, A, 16384, None, None, A, 1 << 20, None) == sz.SZ_ERR_NULL
    assert L.sz_histogram_codebook_batched(2, A, 4, A, 16384, None, A, A, 16, None) == sz.SZ_ERR_WORKSPACE
    assert L.sz_decode_batched(2, A, 4, A + 4, 1 << 20, A, 16384, A, A, 1 << 20, None) == sz.SZ_ERR_ALIGN
    assert L.sz_decode_batched(2, A, 4, A, 1 << 20, A, 16384, A, A, 16, None) == sz.SZ_ERR_WORKSPACE


def test_helpers_check_caller_buffers_before_any_call():
    # every check below raises on the host, before the library is called, so
    # host tensors serve: an undersized workspace or output buffer would
    # otherwise be written past its end by the device
    torch = pytest.importorskip("torch")
    x = torch.zeros(70_000, dtype=torch.bfloat16)
    _, wsb = sz.sz_plan(x.numel())
    small_ws = torch.empty(wsb - 1, dtype=torch.uint8)
    for helper in (sz.encode, sz.compress):
        with pytest.raises(ValueError, match="workspace"):
            helper(x, workspace=small_ws)
    _, wsb1 = sz.sz_plan_one_pass(x.numel())
    with pytest.raises(ValueError, match="workspace"):
        sz.encode_one_pass(x, torch.arange(16, dtype=torch.uint8), workspace=torch.empty(wsb1 - 1, dtype=torch.uint8))
    # the workspace size is counted in bytes, whatever its dtype
    with pytest.raises(ValueError, match="workspace"):
        sz.encode(x, workspace=torch.empty((wsb - 1) // 4, dtype=torch.int32))
    blob = torch.zeros(1000, dtype=torch.uint8)
    with pytest.raises(ValueError, match="room for 300"):
        sz.decode(blob, 300, out=torch.empty(299, dtype=torch.int16))
    with pytest.raises(ValueError, match="room for 300"):
        sz.decode(blob, 300, out=torch.empty(600, dtype=torch.int16)[::2])
    with pytest.raises(ValueError, match="contiguous"):
        sz.decode(torch.zeros(2000, dtype=torch.uint8)[::2], 300)
    assert sz.sz_plan(300)[1] > 0
    with pytest.raises(ValueError, match="workspace"):
        sz.decode(blob, 300, workspace=torch.empty(0, dtype=torch.uint8))
