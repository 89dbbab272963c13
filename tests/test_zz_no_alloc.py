"""sz_encode_static -- compression with no workspace and no allocation.

For callers that cannot allocate device memory when they compress (code
inside an allocator or memory-pool callback, or an engine that reserved all
device memory up front), the library keeps the scratch of one tensor's
compression in its own device array.  This checks, through the C ABI, that
calls in a row give byte for byte the oracle's container and that of the
regular sz_histogram_codebook + sz_encode path: a later call must not see an
earlier call's leftovers in the shared array.  Sizes cover the empty
stream, ragged multi-tile streams, streams whose CTA ranges hold several
tiles, and the largest stream the array allows.
"""
import numpy as np
import pytest

import kvgen
import oracle

torch = pytest.importorskip("torch")
import lossless_bf16_kv_splitzip_b200 as sz  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

DEV = "cuda:0"
MAX_ELEMS = 1 << 28


def regular_path(x):
    d = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(DEV)
    out, size, status = sz.encode(d)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out[: int(size.item())].cpu().numpy().tobytes()


def static_path(x):
    d = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(DEV)
    n = x.size
    cap = sz.max_bytes(n)
    out = torch.empty(max(cap, 16), dtype=torch.uint8, device=DEV)
    size = torch.zeros(1, dtype=torch.int64, device=DEV)
    status = torch.full((1,), -99, dtype=torch.int32, device=DEV)
    cb = torch.zeros(16, dtype=torch.uint8, device=DEV)
    sz.sz_encode_static(d if n else out, n, out, cap, size, cb, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    blob = out[: int(size.item())].cpu().numpy().tobytes()
    assert bytes(cb.cpu().numpy()) == blob[24:40]
    return blob


def test_static_scratch_path_matches_oracle_and_regular_path_twice():
    # several tiles with a ragged tail, then a smaller K-like tensor: the
    # second call reuses the array the first one filled
    a = kvgen.mixed_small(3 * 65536 + 123, seed=4242)
    b = kvgen.contiguous_tensor(1, 0, 0, tokens=300)
    first = static_path(a)
    second = static_path(b)
    assert first == oracle.encode(a)
    assert second == oracle.encode(b)
    assert first == regular_path(a)
    assert second == regular_path(b)


def test_static_scratch_path_empty_stream():
    x = np.zeros(0, np.uint16)
    assert static_path(x) == oracle.encode(x)


def test_static_scratch_path_ranges_of_several_tiles():
    # 458 tiles: CTA ranges of two tiles each, the last one short
    x = kvgen.mixed_small(30_000_000, seed=4243)
    got = static_path(x)
    assert got == oracle.encode(x)
    assert got == regular_path(x)


def test_static_scratch_path_largest_stream():
    # the whole 4K-token Llama-3-8B cache as one stream: 2^28 elements, the
    # array's limit (4096 tiles in ranges of ten)
    x = kvgen.contiguous_cache(1).reshape(-1)
    assert x.size == MAX_ELEMS
    got = static_path(x)
    assert got == oracle.encode(x)
    assert got == regular_path(x)


def test_static_scratch_path_size_limit():
    d = torch.zeros(16, dtype=torch.int16, device=DEV)
    out = torch.zeros(16, dtype=torch.uint8, device=DEV)
    size = torch.zeros(1, dtype=torch.int64, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(sz.SzError) as e:
        sz.sz_encode_static(d, MAX_ELEMS + 1, out, 1 << 40, size, None, status)
    assert e.value.status == sz.SZ_ERR_TOO_LARGE


def test_static_scratch_path_honours_the_wait_limit():
    """The copy thread issues no bulk copy: the static path's stage waits
    run out after the process-wide limit like every other entry point's,
    the call reports SZ_ERR_DEVICE_TIMEOUT with size 0, and the next normal
    call is bit-exact."""
    x = kvgen.mixed_small(9 * 65536 + 5, seed=4244)
    d = torch.from_numpy(x.view(np.int16)).to(DEV)
    cap = sz.max_bytes(x.size)
    out = torch.empty(cap, dtype=torch.uint8, device=DEV)
    size = torch.ones(1, dtype=torch.int64, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    try:
        sz.sz_set_wait_limit_ns(2_000_000)
        sz.sz_debug_set_flags(1)
        sz.sz_encode_static(d, x.size, out, cap, size, None, status)
        torch.cuda.synchronize()
        assert int(status.item()) == sz.SZ_ERR_DEVICE_TIMEOUT and int(size.item()) == 0
    finally:
        sz.sz_debug_set_flags(0)
        sz.sz_set_wait_limit_ns(1_000_000_000)
    assert static_path(x) == oracle.encode(x)
