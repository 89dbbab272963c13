"""sz_encode_static -- compression with no workspace and no allocation.

For callers that cannot allocate device memory when they compress (code
inside an allocator or memory-pool callback, or an engine that reserved all
device memory up front), the library keeps the scratch of one tensor's
compression in its own device array.  This checks, through the C ABI, that
two calls in a row give byte for byte the container of the regular
sz_histogram_codebook + sz_encode path: the second call must not see the
first call's leftovers in the shared array.
"""
import numpy as np
import pytest

import kvgen

torch = pytest.importorskip("torch")
import lossless_bf16_kv_splitzip_b200 as sz  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

DEV = "cuda:0"


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
    out = torch.empty(cap, dtype=torch.uint8, device=DEV)
    size = torch.zeros(1, dtype=torch.int64, device=DEV)
    status = torch.full((1,), -99, dtype=torch.int32, device=DEV)
    cb = torch.zeros(16, dtype=torch.uint8, device=DEV)
    sz.sz_encode_static(d, n, out, cap, size, cb, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    blob = out[: int(size.item())].cpu().numpy().tobytes()
    assert bytes(cb.cpu().numpy()) == blob[24:40]
    return blob


def test_static_scratch_path_matches_regular_path_twice():
    # several tiles with a ragged tail, then a smaller K-like tensor: the
    # second call reuses the array the first one filled
    a = kvgen.mixed_small(3 * 65536 + 123, seed=4242)
    b = kvgen.contiguous_tensor(1, 0, 0, tokens=300)
    first = static_path(a)
    second = static_path(b)
    assert first == regular_path(a)
    assert second == regular_path(b)


def test_static_scratch_path_size_limit():
    d = torch.zeros(16, dtype=torch.int16, device=DEV)
    out = torch.zeros(16, dtype=torch.uint8, device=DEV)
    size = torch.zeros(1, dtype=torch.int64, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(sz.SzError) as e:
        sz.sz_encode_static(d, (1 << 28) + 1, out, 1 << 40, size, None, status)
    assert e.value.status == sz.SZ_ERR_TOO_LARGE
