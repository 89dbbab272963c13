"""The one-GPU compressed transfer: chunked encode, device-to-host and
host-to-device copies through pinned memory on their own streams, decode.
The decoded cache must equal the source bit for bit, the containers that
crossed must be the oracle's, and the raw path must move the same cache."""
import numpy as np
import pytest

import kvgen
import oracle

torch = pytest.importorskip("torch")
import lossless_bf16_kv_splitzip_b200 as sz  # noqa: E402
from lossless_bf16_kv_splitzip_b200.transfer import SplitZipChunks, host_transfer  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

DEV = torch.device("cuda", 0)


@pytest.mark.parametrize("per_chunk", [1, 3])
def test_host_transfer_round_trip(per_chunk):
    host = kvgen.contiguous_cache(1, layers=4, tokens=512)  # 8 tensors of 524,288 values
    S, n = host.shape
    src = torch.from_numpy(host.view(np.int16)).to(DEV)
    out = torch.zeros_like(src)
    staging = torch.empty(2 * S * n + 4096 * S, dtype=torch.uint8, pin_memory=True)
    codec = SplitZipChunks(src, out, per_chunk, DEV)
    res = host_transfer(codec, src, out, per_chunk, staging)
    torch.cuda.synchronize()
    assert codec.statuses_ok()
    assert torch.equal(out, src)
    assert res.chunks == -(-S // per_chunk) and 0 < res.link_bytes < 2 * S * n
    # what crossed the link is the oracle's containers, end to end per chunk
    blob = b"".join(staging[p: p + nb].numpy().tobytes() for p, nb in res.placed)
    ref = b"".join(oracle.encode(host[k]) for k in range(S))
    assert blob == ref and res.link_bytes == len(ref)
    raw_out = torch.zeros_like(src)
    res_raw = host_transfer(None, src, raw_out, per_chunk, staging)
    torch.cuda.synchronize()
    assert torch.equal(raw_out, src) and res_raw.link_bytes == 2 * S * n


def test_host_round_trip_pipelined():
    host = kvgen.contiguous_cache(1, layers=3, tokens=1024)  # 6 tensors
    S, n = host.shape
    h_in = torch.from_numpy(host.view(np.int16)).pin_memory()
    h_out = torch.zeros_like(h_in).pin_memory()
    d_in = torch.zeros((S, n), dtype=torch.int16, device=DEV)
    d_out = torch.zeros_like(d_in)
    codec = SplitZipChunks(d_in, d_out, 2, DEV)
    staging = torch.empty(2 * S * n + 4096 * S, dtype=torch.uint8, pin_memory=True)
    from lossless_bf16_kv_splitzip_b200.transfer import host_round_trip
    t, n_up, n_down = host_round_trip(codec, h_in, h_out, staging)
    torch.cuda.synchronize()
    assert codec.statuses_ok()
    assert torch.equal(h_out, h_in)
    comp = sum(len(oracle.encode(host[k])) for k in range(S))
    assert n_up == 2 * S * n + comp and n_down == comp + 2 * S * n and t > 0
