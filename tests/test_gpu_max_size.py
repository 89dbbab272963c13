"""The largest stream the format allows: n = 2^32 - 1 BF16 values (8 GiB,
odd length), through the single-stream C ABI.  The oracle cannot encode
8 GiB in test time, so what is checked holds at any size: the header, the
codebook (the oracle's top-16 select applied to an exponent histogram that
numpy computes on the host), e = n - (sum of the top-16 counts), the
container size formula, escapes planted at known positions above 2^31 up to
the last element (u32 positions at their limit), sampled sign+mantissa bytes
and code nibbles recomputed on the host, and the bit-exact round trip."""
import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")
import lossless_bf16_kv_splitzip_b200 as sz  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

DEV = "cuda:0"
N = (1 << 32) - 1


def test_max_size_stream():
    g = torch.Generator(device=DEV)
    g.manual_seed(0x5EED0005)
    x = torch.randn(N, generator=g, device=DEV, dtype=torch.float32).to(torch.bfloat16)
    planted = [(1 << 31) + 5, (1 << 32) - 17, N - 2, N - 1]
    vals = [3.0e25, -7.5e-30, 1.0e30, -2.0e-28]  # exponents far outside N(0,1)'s
    for p, v in zip(planted, vals):
        x[p] = v
    xi = x.view(torch.int16)
    out, size, status = sz.encode(xi)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    nbytes = int(size.item())

    host = xi.cpu().numpy().view(np.uint16)
    exps = ((host >> 7) & 0xFF).astype(np.uint8)
    hist = np.bincount(exps, minlength=256).astype(np.uint64)
    cb = oracle.select_top16(hist)
    e = N - int(hist[cb.astype(np.int64)].sum())
    assert nbytes == 48 + N + (N + 1) // 2 + 5 * e

    head = out[:48].cpu().numpy()
    assert bytes(head[:8]) == b"SZKV\x01\x01\x00\x00"
    assert int(head[8:16].view(np.uint64)[0]) == N
    assert int(head[16:24].view(np.uint64)[0]) == e
    assert np.array_equal(head[24:40], cb)

    lut = np.full(256, 0xFF, np.uint8)
    lut[cb] = np.arange(16, dtype=np.uint8)
    rng = np.random.default_rng(7)
    sample = np.concatenate([rng.integers(0, N, 4096), np.array(planted), np.array([0, 1, N - 3])]).astype(np.int64)
    sm = (((host[sample] >> 8) & 0x80) | (host[sample] & 0x7F)).astype(np.uint8)
    got_sm = out[48 + torch.from_numpy(sample).to(DEV)].cpu().numpy()
    assert np.array_equal(got_sm, sm)
    code_bytes = out[48 + N + torch.from_numpy(sample // 2).to(DEV)].cpu().numpy()
    nib = np.where(sample % 2 == 0, code_bytes & 0xF, code_bytes >> 4)
    want = np.where(lut[exps[sample]] == 0xFF, 0, lut[exps[sample]])  # escapes hold the placeholder 0
    assert np.array_equal(nib, want)

    # the escape records: the last ones equal the escapes the host finds in
    # the stream's last 65,536 values (planted ones included, positions up to
    # N - 1), and the one planted above 2^31 is where it belongs
    pos_off = 48 + N + (N + 1) // 2
    t0 = N - 65536
    tail_pos = t0 + np.flatnonzero(lut[exps[t0:]] == 0xFF)
    k = tail_pos.size
    assert k >= 3 and tail_pos[-1] == N - 1
    pos = out[pos_off: pos_off + 4 * e].cpu().numpy().view(np.uint32)
    raw = out[pos_off + 4 * e: pos_off + 5 * e].cpu().numpy()
    assert np.array_equal(pos[-k:].astype(np.int64), tail_pos)
    assert np.array_equal(raw[-k:], exps[tail_pos])
    assert np.all(pos[1:] > pos[:-1])
    i = int(np.searchsorted(pos, planted[0]))
    assert pos[i] == planted[0] and raw[i] == exps[planted[0]]
    del host, exps, pos, raw

    y, dst = sz.decode(out[:nbytes], N)
    torch.cuda.synchronize()
    assert int(dst.item()) == 0
    assert torch.equal(y, xi)
