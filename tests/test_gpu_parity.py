"""GPU parity: the CUDA library against the CPU oracle, through the C ABI.

Integer/byte work, so the bar is bit-exactness: every byte of every
container and every bit of every decoded value must equal the oracle's on
the same seeded inputs.  Covered: ragged sizes around the tile (65536),
sub-tile (16384) and chunk (16) boundaries, single streams at the sizes of
the bench's latency sweep, the exhaustive 65,536-pattern tensor, the golden
containers, every workload at full size in the batched launch the bench
times, scattered paged KV, incompressible input, a caller-chosen codebook,
cross decoding, determinism, corrupt containers and the bounded-wait
timeout path."""
import struct

import numpy as np
import pytest

import kvgen
import oracle
from conftest import load_golden
from oracle_pool import oracle_digests

torch = pytest.importorskip("torch")
import lossless_bf16_kv_splitzip_b200 as sz  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

H = 48
DEV = "cuda:0"
SHORT_ENC = 1 << 20  # sz_compress: streams up to this many elements take the short-stream encode
SHORT_DEC = 1 << 17  # sz_decode: streams up to this many elements take the short-stream decode
SHORT = 1 << 21  # past both limits


def to_dev(x_np):
    return torch.from_numpy(np.ascontiguousarray(x_np).view(np.int16)).to(DEV)


def gpu_encode(x_np):
    out, size, status = sz.encode(to_dev(x_np))
    torch.cuda.synchronize()
    assert int(status.item()) == 0, sz.STATUS.get(int(status.item()))
    return out[: int(size.item())].cpu().numpy().tobytes()


def gpu_decode(blob, n):
    c = torch.from_numpy(np.frombuffer(blob, np.uint8).copy()).to(DEV) if len(blob) else \
        torch.zeros(16, dtype=torch.uint8, device=DEV)
    nbytes = len(blob)
    _, wsb = sz.sz_plan(n)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    out = torch.zeros(max(n, 1), dtype=torch.int16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    sz.sz_decode(c, nbytes, out, n, status, ws, wsb)
    torch.cuda.synchronize()
    return int(status.item()), out[:n].cpu().numpy().view(np.uint16)


def assert_parity(x):
    ref = oracle.encode(x)
    got = gpu_encode(x)
    assert len(got) == len(ref)
    if got != ref:
        a = np.frombuffer(got, np.uint8)
        b = np.frombuffer(ref, np.uint8)
        i = int(np.flatnonzero(a != b)[0])
        raise AssertionError("first differing byte %d of %d: gpu %02x oracle %02x" % (i, len(ref), a[i], b[i]))
    st, y = gpu_decode(got, x.size)
    assert st == 0
    assert np.array_equal(y, x)
    return ref


# -------------------------------------------------------------- small cases
RAGGED = [0, 1, 2, 3, 7, 8, 15, 16, 17, 31, 33, 100, 255, 4095, 4096, 4097, 8191, 16383, 16384, 16385,
          16400, 32768, 3 * 16384 + 5, 65535, 65536, 65537, 65536 + 16384 + 8, 100003, 3 * 65536 + 100,
          262147]


@pytest.mark.parametrize("n", RAGGED)
def test_ragged_sizes_bit_exact(n):
    assert_parity(kvgen.mixed_small(n, seed=5000 + n))


# ragged streams longer than the short-stream limit: the pipelined paths
@pytest.mark.parametrize("n", [SHORT + 1, SHORT + 16383, SHORT + 65537 + 7])
def test_ragged_large_sizes_bit_exact(n):
    assert_parity(kvgen.mixed_small(n, seed=n % 1000))


@pytest.mark.parametrize("n", [1, 16, 17, 16384, 16385, 70001])
def test_incompressible_bit_exact(n):
    x = kvgen.uniform_u16(n, seed=n)
    blob = assert_parity(x)
    assert len(blob) <= sz.max_bytes(n)


def test_exhaustive_patterns_bit_exact():
    x = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    blob = assert_parity(x)
    assert len(blob) == 405552


def test_each_pattern_alone():
    for v in list(range(0, 65536, 4099)) + [0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0xFFC1, 0x0001, 0x8001]:
        assert_parity(np.array([v], np.uint16))


def test_goldens_gpu(golden_names):
    for name in golden_names:
        n, inp, cont = load_golden(name)
        x = np.array(inp, np.uint16)
        assert gpu_encode(x) == cont, name
        st, y = gpu_decode(cont, n)
        assert st == 0 and np.array_equal(y, x), name


def test_workload0_tiny_k_tensor():
    x = kvgen.tiny_k_tensor()
    blob = assert_parity(x)
    e = struct.unpack_from("<Q", blob, 16)[0]
    assert e >= 1049 // 2


def test_single_exponent_and_seventeen_equal():
    rng = np.random.default_rng(3)
    x = (np.uint16(131 << 7) | (rng.integers(0, 1 << 16, 50000).astype(np.uint16) & np.uint16(0x807F)))
    assert_parity(x)
    x = ((np.repeat(np.arange(100, 117), 2000).astype(np.uint16) << 7) | np.uint16(3))
    assert_parity(np.random.default_rng(4).permutation(x))


_SWEEP_SRC = {}


def sweep_prefix(nbytes):
    """The first nbytes of the 32K-token workload's buffer, as the bench's
    latency sweep codes them: one stream, one codebook."""
    n = nbytes // 2
    nt = kvgen.HEADS * 32768 * kvgen.HEAD_DIM
    parts = []
    for k in range(-(-n // nt)):
        if k not in _SWEEP_SRC:
            _SWEEP_SRC[k] = kvgen.contiguous_tensor(2, k // 2, k % 2)
        parts.append(_SWEEP_SRC[k])
    return np.concatenate(parts)[:n] if len(parts) > 1 else parts[0][:n]


@pytest.mark.parametrize("nbytes", [1 << 16, 1 << 18, 1 << 20, 1 << 22, 1 << 24, 1 << 26])
def test_sweep_prefix_single_stream(nbytes):
    assert_parity(sweep_prefix(nbytes))


@pytest.mark.slow
def test_sweep_prefix_spanning_tensors():
    # 256 MiB: layer 0-1 K and V as one stream under one codebook
    assert_parity(sweep_prefix(1 << 28))


def test_cross_decode():
    x = kvgen.mixed_small(123457, seed=77)
    ref = oracle.encode(x)
    st, y = gpu_decode(ref, x.size)  # GPU decodes the oracle's container
    assert st == 0 and np.array_equal(y, x)
    got = gpu_encode(x)
    assert np.array_equal(oracle.decode(got, x.size), x)  # oracle decodes the GPU's


def test_deterministic_over_runs():
    x = kvgen.contiguous_tensor(3, 0, 0, tokens=512)  # heavy tails, many escapes
    blobs = {gpu_encode(x) for _ in range(3)}
    assert len(blobs) == 1


def test_given_codebook_path():
    x = kvgen.mixed_small(200003, seed=8)
    d = to_dev(x)
    n = x.size
    cap, wsb = sz.sz_plan(n)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    cb_auto = torch.empty(16, dtype=torch.uint8, device=DEV)
    hist = torch.zeros(256, dtype=torch.int32, device=DEV)
    sz.sz_histogram_codebook(d, n, cb_auto, hist, ws, wsb)
    torch.cuda.synchronize()
    assert np.array_equal(hist.cpu().numpy().view(np.uint32).astype(np.uint64), oracle.histogram(x))
    assert np.array_equal(cb_auto.cpu().numpy(), oracle.select_top16(oracle.histogram(x)))
    cb = np.arange(118, 134, dtype=np.uint8)
    out = torch.empty(oracle.container_size(n, n), dtype=torch.uint8, device=DEV)
    size = torch.zeros(1, dtype=torch.int64, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    sz.sz_encode(d, n, torch.from_numpy(cb).to(DEV), out, out.numel(), size, st, ws, wsb)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = out[: int(size.item())].cpu().numpy().tobytes()
    assert got == oracle.encode(x, codebook=cb)


def test_repeated_codebook_is_rejected():
    x = kvgen.mixed_small(5000, seed=9)
    d = to_dev(x)
    cap, wsb = sz.sz_plan(x.size)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    cb = torch.empty(16, dtype=torch.uint8, device=DEV)
    sz.sz_histogram_codebook(d, x.size, cb, None, ws, wsb)
    bad = torch.full((16,), 120, dtype=torch.uint8, device=DEV)
    out = torch.empty(cap, dtype=torch.uint8, device=DEV)
    size = torch.ones(1, dtype=torch.int64, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    sz.sz_encode(d, x.size, bad, out, cap, size, st, ws, wsb)
    torch.cuda.synchronize()
    assert int(st.item()) == sz.SZ_ERR_INVALID and int(size.item()) == 0


def test_capacity_checked_on_device():
    # a caller codebook that matches nothing needs 48 + 6.5n bytes; give less
    x = kvgen.mixed_small(4000, seed=10)
    d = to_dev(x)
    cap, wsb = sz.sz_plan(x.size)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    cb = torch.empty(16, dtype=torch.uint8, device=DEV)
    sz.sz_histogram_codebook(d, x.size, cb, None, ws, wsb)
    far = torch.arange(200, 216, dtype=torch.uint8, device=DEV)
    small = H + x.size + (x.size + 1) // 2 + 100
    out = torch.empty(small, dtype=torch.uint8, device=DEV)
    size = torch.ones(1, dtype=torch.int64, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    sz.sz_encode(d, x.size, far, out, small, size, st, ws, wsb)
    torch.cuda.synchronize()
    assert int(st.item()) == sz.SZ_ERR_CAPACITY and int(size.item()) == 0


def test_stale_workspace_histogram_is_reported():
    # encode input B with the histogram of input A: the escape count differs
    a = kvgen.mixed_small(40000, seed=11)
    b = kvgen.uniform_u16(40000, seed=12)
    cap, wsb = sz.sz_plan(a.size)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    cb = torch.empty(16, dtype=torch.uint8, device=DEV)
    sz.sz_histogram_codebook(to_dev(a), a.size, cb, None, ws, wsb)
    out = torch.empty(cap, dtype=torch.uint8, device=DEV)
    size = torch.ones(1, dtype=torch.int64, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    sz.sz_encode(to_dev(b), b.size, cb, out, cap, size, st, ws, wsb)
    torch.cuda.synchronize()
    assert int(st.item()) == sz.SZ_ERR_CORRUPT and int(size.item()) == 0


@pytest.mark.parametrize("tile", [0, 4, 8])
def test_stale_workspace_on_several_ranges_keeps_size_zero(tile):
    """A stream of 8 x 65,536 + 5 elements is encoded by several CTAs, each
    a range of tiles.  Its input changes after the histogram in one 65,536-
    element stretch only, so the CTAs there find more escapes than the
    workspace counted: the status is SZ_ERR_CORRUPT and the size stays 0,
    whichever CTA finishes the stream last."""
    n = 8 * 65536 + 5
    a = kvgen.mixed_small(n, seed=13)
    cap, wsb = sz.sz_plan(n)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    cb = torch.empty(16, dtype=torch.uint8, device=DEV)
    sz.sz_histogram_codebook(to_dev(a), n, cb, None, ws, wsb)
    torch.cuda.synchronize()
    code = cb.cpu().numpy()
    outside = next(e for e in range(1, 255) if e not in set(code.tolist()))
    b = a.copy()
    lo = tile * 65536
    idx = np.arange(lo, min(lo + 65536, n), 97)
    b[idx] = (b[idx] & 0x807F) | (outside << 7)  # escapes the histogram never saw
    out = torch.empty(cap, dtype=torch.uint8, device=DEV)
    size = torch.ones(1, dtype=torch.int64, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    sz.sz_encode(to_dev(b), n, cb, out, cap, size, st, ws, wsb)
    torch.cuda.synchronize()
    assert int(st.item()) == sz.SZ_ERR_CORRUPT and int(size.item()) == 0
    # the same workspace still encodes the input it describes
    sz.sz_encode(to_dev(a), n, cb, out, cap, size, st, ws, wsb)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert out[: int(size.item())].cpu().numpy().tobytes() == oracle.encode(a)


# ------------------------------------------------------ corrupt containers
def corruptions(blob, n):
    b = bytearray(blob)
    e = struct.unpack_from("<Q", b, 16)[0]
    off_pos = H + n + (n + 1) // 2
    out = {}

    def mut(name, f):
        c = bytearray(b)
        f(c)
        out[name] = bytes(c)

    mut("magic", lambda c: c.__setitem__(0, ord("X")))
    mut("version", lambda c: c.__setitem__(4, 2))
    mut("dtype", lambda c: c.__setitem__(5, 2))
    mut("flags", lambda c: c.__setitem__(6, 1))
    mut("reserved", lambda c: c.__setitem__(44, 1))
    mut("n", lambda c: struct.pack_into("<Q", c, 8, n + 1))
    mut("escapes_past_end", lambda c: struct.pack_into("<Q", c, 16, e + 1000))
    mut("dup_codebook", lambda c: c.__setitem__(25, c[24]))
    mut("unsorted", lambda c: struct.pack_into("<I", c, off_pos + 4, 0))
    mut("pos_range", lambda c: struct.pack_into("<I", c, off_pos, n + 5))
    mut("pos_last_range", lambda c: struct.pack_into("<I", c, off_pos + 4 * (e - 1), n + 5))
    mut("pos_dup", lambda c: struct.pack_into("<I", c, off_pos + 4, struct.unpack_from("<I", c, off_pos)[0]))
    mut("raw_in_codebook", lambda c: c.__setitem__(off_pos + 4 * e, c[24]))
    p = struct.unpack_from("<I", b, off_pos)[0]
    mut("placeholder", lambda c: c.__setitem__(H + n + p // 2, c[H + n + p // 2] | ((1 << 4) if p % 2 else 1)))
    out["truncated"] = bytes(b[:-1])
    return out


# short streams take the one-launch decode, longer ones the index +
# pipelined decode: both must reject every corruption
@pytest.mark.parametrize("n", [3001, 40000, 3 * 16384 + 11, 65536 + 3001, SHORT_DEC, SHORT_DEC + 3001,
                               SHORT + 3001, SHORT + 16 * 17])
def test_corrupt_containers_rejected(n):
    x = kvgen.mixed_small(n, seed=21 + n)
    blob = gpu_encode(x)
    assert struct.unpack_from("<Q", blob, 16)[0] >= 2
    for name, c in corruptions(blob, n).items():
        st_o, _ = oracle.decode_status(c, n)
        st_g, _ = gpu_decode(c, n)
        assert st_o == oracle.ERR_CORRUPT, name
        assert st_g == sz.SZ_ERR_CORRUPT, name


def test_odd_tail_nibble_rejected():
    x = np.array([0x3F80, 0x3F80, 0x3F80], np.uint16)
    c = bytearray(gpu_encode(x))
    c[H + 3 + 1] |= 0x10
    assert gpu_decode(bytes(c), 3)[0] == sz.SZ_ERR_CORRUPT
    n = SHORT + 1001  # the pipelined decode's path
    x = kvgen.mixed_small(n, seed=23)
    c = bytearray(gpu_encode(x))
    c[H + n + (n + 1) // 2 - 1] |= 0x10  # high nibble of the last code byte
    assert gpu_decode(bytes(c), n)[0] == sz.SZ_ERR_CORRUPT


# -------------------------------------------------- one-call compression
@pytest.mark.parametrize("n", [0, 1, 17, 4095, 4096, 4097, 32769, 65537, 3 * 65536 + 100, SHORT_ENC,
                               SHORT_ENC + 1, SHORT, SHORT + 1,
                               (1 << 23) + 7, (1 << 25) + 12345, (1 << 26) + 33, (1 << 27) - 5, (1 << 27) + 16])
def test_compress_one_call_equals_oracle(n):
    """sz_compress: short streams by 4,096-element blocks in two launches,
    longer ones by the histogram and encode kernels (16,384-element tiles
    below 2^27 elements, 65,536 from there); the same bytes as the oracle
    (and as the two-call path), and the codebook it reports is the
    header's."""
    x = kvgen.mixed_small(n, seed=300 + n % 101)
    cb = torch.zeros(16, dtype=torch.uint8, device=DEV)
    out, size, status = sz.compress(to_dev(x), codebook=cb)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = out[: int(size.item())].cpu().numpy().tobytes()
    assert got == oracle.encode(x)
    assert bytes(cb.cpu().numpy()) == got[24:40]


@pytest.mark.parametrize("n", [30000, SHORT + 70000])  # the short-stream path and the kernels' path
def test_compress_capacity_checked_on_device(n):
    x = kvgen.uniform_u16(n, seed=301)  # incompressible: many escapes
    d = to_dev(x)
    cap, wsb = sz.sz_plan(x.size)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    small = H + x.size + (x.size + 1) // 2 + 64
    out = torch.empty(small, dtype=torch.uint8, device=DEV)
    size = torch.ones(1, dtype=torch.int64, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    sz.sz_compress(d, x.size, out, small, size, None, st, ws, wsb)
    torch.cuda.synchronize()
    assert int(st.item()) == sz.SZ_ERR_CAPACITY and int(size.item()) == 0


# -------------------------------------------------------- bounded waits
def test_stage_wait_times_out_cleanly():
    """The copy thread issues no bulk copy, so every stage wait runs out:
    the kernel reports SZ_ERR_DEVICE_TIMEOUT and returns; the context stays
    usable and the next normal call is bit-exact."""
    x = kvgen.mixed_small(4 * 16384, seed=31)
    try:
        sz.sz_set_wait_limit_ns(2_000_000)  # 2 ms
        sz.sz_debug_set_flags(1)
        out, size, status = sz.encode(to_dev(x))
        torch.cuda.synchronize()
        assert int(status.item()) == sz.SZ_ERR_DEVICE_TIMEOUT
        assert int(size.item()) == 0
    finally:
        sz.sz_debug_set_flags(0)
        sz.sz_set_wait_limit_ns(1_000_000_000)
    assert gpu_encode(x) == oracle.encode(x)


def test_stage_wait_timeout_on_several_ranges_and_one_pass():
    """Every stage wait runs out on a stream of several CTA ranges (two-pass
    and one-pass encode) and on a batch of several segments (encode and
    decode): every status is SZ_ERR_DEVICE_TIMEOUT and every size 0."""
    n = 8 * 65536 + 5
    x = kvgen.mixed_small(n, seed=33)
    lens = [3 * 65536 + 7, 16384, 5 * 65536]
    streams = [kvgen.mixed_small(m, seed=34 + i) for i, m in enumerate(lens)]
    starts = [0]
    for m in lens[:-1]:
        starts.append(starts[-1] + -(-m // 64) * 64)  # 16-byte aligned pages
    flat = np.zeros(starts[-1] + lens[-1], np.uint16)
    for s_, x_ in zip(starts, streams):
        flat[s_: s_ + x_.size] = x_
    pool = torch.from_numpy(flat.view(np.int16)).to(DEV)
    plan = sz.BatchPlan(lens, max(lens), device=DEV)
    ptrs = torch.from_numpy((np.array(starts) * 2 + pool.data_ptr()).astype(np.int64)).to(DEV)
    try:
        sz.sz_set_wait_limit_ns(2_000_000)
        sz.sz_debug_set_flags(1)
        out, size, status = sz.encode(to_dev(x))
        out1, size1, status1 = sz.encode_one_pass(to_dev(x), torch.arange(120, 136, dtype=torch.uint8, device=DEV))
        plan.encode(ptrs)
        torch.cuda.synchronize()
        assert int(status.item()) == sz.SZ_ERR_DEVICE_TIMEOUT and int(size.item()) == 0
        assert int(status1.item()) == sz.SZ_ERR_DEVICE_TIMEOUT and int(size1.item()) == 0
        assert plan.enc_status.cpu().tolist() == [sz.SZ_ERR_DEVICE_TIMEOUT] * 3
        assert plan.sizes.cpu().tolist() == [0, 0, 0]
    finally:
        sz.sz_debug_set_flags(0)
        sz.sz_set_wait_limit_ns(1_000_000_000)
    assert gpu_encode(x) == oracle.encode(x)
    plan.encode(ptrs)
    torch.cuda.synchronize()
    assert plan.enc_status.abs().sum().item() == 0
    dst = torch.zeros_like(pool)
    dptrs = torch.from_numpy((np.array(starts) * 2 + dst.data_ptr()).astype(np.int64)).to(DEV)
    try:
        sz.sz_set_wait_limit_ns(2_000_000)
        sz.sz_debug_set_flags(1)
        plan.decode(dptrs)
        torch.cuda.synchronize()
        assert plan.dec_status.cpu().tolist() == [sz.SZ_ERR_DEVICE_TIMEOUT] * 3
    finally:
        sz.sz_debug_set_flags(0)
        sz.sz_set_wait_limit_ns(1_000_000_000)
    plan.decode(dptrs)
    torch.cuda.synchronize()
    assert plan.dec_status.abs().sum().item() == 0
    assert torch.equal(dst, pool)
    for k, s_ in enumerate(streams):
        off, z = int(plan.out_offset[k]), int(plan.sizes[k].item())
        assert plan.container[off: off + z].cpu().numpy().tobytes() == oracle.encode(s_)


@pytest.mark.parametrize("n", [SHORT + 5, (1 << 24) + 3])
def test_compress_wait_times_out_cleanly(n):
    """sz_compress of a stream past the short-stream limit: every stage wait
    of its encode kernel runs out; status SZ_ERR_DEVICE_TIMEOUT, size 0, and
    the next call is bit-exact."""
    x = kvgen.mixed_small(n, seed=36)
    try:
        sz.sz_set_wait_limit_ns(2_000_000)
        sz.sz_debug_set_flags(1)
        out, size, status = sz.compress(to_dev(x))
        torch.cuda.synchronize()
        assert int(status.item()) == sz.SZ_ERR_DEVICE_TIMEOUT and int(size.item()) == 0
    finally:
        sz.sz_debug_set_flags(0)
        sz.sz_set_wait_limit_ns(1_000_000_000)
    out, size, status = sz.compress(to_dev(x))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert out[: int(size.item())].cpu().numpy().tobytes() == oracle.encode(x)


def test_decode_escape_wait_times_out_cleanly():
    """The decode's values are stored before the index is ready; a wait for
    a stage's escape part that runs out (bit 1: only values parts are ever
    published) gives SZ_ERR_DEVICE_TIMEOUT for the stream and for every
    segment of a batch, and the next call is bit-exact."""
    x = kvgen.mixed_small(SHORT + 5, seed=33)
    blob = oracle.encode(x)
    c = torch.from_numpy(np.frombuffer(blob, np.uint8).copy()).to(DEV)
    lens = [300000, 5 * 65536 + 11, 65536]
    streams = [kvgen.mixed_small(m, seed=40 + i) for i, m in enumerate(lens)]
    starts = [0]
    for m in lens[:-1]:
        starts.append(starts[-1] + -(-m // 64) * 64)  # 16-byte aligned pages
    flat = np.zeros(starts[-1] + lens[-1], np.uint16)
    for s_, x_ in zip(starts, streams):
        flat[s_: s_ + x_.size] = x_
    pool = torch.from_numpy(flat.view(np.int16)).to(DEV)
    plan = sz.BatchPlan(lens, max(lens), device=DEV)
    ptrs = torch.from_numpy((np.array(starts) * 2 + pool.data_ptr()).astype(np.int64)).to(DEV)
    plan.encode(ptrs)
    torch.cuda.synchronize()
    assert plan.enc_status.abs().sum().item() == 0
    dst = torch.zeros_like(pool)
    dptrs = torch.from_numpy((np.array(starts) * 2 + dst.data_ptr()).astype(np.int64)).to(DEV)
    try:
        sz.sz_set_wait_limit_ns(2_000_000)
        sz.sz_debug_set_flags(2)
        _, status = sz.decode(c, x.size)
        plan.decode(dptrs)
        torch.cuda.synchronize()
        assert int(status.item()) == sz.SZ_ERR_DEVICE_TIMEOUT
        assert all(int(v) == sz.SZ_ERR_DEVICE_TIMEOUT for v in plan.dec_status.cpu().tolist())
    finally:
        sz.sz_debug_set_flags(0)
        sz.sz_set_wait_limit_ns(1_000_000_000)
    y, status = sz.decode(c, x.size)
    plan.decode(dptrs)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(y.cpu().numpy().view(np.uint16), x)
    assert plan.dec_status.abs().sum().item() == 0
    assert torch.equal(dst, pool)


def test_decode_stage_wait_times_out_cleanly():
    x = kvgen.mixed_small(SHORT + 5, seed=32)  # the pipelined decode (it has the waits)
    blob = oracle.encode(x)
    c = torch.from_numpy(np.frombuffer(blob, np.uint8).copy()).to(DEV)
    try:
        sz.sz_set_wait_limit_ns(2_000_000)
        sz.sz_debug_set_flags(1)
        _, status = sz.decode(c, x.size)
        torch.cuda.synchronize()
        assert int(status.item()) == sz.SZ_ERR_DEVICE_TIMEOUT
    finally:
        sz.sz_debug_set_flags(0)
        sz.sz_set_wait_limit_ns(1_000_000_000)
    out, status = sz.decode(c, x.size)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(out.cpu().numpy().view(np.uint16), x)


# ----------------------------------------------------- batched / paged
def batched_contiguous(cache):
    """Encode + decode a [S, n] cache with one batched call each, the launch
    the bench times.  Returns (plan, decoded device tensor)."""
    S, n = cache.shape
    d_in = torch.from_numpy(cache.view(np.int16)).to(DEV)
    plan = sz.BatchPlan([n] * S, n, device=DEV)
    ptrs = torch.tensor([d_in.data_ptr() + 2 * n * k for k in range(S)], dtype=torch.int64, device=DEV)
    plan.encode(ptrs)
    d_out = torch.empty_like(d_in)
    optrs = torch.tensor([d_out.data_ptr() + 2 * n * k for k in range(S)], dtype=torch.int64, device=DEV)
    plan.decode(optrs)
    torch.cuda.synchronize()
    assert plan.enc_status.abs().sum().item() == 0
    assert plan.dec_status.abs().sum().item() == 0
    assert torch.equal(d_out, d_in)
    return plan


def check_batch_against_oracle(plan, streams):
    sizes = plan.sizes.cpu().numpy()
    host = plan.container.cpu().numpy()
    for k, x in enumerate(streams):
        off = int(plan.out_offset[k])
        got = host[off: off + int(sizes[k])].tobytes()
        ref = oracle.encode(x)
        assert got == ref, "segment %d" % k
    return sizes


@pytest.mark.parametrize("tokens", [1, 7, 300, 4096])
def test_batched_workload1_shapes(tokens):
    cache = kvgen.contiguous_cache(1, layers=2, tokens=tokens)
    plan = batched_contiguous(cache)
    check_batch_against_oracle(plan, list(cache))


@pytest.mark.slow
@pytest.mark.parametrize("workload", [1, 2, 3])
def test_batched_full_workload(workload):
    cache = kvgen.contiguous_cache(workload)
    plan = batched_contiguous(cache)
    sizes = check_batch_against_oracle(plan, list(cache))
    n = cache.shape[1]
    e = (sizes - (H + n + (n + 1) // 2)) // 5
    frac = e.sum() / cache.size
    if workload == 3:
        assert 0.03 <= frac <= 0.05, frac   # heavy tails: 3-5% escapes
    else:
        assert frac < 0.01


def paged_run(batch, page_elems=kvgen.PAGE_ELEMS, dst_seed=99):
    """Scatter the batch's pages into a pool, encode all requests with one
    batched call, decode into a second pool under another page table."""
    R = batch.n_requests
    pool_pages = batch.pool_pages
    pool = torch.zeros((pool_pages, page_elems), dtype=torch.int16, device=DEV)
    src_slots = np.concatenate(batch.page_table)
    data = np.concatenate(batch.pages).view(np.int16)
    pool[torch.from_numpy(src_slots).to(DEV)] = torch.from_numpy(data).to(DEV)
    del data
    base = pool.data_ptr()
    ptrs = torch.from_numpy(src_slots * (2 * page_elems) + base).to(DEV)
    plan = sz.BatchPlan([int(l) * kvgen.HEADS * kvgen.HEAD_DIM for l in batch.lengths], page_elems, device=DEV)
    assert plan.total_pages == src_slots.size
    plan.encode(ptrs)
    dst = torch.zeros_like(pool)
    dst_slots = np.random.default_rng(dst_seed).permutation(pool_pages)[: src_slots.size]
    dptrs = torch.from_numpy(dst_slots * (2 * page_elems) + dst.data_ptr()).to(DEV)
    plan.decode(dptrs)
    torch.cuda.synchronize()
    assert plan.enc_status.abs().sum().item() == 0
    assert plan.dec_status.abs().sum().item() == 0
    assert torch.equal(dst[torch.from_numpy(dst_slots).to(DEV)], pool[torch.from_numpy(src_slots).to(DEV)])
    return plan


def test_paged_small_batch():
    b = kvgen.paged_batch(n_requests=12, min_tokens=16, max_tokens=600, pool_pages=2048)
    plan = paged_run(b)
    check_batch_against_oracle(plan, [b.request_stream(r) for r in range(b.n_requests)])


@pytest.mark.slow
def test_paged_full_workload4():
    b = kvgen.paged_batch()
    plan = paged_run(b)
    check_batch_against_oracle(plan, [b.request_stream(r) for r in range(b.n_requests)])


@pytest.mark.slow
def test_paged_full_workload4_adversarial():
    # uniform random 16-bit patterns in every page: about 94 % escapes, so
    # every tile writes past the staged escape records; every request's
    # container is compared with the oracle's
    import hashlib
    b = kvgen.paged_batch(adversarial=True)
    plan = paged_run(b)
    sizes = plan.sizes.cpu().numpy()
    for r in range(b.n_requests):
        n = int(b.lengths[r]) * kvgen.HEADS * kvgen.HEAD_DIM
        assert sizes[r] <= sz.max_bytes(n)
    host = plan.container.cpu().numpy()
    want = oracle_digests([b.request_stream(r) for r in range(b.n_requests)])
    for r in range(b.n_requests):
        off = int(plan.out_offset[r])
        got = hashlib.sha256(host[off: off + int(sizes[r])].tobytes()).hexdigest()
        assert got == want[r], "request %d differs from the oracle" % r


@pytest.mark.parametrize("page", [39936, 150016])
def test_pages_with_partial_last_page(page):
    # 39936: pages shorter than a tile (ragged sub-tiles); 150016: three
    # tiles per page (65536 + 65536 + 18944)
    lens = [page * 2 + 1000, 17, page, 5 * page + 64]
    streams = [kvgen.mixed_small(n, seed=600 + i) for i, n in enumerate(lens)]
    plan = sz.BatchPlan(lens, page, device=DEV)
    pages_src = []
    for x in streams:
        for p in range(0, x.size, page):
            chunk = np.zeros(page, np.uint16)
            seg = x[p: p + page]
            chunk[: seg.size] = seg
            pages_src.append(chunk)
    pool = torch.from_numpy(np.stack(pages_src).view(np.int16)).to(DEV)
    perm = np.random.default_rng(5).permutation(len(pages_src))
    pool_perm = pool[torch.from_numpy(perm).to(DEV)].contiguous()
    inv = np.argsort(perm)
    ptrs = torch.from_numpy(inv * (2 * page) + pool_perm.data_ptr()).to(DEV)
    plan.encode(ptrs)
    out = torch.zeros_like(pool)
    optrs = torch.from_numpy(np.arange(len(pages_src)) * (2 * page) + out.data_ptr()).to(DEV)
    plan.decode(optrs)
    torch.cuda.synchronize()
    assert plan.enc_status.abs().sum().item() == 0 and plan.dec_status.abs().sum().item() == 0
    check_batch_against_oracle(plan, streams)
    got = out.cpu().numpy().view(np.uint16)
    i = 0
    for x in streams:
        for p in range(0, x.size, page):
            seg = x[p: p + page]
            assert np.array_equal(got[i, : seg.size], seg)
            i += 1


@pytest.mark.parametrize("dst_page", [8192, 32768, 24576])
def test_decode_into_other_page_size(dst_page):
    """Requests encoded from 16-token pages are decoded straight into a pool
    of another page size under another page table; a request whose length
    is not a multiple of the new page size ends in a partial page.  The
    container of a segment does not depend on paging, and a plan places it
    at an offset that depends only on the segment lengths."""
    b = kvgen.paged_batch(n_requests=10, min_tokens=16, max_tokens=900, pool_pages=4096)
    lens = [int(l) * kvgen.HEADS * kvgen.HEAD_DIM for l in b.lengths]
    src = sz.BatchPlan(lens, kvgen.PAGE_ELEMS, device=DEV)
    pool = torch.zeros((b.pool_pages, kvgen.PAGE_ELEMS), dtype=torch.int16, device=DEV)
    src_slots = np.concatenate(b.page_table)
    pool[torch.from_numpy(src_slots).to(DEV)] = torch.from_numpy(np.concatenate(b.pages).view(np.int16)).to(DEV)
    src.encode(torch.from_numpy(src_slots * (2 * kvgen.PAGE_ELEMS) + pool.data_ptr()).to(DEV))
    dst = sz.BatchPlan(lens, dst_page, device=DEV)
    assert np.array_equal(dst.out_offset, src.out_offset)
    dst_pool = torch.zeros((dst.total_pages + 7, dst_page), dtype=torch.int16, device=DEV)
    slots = np.random.default_rng(77).permutation(dst.total_pages + 7)[: dst.total_pages]
    dst.decode(torch.from_numpy(slots * (2 * dst_page) + dst_pool.data_ptr()).to(DEV), container=src.container)
    torch.cuda.synchronize()
    assert src.enc_status.abs().sum().item() == 0 and dst.dec_status.abs().sum().item() == 0
    got = dst_pool.cpu().numpy().view(np.uint16)
    for r in range(b.n_requests):
        x = b.request_stream(r)
        pages = slots[int(dst.page_begin[r]): int(dst.page_begin[r]) + -(-x.size // dst_page)]
        flat = got[pages].reshape(-1)[: x.size]
        assert np.array_equal(flat, x), "request %d" % r
    check_batch_against_oracle(src, [b.request_stream(r) for r in range(b.n_requests)])


@pytest.mark.parametrize("page,seed", [(64, 1), (64, 2), (192, 3)])
def test_batched_small_pages_cut_ranges_everywhere(page, seed):
    """Hundreds of segments over thousands of small pages (one tile per
    page), so every CTA's range of tiles is cut by segment boundaries at
    every position: segments opening, closing or inside a range, spanning
    many ranges, empty ones, and more segments than the shared-memory
    segment cache holds."""
    rng = np.random.default_rng(seed)
    lens = [int(v) for v in rng.integers(0, 3000, size=300)]
    lens[5] = 0
    lens[17] = page
    lens[18] = 5 * page
    streams = [kvgen.mixed_small(n, seed=1000 * seed + i) for i, n in enumerate(lens)]
    plan = sz.BatchPlan(lens, page, device=DEV)
    pages_src = []
    for x in streams:
        for p in range(0, x.size, page):
            chunk = np.zeros(page, np.uint16)
            seg = x[p: p + page]
            chunk[: seg.size] = seg
            pages_src.append(chunk)
    assert len(pages_src) == plan.total_pages and plan.n_tiles == plan.total_pages
    pool = torch.from_numpy(np.stack(pages_src).view(np.int16)).to(DEV)
    perm = rng.permutation(len(pages_src))
    pool_perm = pool[torch.from_numpy(perm).to(DEV)].contiguous()
    ptrs = torch.from_numpy(np.argsort(perm) * (2 * page) + pool_perm.data_ptr()).to(DEV)
    plan.encode(ptrs)
    out = torch.zeros_like(pool)
    plan.decode(torch.from_numpy(np.arange(len(pages_src)) * (2 * page) + out.data_ptr()).to(DEV))
    torch.cuda.synchronize()
    assert plan.enc_status.abs().sum().item() == 0 and plan.dec_status.abs().sum().item() == 0
    check_batch_against_oracle(plan, streams)
    assert torch.equal(out, pool)
