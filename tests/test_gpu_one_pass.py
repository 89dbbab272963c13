"""GPU parity of the one-pass encode with caller codebooks, through the C ABI.

The container of sz_encode_one_pass(_batched) must equal, byte for byte,
the oracle's container for the same input and the same codebook -- the
tensor's own top 16 (then also the two-pass path's container) or any other
16 distinct exponents.  Covered: ragged sizes, multi-tile streams, foreign
codebooks whose escapes overflow the per-tile record slots (the placement
kernel reads those tiles again), incompressible input, an invalid codebook,
a container that does not fit, empty segments, batches whose CTA ranges are
cut by segment boundaries everywhere, and decoding the result."""
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
FOREIGN = np.arange(118, 134, dtype=np.uint8)  # exponents 2^-9 .. 2^6: not the tensors' own order
FAR = np.arange(200, 216, dtype=np.uint8)      # nothing the generators draw: every element escapes


def to_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(DEV)


def own_codebook(x):
    return oracle.select_top16(oracle.histogram(x)).astype(np.uint8)


def skewed_codebook(x):
    """The tensor's own top 16 with its two most frequent exponents swapped
    for unused ones: a large share of escapes, still within the
    top-16 container bound."""
    cb = own_codebook(x).copy()
    cb[0], cb[1] = 200, 201
    return cb


def one_pass(x, cb):
    out, size, status = sz.encode_one_pass(to_dev(x), torch.from_numpy(np.ascontiguousarray(cb)).to(DEV))
    torch.cuda.synchronize()
    return int(status.item()), out[: int(size.item())].cpu().numpy().tobytes()


@pytest.mark.parametrize("n", [0, 1, 17, 16383, 16384, 65536, 65537, 3 * 65536 + 100, 1000003])
def test_own_codebook_equals_oracle(n):
    x = kvgen.mixed_small(n, seed=700 + n % 97)
    cb = own_codebook(x) if n else np.arange(16, dtype=np.uint8)
    st, got = one_pass(x, cb)
    assert st == 0
    assert got == oracle.encode(x)


@pytest.mark.parametrize("n", [5000, 65536 + 3, 4 * 65536 + 999])
def test_foreign_codebook(n):
    x = kvgen.mixed_small(n, seed=800 + n % 89)
    st, got = one_pass(x, FOREIGN)
    assert st == 0
    assert got == oracle.encode(x, codebook=FOREIGN)


@pytest.mark.parametrize("n", [65536 + 3, 4 * 65536 + 999])
@pytest.mark.parametrize("kind", ["far", "skewed"])
def test_escapes_overflowing_tile_slots(n, kind):
    # every full tile holds more than the 4,096 records its slot keeps: the
    # placement kernel finds them again in the input
    x = kvgen.mixed_small(n, seed=810 + n % 83)
    cb = FAR if kind == "far" else skewed_codebook(x)
    st, got = one_pass(x, cb)
    assert st == 0
    assert got == oracle.encode(x, codebook=cb)
    e = int(np.frombuffer(got[16:24], np.uint64)[0])
    assert e > 4096 * (n // 65536)


def test_incompressible_input():
    x = kvgen.uniform_u16(3 * 65536 + 77, seed=801)
    cb = own_codebook(x)
    st, got = one_pass(x, cb)
    assert st == 0 and got == oracle.encode(x)
    assert len(got) <= sz.max_bytes(x.size)


def test_decodes_back():
    x = kvgen.contiguous_tensor(3, 1, 0, tokens=256)  # heavy tails
    st, got = one_pass(x, FOREIGN)
    assert st == 0
    c = torch.from_numpy(np.frombuffer(got, np.uint8).copy()).to(DEV)
    y, dst = sz.decode(c, x.size)
    torch.cuda.synchronize()
    assert int(dst.item()) == 0
    assert np.array_equal(y.cpu().numpy().view(np.uint16), x)


def test_repeated_codebook_is_rejected():
    x = kvgen.mixed_small(70000, seed=802)
    bad = np.full(16, 120, np.uint8)
    st, got = one_pass(x, bad)
    assert st == sz.SZ_ERR_INVALID and got == b""


def test_container_that_does_not_fit():
    x = kvgen.mixed_small(70000, seed=803)
    n = x.size
    small = 48 + n + (n + 1) // 2 + 10
    _, wsb = sz.sz_plan_one_pass(n)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    out = torch.empty(small, dtype=torch.uint8, device=DEV)
    size = torch.ones(1, dtype=torch.int64, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    sz.sz_encode_one_pass(to_dev(x), n, torch.from_numpy(FOREIGN).to(DEV), out, small, size, st, ws, wsb)
    torch.cuda.synchronize()
    assert int(st.item()) == sz.SZ_ERR_CAPACITY and int(size.item()) == 0


def paged_pool(streams, page):
    pages = []
    for x in streams:
        for p in range(0, x.size, page):
            chunk = np.zeros(page, np.uint16)
            seg = x[p: p + page]
            chunk[: seg.size] = seg
            pages.append(chunk)
    return torch.from_numpy(np.stack(pages).view(np.int16)).to(DEV)


@pytest.mark.parametrize("page,seed", [(64, 11), (192, 12), (16384, 13)])
def test_batched_matches_two_pass_and_oracle(page, seed):
    rng = np.random.default_rng(seed)
    lens = [int(v) for v in rng.integers(0, 3000 if page < 1024 else 200000, size=120)]
    lens[3] = 0
    streams = [kvgen.mixed_small(n, seed=2000 * seed + i) for i, n in enumerate(lens)]
    pool = paged_pool(streams, page)
    ptrs = torch.from_numpy(np.arange(pool.shape[0]) * (2 * page) + pool.data_ptr()).to(DEV)
    # own codebooks for most segments, skewed ones (many escapes) for every fifth
    def pick(i, x):
        if x.size == 0:
            return np.arange(16, dtype=np.uint8)
        return skewed_codebook(x) if i % 5 == 4 else own_codebook(x)
    cbs = np.stack([pick(i, x) for i, x in enumerate(streams)])
    one = sz.BatchPlan(lens, page, device=DEV)
    one.encode_one_pass(ptrs, torch.from_numpy(cbs).to(DEV))
    two = sz.BatchPlan(lens, page, device=DEV)
    two.encode(ptrs)
    torch.cuda.synchronize()
    assert one.enc_status.abs().sum().item() == 0 and two.enc_status.abs().sum().item() == 0
    s1, s2 = one.sizes.cpu().numpy(), two.sizes.cpu().numpy()
    h1, h2 = one.container.cpu().numpy(), two.container.cpu().numpy()
    for k, x in enumerate(streams):
        o = int(one.out_offset[k])
        got = h1[o: o + int(s1[k])].tobytes()
        if k % 5 == 4 and x.size:
            assert got == oracle.encode(x, codebook=cbs[k]), k
        else:
            assert got == h2[o: o + int(s2[k])].tobytes(), k
            assert got == oracle.encode(x), k
    # and the decode restores every page
    out = torch.zeros_like(pool)
    one.decode(torch.from_numpy(np.arange(pool.shape[0]) * (2 * page) + out.data_ptr()).to(DEV))
    torch.cuda.synchronize()
    assert one.dec_status.abs().sum().item() == 0
    assert torch.equal(out, pool)


def test_batched_workload1_reuses_codebooks_bit_exactly():
    """The 4K-token Llama-3-8B cache (64 tensors, 512 MiB): codebooks kept
    from a two-pass encode give the same containers in one pass."""
    layers, tokens = kvgen.CONTIGUOUS[1]
    n = kvgen.HEADS * tokens * kvgen.HEAD_DIM
    host = np.empty((2 * layers, n), np.uint16)
    kvgen.contiguous_cache(1, layers=layers, out=host)
    d = torch.from_numpy(host.view(np.int16)).to(DEV)
    ptrs = torch.tensor([d.data_ptr() + 2 * n * k for k in range(2 * layers)], dtype=torch.int64, device=DEV)
    two = sz.BatchPlan([n] * (2 * layers), n, device=DEV)
    two.encode(ptrs)
    one = sz.BatchPlan([n] * (2 * layers), n, device=DEV)
    one.encode_one_pass(ptrs, two.codebooks)
    torch.cuda.synchronize()
    assert one.enc_status.abs().sum().item() == 0
    assert torch.equal(one.sizes, two.sizes)
    for k in range(2 * layers):
        o = int(one.out_offset[k])
        z = int(one.sizes[k])
        assert torch.equal(one.container[o: o + z], two.container[o: o + z]), k
    k = 2 * layers - 1
    o = int(one.out_offset[k])
    assert one.container[o: o + int(one.sizes[k])].cpu().numpy().tobytes() == oracle.encode(host[k])


@pytest.mark.parametrize("workload,tokens", [(1, 1024), (3, 512)])
def test_previous_layer_codebooks_equal_oracle(workload, tokens):
    """Codebook reuse across layers, as the bench measures it: layer L's K
    and V tensors encoded in one pass with layer L-1's K and V codebooks
    (layer 0 with its own).  Every container is the oracle's container for
    that codebook, and decodes back."""
    layers = 4
    cache = kvgen.contiguous_cache(workload, layers=layers, tokens=tokens)
    S, n = cache.shape
    own = np.stack([own_codebook(x) for x in cache])
    prev = own.copy()
    prev[2:] = own[:-2]
    d = torch.from_numpy(cache.view(np.int16)).to(DEV)
    ptrs = torch.tensor([d.data_ptr() + 2 * n * k for k in range(S)], dtype=torch.int64, device=DEV)
    plan = sz.BatchPlan([n] * S, n, device=DEV)
    plan.encode_one_pass(ptrs, torch.from_numpy(prev).to(DEV))
    torch.cuda.synchronize()
    assert plan.enc_status.abs().sum().item() == 0
    sizes = plan.sizes.cpu().numpy()
    host = plan.container.cpu().numpy()
    for k in range(S):
        o = int(plan.out_offset[k])
        assert host[o: o + int(sizes[k])].tobytes() == oracle.encode(cache[k], codebook=prev[k]), k
    out = torch.zeros_like(d)
    plan.decode(torch.tensor([out.data_ptr() + 2 * n * k for k in range(S)], dtype=torch.int64, device=DEV))
    torch.cuda.synchronize()
    assert plan.dec_status.abs().sum().item() == 0 and torch.equal(out, d)
