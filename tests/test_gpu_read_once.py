"""GPU parity of the read-once encode: exponent histograms kept while the
KV cache is written (sz_histogram_accumulate(_batched)), the exact
codebooks chosen from them (sz_select_codebook(_batched)) and the one-pass
encode with those codebooks.

The accumulated histograms must equal the oracle's histogram of each whole
tensor or request bin by bin, the codebooks and escape counts the oracle's
choice, and the containers the oracle's containers byte for byte -- for
streams appended in chunks of every shape: ragged single-stream chunks, the
heads' token slices of Llama-shaped tensors (several segments into one
histogram), paged requests whose pages arrive over several prefill chunks,
and workloads 1-4 at full size (the bench's read-once encode)."""
import hashlib

import numpy as np
import pytest

import kvgen
import oracle
from oracle_pool import oracle_digests, oracle_digests_and_histograms

torch = pytest.importorskip("torch")
import lossless_bf16_kv_splitzip_b200 as sz  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

DEV = "cuda:0"


def to_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(DEV)


def u32(t):
    return t.cpu().numpy().view(np.uint32).astype(np.uint64)


@pytest.mark.parametrize("n,seed", [(1, 1), (4095, 2), (1_000_003, 3), (3 * 65536 + 8, 4)])
def test_single_stream_in_ragged_chunks(n, seed):
    x = kvgen.mixed_small(n, seed=500 + seed)
    d = to_dev(x)
    hist = torch.zeros(256, dtype=torch.int32, device=DEV)
    rng = np.random.default_rng(seed)
    cuts = np.unique(np.concatenate([[0, n], rng.integers(0, n + 1, size=6) // 8 * 8]))
    for a, b in zip(cuts[:-1], cuts[1:]):  # chunk starts on 16-byte boundaries
        sz.sz_histogram_accumulate(d[a:b], int(b - a), hist)
    cb = torch.empty(16, dtype=torch.uint8, device=DEV)
    esc = torch.zeros(1, dtype=torch.int64, device=DEV)
    sz.sz_select_codebook(hist, cb, esc)
    torch.cuda.synchronize()
    h_ref = oracle.histogram(x)
    assert np.array_equal(u32(hist), h_ref)
    cb_ref = oracle.select_top16(h_ref)
    assert np.array_equal(cb.cpu().numpy(), cb_ref)
    assert int(esc.item()) == n - int(h_ref[cb_ref.astype(np.int64)].sum())
    out, size, status = sz.encode_one_pass(d, cb)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert out[: int(size.item())].cpu().numpy().tobytes() == oracle.encode(x)


def test_empty_and_argument_errors():
    hist = torch.zeros(256, dtype=torch.int32, device=DEV)
    sz.sz_histogram_accumulate(None, 0, hist)  # nothing to add
    torch.cuda.synchronize()
    assert int(hist.abs().sum().item()) == 0
    d = torch.zeros(64, dtype=torch.int16, device=DEV)
    with pytest.raises(sz.SzError) as e:
        sz.sz_histogram_accumulate(d.data_ptr() + 2, 16, hist)
    assert e.value.status == sz.SZ_ERR_ALIGN
    with pytest.raises(sz.SzError) as e:
        sz.sz_histogram_accumulate(d, 16, None)
    assert e.value.status == sz.SZ_ERR_NULL


def test_select_of_an_empty_histogram_is_exponents_0_to_15():
    hists = torch.zeros((3, 256), dtype=torch.int32, device=DEV)
    hists[1, 200] = 7
    cbs, esc = sz.select_codebooks(hists)
    torch.cuda.synchronize()
    assert np.array_equal(cbs[0].cpu().numpy(), np.arange(16))
    assert list(cbs[1].cpu().numpy()) == [200] + list(range(15))
    assert esc.cpu().tolist() == [0, 0, 0]


def head_chunks(cache, tokens, chunk):
    """The new data of each prefill chunk of a [S][8 h][T][128] cache: for
    every tensor and head, tokens [c*chunk, (c+1)*chunk) -- a contiguous run
    of chunk*128 elements.  Yields (page pointers, lengths, hist rows)."""
    S = cache.shape[0]
    d_in = cache  # a device tensor [S, 8*T*128]
    for c0 in range(0, tokens, chunk):
        t = min(chunk, tokens - c0)
        ptrs, rows = [], []
        for k in range(S):
            for h in range(kvgen.HEADS):
                ptrs.append(d_in.data_ptr() + 2 * ((h * tokens + c0) * kvgen.HEAD_DIM) + 2 * k * d_in.shape[1])
                rows.append(k)
        yield ptrs, [t * kvgen.HEAD_DIM] * len(ptrs), rows


def read_once_contiguous(d_cache, tokens, chunk):
    """Accumulate the cache chunk by chunk, select, one-pass encode the
    whole cache.  Returns (histograms, codebooks, escapes, plan)."""
    S, n = d_cache.shape
    hists = torch.zeros((S, 256), dtype=torch.int32, device=DEV)
    for ptrs, lens, rows in head_chunks(d_cache, tokens, chunk):
        p = sz.BatchPlan(lens, lens[0], device=DEV, buffers=False)
        p.accumulate(torch.tensor(ptrs, dtype=torch.int64, device=DEV), hists,
                     torch.tensor(rows, dtype=torch.int32, device=DEV))
        torch.cuda.synchronize()
        assert p.acc_status.abs().sum().item() == 0
    cbs, esc = sz.select_codebooks(hists)
    plan = sz.BatchPlan([n] * S, n, device=DEV)
    ptrs = torch.tensor([d_cache.data_ptr() + 2 * n * k for k in range(S)], dtype=torch.int64, device=DEV)
    plan.encode_one_pass(ptrs, cbs)
    torch.cuda.synchronize()
    assert plan.enc_status.abs().sum().item() == 0
    return hists, cbs, esc, plan


def container_digests(plan):
    sizes = plan.sizes.cpu().numpy()
    host = plan.container.cpu().numpy()
    return [hashlib.sha256(host[int(plan.out_offset[k]): int(plan.out_offset[k]) + int(sizes[k])].tobytes())
            .hexdigest() for k in range(plan.n_segs)]


@pytest.mark.parametrize("tokens,chunk", [(4096, 1024), (300, 128), (7, 7)])
def test_heads_token_chunks_into_tensor_histograms(tokens, chunk):
    cache = kvgen.contiguous_cache(1, layers=2, tokens=tokens)
    hists, cbs, esc, plan = read_once_contiguous(to_dev(cache), tokens, chunk)
    for k in range(cache.shape[0]):
        h_ref = oracle.histogram(cache[k])
        assert np.array_equal(u32(hists[k]), h_ref), "tensor %d" % k
        cb_ref = oracle.select_top16(h_ref)
        assert np.array_equal(cbs[k].cpu().numpy(), cb_ref)
        assert int(esc[k].item()) == cache.shape[1] - int(h_ref[cb_ref.astype(np.int64)].sum())
    assert container_digests(plan) == [hashlib.sha256(oracle.encode(x)).hexdigest() for x in cache]


def test_misaligned_page_is_reported():
    pool = torch.zeros(4096, dtype=torch.int16, device=DEV)
    p = sz.BatchPlan([64, 64], 64, device=DEV, buffers=False)
    hists = torch.zeros((2, 256), dtype=torch.int32, device=DEV)
    ptrs = torch.tensor([pool.data_ptr(), pool.data_ptr() + 130], dtype=torch.int64, device=DEV)
    p.accumulate(ptrs, hists)
    torch.cuda.synchronize()
    assert p.acc_status.cpu().tolist() == [0, sz.SZ_ERR_ALIGN]
    assert int(hists[0].sum().item()) == 64


def paged_read_once(b, n_chunks=3):
    """A paged batch whose pages are written over n_chunks prefill chunks
    (request r's pages split into n_chunks runs), each chunk's new pages
    accumulated in one batched call; then select and one pass over the
    whole batch.  Returns (hists, plan)."""
    P = kvgen.PAGE_ELEMS
    pool = torch.zeros((b.pool_pages, P), dtype=torch.int16, device=DEV)
    for r in range(b.n_requests):
        pool[torch.from_numpy(b.page_table[r]).to(DEV)] = torch.from_numpy(b.pages[r].view(np.int16)).to(DEV)
    base = pool.data_ptr()
    hists = torch.zeros((b.n_requests, 256), dtype=torch.int32, device=DEV)
    for c in range(n_chunks):
        lens, ptrs, rows = [], [], []
        for r in range(b.n_requests):
            slots = np.array_split(b.page_table[r], n_chunks)[c]
            if slots.size == 0:
                continue
            lens.append(slots.size * P)
            ptrs.extend(int(base + 2 * P * s) for s in slots)
            rows.append(r)
        p = sz.BatchPlan(lens, P, device=DEV, buffers=False)
        p.accumulate(torch.tensor(ptrs, dtype=torch.int64, device=DEV), hists,
                     torch.tensor(rows, dtype=torch.int32, device=DEV))
        torch.cuda.synchronize()
        assert p.acc_status[: len(lens)].abs().sum().item() == 0
    cbs, _ = sz.select_codebooks(hists)
    lens = [int(v) * kvgen.HEADS * kvgen.HEAD_DIM for v in b.lengths]
    plan = sz.BatchPlan(lens, P, device=DEV)
    src = np.concatenate(b.page_table)
    plan.encode_one_pass(torch.from_numpy(src * (2 * P) + base).to(DEV), cbs)
    torch.cuda.synchronize()
    assert plan.enc_status.abs().sum().item() == 0
    return hists, plan


def test_paged_requests_over_prefill_chunks():
    b = kvgen.paged_batch(n_requests=12, min_tokens=16, max_tokens=600, pool_pages=2048)
    hists, plan = paged_read_once(b)
    streams = [b.request_stream(r) for r in range(b.n_requests)]
    for r, x in enumerate(streams):
        assert np.array_equal(u32(hists[r]), oracle.histogram(x)), "request %d" % r
    assert container_digests(plan) == [hashlib.sha256(oracle.encode(x)).hexdigest() for x in streams]


@pytest.mark.slow
@pytest.mark.parametrize("workload,chunk", [(1, 1024), (2, 4096), (3, 2048)])
def test_full_workload_read_once(workload, chunk):
    layers, tokens = kvgen.CONTIGUOUS[workload]
    cache = kvgen.contiguous_cache(workload)
    d = to_dev(cache)
    del cache
    hists, cbs, esc, plan = read_once_contiguous(d, tokens, chunk)
    want = oracle_digests_and_histograms(kvgen.contiguous_tensor,
                                         [(workload, k // 2, k % 2) for k in range(2 * layers)])
    got = container_digests(plan)
    H = u32(hists)
    for k, (dig, h_ref) in enumerate(want):
        assert np.array_equal(H[k], np.array(h_ref, np.uint64)), "tensor %d histogram" % k
        assert got[k] == dig, "tensor %d container" % k


@pytest.mark.slow
def test_full_workload4_read_once():
    b = kvgen.paged_batch()
    hists, plan = paged_read_once(b, n_chunks=4)
    streams = [b.request_stream(r) for r in range(b.n_requests)]
    H = u32(hists)
    for r, x in enumerate(streams):
        assert np.array_equal(H[r], oracle.histogram(x)), "request %d" % r
    assert container_digests(plan) == oracle_digests(streams)
