"""Pins of the CPU oracle against facts that do not come from the oracle.

The oracle (oracle/sz_oracle.c) is what the CUDA library is checked against, so it is
itself checked here against what the SplitZip explainer and arithmetic fix:

* field split vs IEEE-754 arithmetic (frexp) on all 65,536 BF16 patterns
  (explainer section 1, "La structure de la Note");
* the exhaustive closed form: every exponent occurs 256 times, so the
  codebook is 0..15, e = 61,440 and the container is 405,552 bytes;
* top-16 validity by brute force (explainer section 3, "Top 16");
* escape count e = N - sum of the codebook's counts, and the size formula
  48 + N + ceil(N/2) + 5e;
* losslessness, decode(encode(x)) == x bit for bit ("Les Resultats");
* hand-written golden containers (tests/golden), written from the container
  specification, not from code;
* rejection of corrupt containers;
* planted mistakes: mutated copies of the oracle must fail these pins.
"""
import os
import shutil
import struct
import subprocess

import numpy as np
import pytest

import kvgen
import oracle
from conftest import ROOT, load_golden

H = 48


def ieee_fields(bits: np.ndarray):
    """(sign, exponent field, mantissa field) of BF16 bit patterns derived
    from the float value by IEEE-754 arithmetic, not by bit masks."""
    with np.errstate(invalid="ignore"):
        f = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    sign = np.signbit(f).astype(np.int64)
    a = np.abs(f)
    E = np.zeros(bits.shape, np.int64)
    M = np.zeros(bits.shape, np.int64)
    nan = np.isnan(f)
    inf = np.isinf(f)
    sub = (a < 2.0 ** -126) & ~nan
    normal = ~(nan | inf | sub)
    mant, k = np.frexp(a[normal])          # a = mant * 2**k, mant in [0.5, 1)
    E[normal] = k + 126
    M[normal] = np.rint((mant * 2.0 - 1.0) * 128.0).astype(np.int64)
    E[sub] = 0
    M[sub] = np.rint(a[sub] / 2.0 ** -133).astype(np.int64)
    E[inf] = 255
    M[inf] = 0
    E[nan] = 255
    M[nan] = -1                            # payload not derivable from the value
    return sign, E, M


def parse(blob: bytes):
    n, e = struct.unpack_from("<QQ", blob, 8)
    cb = np.frombuffer(blob, np.uint8, 16, 24)
    sm = np.frombuffer(blob, np.uint8, n, H)
    codes = np.frombuffer(blob, np.uint8, (n + 1) // 2, H + n)
    off = H + n + (n + 1) // 2
    pos = np.frombuffer(blob, "<u4", e, off).astype(np.int64)
    raw = np.frombuffer(blob, np.uint8, e, off + 4 * e)
    nib = np.empty(2 * codes.size, np.uint8)
    nib[0::2] = codes & 0x0F
    nib[1::2] = codes >> 4
    return n, e, cb, sm, nib[:n], pos, raw


def exponents_from_container(blob):
    n, e, cb, sm, nib, pos, raw = parse(blob)
    E = cb[nib].astype(np.int64)
    E[pos] = raw
    return E, sm


# ---------------------------------------------------------------- field split
def test_field_split_matches_ieee_on_all_patterns():
    x = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    blob = oracle.encode(x)
    E, sm = exponents_from_container(blob)
    sign, E_ref, M_ref = ieee_fields(x)
    assert np.array_equal(E, E_ref)
    assert np.array_equal((sm >> 7).astype(np.int64), sign)
    ok = M_ref >= 0
    assert np.array_equal((sm & 0x7F).astype(np.int64)[ok], M_ref[ok])
    # NaN patterns: a nonzero mantissa, carried through unchanged
    assert np.all((sm & 0x7F)[~ok] != 0)


def test_histogram_matches_ieee_bincount():
    x = kvgen.mixed_small(50_000, seed=11)
    _, E_ref, _ = ieee_fields(x)
    assert np.array_equal(oracle.histogram(x), np.bincount(E_ref, minlength=256).astype(np.uint64))


# ------------------------------------------------------------ closed forms
def test_exhaustive_closed_form():
    x = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    blob = oracle.encode(x)
    n, e, cb, *_ = parse(blob)
    assert n == 65536
    assert list(cb) == list(range(16))
    assert e == 61440
    assert len(blob) == 405552
    assert np.array_equal(oracle.decode(blob, n), x)


def test_each_pattern_alone_roundtrips():
    # a one-element tensor: its exponent is the only one that occurs, so it
    # must get code 0 and there is no escape
    _, E_ref, _ = ieee_fields(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    for v in range(0, 65536, 7):
        x = np.array([v], np.uint16)
        blob = oracle.encode(x)
        assert len(blob) == H + 1 + 1
        assert blob[24] == E_ref[v]
        assert blob[16] == 0
        assert oracle.decode(blob, 1)[0] == v


def test_single_exponent_has_no_escapes():
    rng = np.random.default_rng(3)
    n = 10_001
    sign = rng.integers(0, 2, n).astype(np.uint16) << 15
    mant = rng.integers(0, 128, n).astype(np.uint16)
    x = sign | np.uint16(130 << 7) | mant
    blob = oracle.encode(x)
    n_, e, cb, *_ = parse(blob)
    assert e == 0 and cb[0] == 130
    assert list(cb[1:]) == [v for v in range(16) if v != 130][:15]
    assert len(blob) == H + n + (n + 1) // 2
    assert np.array_equal(oracle.decode(blob, n), x)


def test_seventeen_equal_counts_highest_escapes():
    exps = np.arange(100, 117)
    reps = 9
    x = (np.repeat(exps, reps).astype(np.uint16) << 7) | np.uint16(5)
    x = np.random.default_rng(4).permutation(x)
    blob = oracle.encode(x)
    n, e, cb, sm, nib, pos, raw = parse(blob)
    assert list(cb) == list(range(100, 116))
    assert e == reps and np.all(raw == 116)
    assert np.array_equal(pos, np.flatnonzero((x >> 7) == 116))
    assert np.array_equal(oracle.decode(blob, n), x)


def test_fewer_than_16_exponents_fill_ascending():
    x = np.array([200 << 7, 3 << 7, 200 << 7, 64 << 7], np.uint16)
    cb = parse(oracle.encode(x))[2]
    # 200 (count 2) first, then 3 and 64 (count 1, ascending), then unused 0,1,2,4,...
    assert list(cb) == [200, 3, 64, 0, 1, 2, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13]


# ----------------------------------------------------------- top-16 validity
@pytest.mark.parametrize("seed", range(40))
def test_top16_is_a_valid_selection_brute_force(seed):
    rng = np.random.default_rng([77, seed])
    n_exp = int(rng.integers(1, 60))
    exps = rng.choice(256, n_exp, replace=False)
    counts = rng.integers(1, 6, n_exp)            # small counts -> many ties
    x = np.repeat(exps, counts).astype(np.uint16) << 7
    x |= rng.integers(0, 1 << 16, x.size).astype(np.uint16) & np.uint16(0x807F)
    x = rng.permutation(x)
    blob = oracle.encode(x)
    n, e, cb, *_ = parse(blob)
    cnt = np.zeros(256, np.int64)
    cnt[exps] = counts
    members = [int(v) for v in cb]
    assert len(set(members)) == 16
    # every member beats every non-member under (count desc, exponent asc)
    for m in members:
        for o in range(256):
            if o in members:
                continue
            assert cnt[m] > cnt[o] or (cnt[m] == cnt[o] and m < o)
    # the codebook itself is listed in that order
    for a, b in zip(members, members[1:]):
        assert cnt[a] > cnt[b] or (cnt[a] == cnt[b] and a < b)
    # escapes: exactly the elements whose exponent is not a member
    assert e == x.size - sum(int(cnt[m]) for m in members)
    assert np.array_equal(oracle.decode(blob, n), x)


# ---------------------------------------------------- invariants and sizes
@pytest.mark.parametrize("n", [0, 1, 2, 3, 15, 16, 17, 31, 33, 4095, 4097, 65537])
def test_small_sizes_roundtrip_and_size_formula(n):
    x = kvgen.mixed_small(n, seed=n + 1000)
    blob = oracle.encode(x)
    n_, e, cb, *_ = parse(blob)
    assert n_ == n
    assert len(blob) == H + n + (n + 1) // 2 + 5 * e
    h = oracle.histogram(x)
    assert e == n - int(sum(h[int(c)] for c in cb))
    assert np.array_equal(oracle.decode(blob, n), x)


def test_kv_workload0_invariants():
    x = kvgen.tiny_k_tensor()
    blob = oracle.encode(x)
    n, e, cb, sm, nib, pos, raw = parse(blob)
    _, E_ref, _ = ieee_fields(x)
    member = np.isin(E_ref, cb)
    assert e == int((~member).sum())
    assert np.array_equal(pos, np.flatnonzero(~member))
    assert np.array_equal(raw.astype(np.int64), E_ref[~member])
    assert np.all(nib[~member] == 0)
    assert e >= 1049 * 0.5                # the forced outliers escape
    ratio = 2 * n / len(blob)
    assert 1.25 < ratio < 4 / 3
    assert np.array_equal(oracle.decode(blob, n), x)


def test_adversarial_within_worst_case_bound():
    n = 1 << 20
    x = kvgen.uniform_u16(n, seed=5)
    blob = oracle.encode(x)
    bound = H + n + (n + 1) // 2 + 5 * (n - (n + 15) // 16)
    assert len(blob) <= bound
    e = parse(blob)[1]
    assert abs(e / n - 15 / 16) < 0.01
    assert np.array_equal(oracle.decode(blob, n), x)


def test_given_codebook_roundtrip():
    x = kvgen.mixed_small(20_000, seed=9)
    cb = np.arange(120, 136, dtype=np.uint8)
    blob = oracle.encode(x, codebook=cb)
    n, e, cb2, *_ = parse(blob)
    assert list(cb2) == list(cb)
    _, E_ref, _ = ieee_fields(x)
    assert e == int((~np.isin(E_ref, cb)).sum())
    assert np.array_equal(oracle.decode(blob, n), x)


# --------------------------------------------------------------- goldens
def test_goldens(golden_names):
    assert len(golden_names) >= 5
    for name in golden_names:
        n, inp, cont = load_golden(name)
        x = np.array(inp, np.uint16)
        assert x.size == n
        assert oracle.encode(x) == cont, name
        assert np.array_equal(oracle.decode(cont, n), x), name


# ------------------------------------------------------- corrupt containers
def _corruptions(blob, n):
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
    if e >= 2:
        mut("unsorted", lambda c: struct.pack_into("<I", c, off_pos + 4, 0))
        mut("pos_range", lambda c: struct.pack_into("<I", c, off_pos, n + 5))
        mut("raw_in_codebook", lambda c: c.__setitem__(off_pos + 4 * e, c[24]))
    out["truncated"] = bytes(b[:-1])
    return out


def test_corrupt_containers_are_rejected():
    x = kvgen.mixed_small(3001, seed=21)
    blob = oracle.encode(x)
    assert parse(blob)[1] >= 2
    bad = _corruptions(blob, x.size)
    assert len(bad) >= 11
    for name, c in bad.items():
        st, _ = oracle.decode_status(c, x.size)
        assert st == oracle.ERR_CORRUPT, name
    # placeholder nibble of an escaped element must be 0
    n, e, cb, sm, nib, pos, raw = parse(blob)
    p = int(pos[0])
    c = bytearray(blob)
    c[H + n + p // 2] |= (1 << 4) if p % 2 else 1
    assert oracle.decode_status(bytes(c), n)[0] == oracle.ERR_CORRUPT
    # odd count: the unused high nibble must be 0
    x3 = np.array([0x3F80, 0x3F80, 0x3F80], np.uint16)
    c = bytearray(oracle.encode(x3))
    c[H + 3 + 1] |= 0x10
    assert oracle.decode_status(bytes(c), 3)[0] == oracle.ERR_CORRUPT


# ----------------------------------------------------------- planted mistakes
MUTANTS = {
    # swapped nibble order inside a code byte
    "nibble_order": ("out[off_codes + i / 2] |= (uint8_t)nibble;\n",
                     "out[off_codes + i / 2] |= (uint8_t)(nibble << 4);\n", 1),
    # reversed tie-break
    "tie_break": ("return a->exponent < b->exponent ? -1 : 1;",
                  "return a->exponent > b->exponent ? -1 : 1;", 1),
    # sign bit dropped from the sm byte
    "sign": ("return (uint8_t)((field_sign(x) << 7) | field_mantissa(x));",
             "return (uint8_t)(field_mantissa(x));", 1),
    # escape position off by one
    "pos_index": ("put_u32(out + off_pos + 4 * k_esc, (uint32_t)i);",
                  "put_u32(out + off_pos + 4 * k_esc, (uint32_t)(i + 1));", 1),
    # least common first
    "count_order": ("return a->count > b->count ? -1 : 1;",
                    "return a->count < b->count ? -1 : 1;", 1),
}


def _build_mutant(tmp_path, name):
    old, new, count = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "sz_oracle.c")).read()
    assert src.count(old) == count, name
    d = tmp_path / name
    d.mkdir()
    shutil.copy(os.path.join(ROOT, "oracle", "sz_oracle.h"), d / "sz_oracle.h")
    (d / "sz_oracle.c").write_text(src.replace(old, new))
    so = d / "libmut.so"
    subprocess.check_call(["gcc", "-O1", "-shared", "-fPIC", "-o", str(so), str(d / "sz_oracle.c")])
    return str(so)


def _mutant_passes_pins(so):
    import ctypes
    lib = ctypes.CDLL(so)
    u64 = ctypes.c_uint64
    lib.szo_encode.argtypes = [ctypes.c_void_p, u64, ctypes.c_void_p, u64, ctypes.c_void_p,
                               ctypes.c_void_p]
    lib.szo_encode.restype = ctypes.c_int

    def enc(x):
        cap = H + x.size + (x.size + 1) // 2 + 5 * x.size
        out = np.zeros(cap, np.uint8)
        sz = ctypes.c_uint64(0)
        es = ctypes.c_uint64(0)
        st = lib.szo_encode(x.ctypes.data, x.size, out.ctypes.data, cap, ctypes.byref(sz),
                            ctypes.byref(es))
        return None if st else out[: sz.value].tobytes()

    for name in sorted(os.listdir(os.path.join(ROOT, "tests", "golden"))):
        n, inp, cont = load_golden(name)
        if enc(np.array(inp, np.uint16)) != cont:
            return False
    x = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    blob = enc(x)
    if blob is None or len(blob) != 405552 or list(blob[24:40]) != list(range(16)):
        return False
    return True


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    assert not _mutant_passes_pins(_build_mutant(tmp_path, name))


def test_unmutated_copy_passes_pins(tmp_path):
    d = tmp_path / "clean"
    d.mkdir()
    shutil.copy(os.path.join(ROOT, "oracle", "sz_oracle.h"), d / "sz_oracle.h")
    shutil.copy(os.path.join(ROOT, "oracle", "sz_oracle.c"), d / "sz_oracle.c")
    so = d / "lib.so"
    subprocess.check_call(["gcc", "-O1", "-shared", "-fPIC", "-o", str(so), str(d / "sz_oracle.c")])
    assert _mutant_passes_pins(str(so))
