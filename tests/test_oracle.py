"""Pins for the fp64 oracle (CPU only).

The source pages print no worked attention example, no closed form and no error bound
(they only name DiT joint attention, the USP Ring split and an FP8 attention backend), so
the oracle is pinned by mathematics: an independent long-double brute force, a library
cross-check, closed forms, invariants, and checks that plausible mistakes planted into
the oracle are caught by at least one pin.
"""

import math

import numpy as np
import pytest

import oracle
import oracle.attn as oatt
from oracle import brute, fp8
from workloads import chunk_bounds, make_tensor

REL = 1e-12


def _rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    denom = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / denom)


def _qkv(B, H, Sq, Skv, D, seed, std=1.0):
    return (make_tensor((B, H, Sq, D), seed, std), make_tensor((B, H, Skv, D), seed + 1, std),
            make_tensor((B, H, Skv, D), seed + 2, std))


# ----------------------------------------------------------------------------------------
# Pins: each takes the attention and merge functions under test and raises on failure.
# ----------------------------------------------------------------------------------------

def pin_brute_force(attn, mrg):
    """fp64 NumPy oracle vs long-double triple loop on tiny shapes and sub-ranges."""
    seed = 100
    for S in (1, 2, 3, 7, 16, 64):
        for D in (1, 4, 64):
            q, k, v = _qkv(1, 2, S, S, D, seed)
            seed += 3
            scale = 1.0 / math.sqrt(D)
            for k0, k1 in {(0, S), (0, (S + 1) // 2), (S // 3, S), (S // 2, S // 2)}:
                o, l = attn(q, k, v, scale, k0, k1)
                ob, lb = brute.brute_attention(q, k, v, scale, k0, k1)
                if k0 == k1:
                    assert np.all(o == 0) and np.all(np.isneginf(l))
                    continue
                assert _rel_err(o, ob) < REL, (S, D, k0, k1)
                assert _rel_err(l, lb) < REL, (S, D, k0, k1)


def pin_library_sdpa(attn, mrg):
    """Cross-check against torch's CPU scaled_dot_product_attention in float64."""
    import torch
    q, k, v = _qkv(2, 3, 40, 53, 16, 7)
    scale = 0.3
    o, _ = attn(q, k, v, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.astype(np.float64)), torch.from_numpy(k.astype(np.float64)),
        torch.from_numpy(v.astype(np.float64)), scale=scale).numpy()
    assert _rel_err(o, ref) < REL


def pin_equal_keys(attn, mrg):
    """All keys equal: uniform weights, out = mean of V rows, lse = s q.k + log n."""
    q, _, v = _qkv(1, 2, 9, 37, 8, 11)
    k_row = make_tensor((8,), 99)
    k = np.broadcast_to(k_row, (1, 2, 37, 8)).copy()
    for k0, k1 in ((0, 37), (5, 20)):
        o, l = attn(q, k, v, 0.7, k0, k1)
        mean_v = v[:, :, k0:k1].astype(np.float64).mean(axis=2, keepdims=True)
        assert _rel_err(o, np.broadcast_to(mean_v, o.shape)) < REL
        lse_ref = 0.7 * (q.astype(np.float64) @ k_row.astype(np.float64)) + math.log(k1 - k0)
        assert _rel_err(l, lse_ref) < REL


def pin_dominant_key(attn, mrg):
    """One key aligned with the query and 60+ nats above the rest: out = its V row."""
    rng = np.random.default_rng(5)
    D, N = 16, 50
    for trial in range(4):
        q = make_tensor((1, 1, 1, D), 200 + trial)
        k = make_tensor((1, 1, N, D), 300 + trial, std=0.1)
        v = make_tensor((1, 1, N, D), 400 + trial)
        j = int(rng.integers(N))
        qn = q[0, 0, 0].astype(np.float64)
        k[0, 0, j] = (40.0 * qn / np.linalg.norm(qn)).astype(np.float32)
        scale = 1.0
        x = scale * (k[0, 0].astype(np.float64) @ qn)
        gap = x[j] - np.max(np.delete(x, j))
        assert gap > 60.0
        o, l = attn(q, k, v, scale)
        assert np.max(np.abs(o[0, 0, 0] - v[0, 0, j])) < N * math.exp(-60.0) * 10
        assert abs(l[0, 0, 0] - x[j]) < 1e-12 * abs(x[j]) + 1e-12


def pin_single_key(attn, mrg):
    """S_kv = 1: out = v_0, lse = s q.k_0."""
    q, k, v = _qkv(2, 2, 5, 1, 8, 21)
    o, l = attn(q, k, v, 0.25)
    assert _rel_err(o, np.broadcast_to(v, o.shape)) < REL
    ref = 0.25 * np.einsum("bhsd,bhd->bhs", q.astype(np.float64), k[:, :, 0].astype(np.float64))
    assert _rel_err(l, ref) < REL


def pin_kv_permutation(attn, mrg):
    q, k, v = _qkv(1, 2, 20, 45, 8, 31)
    perm = np.random.default_rng(1).permutation(45)
    o1, l1 = attn(q, k, v, 0.5)
    o2, l2 = attn(q, k[:, :, perm], v[:, :, perm], 0.5)
    assert _rel_err(o2, o1) < REL and _rel_err(l2, l1) < REL


def pin_q_permutation(attn, mrg):
    q, k, v = _qkv(1, 2, 20, 45, 8, 41)
    perm = np.random.default_rng(2).permutation(20)
    o1, l1 = attn(q, k, v, 0.5)
    o2, l2 = attn(q[:, :, perm], k, v, 0.5)
    assert _rel_err(o2, o1[:, :, perm]) < REL and _rel_err(l2, l1[:, :, perm]) < REL


def pin_key_shift(attn, mrg):
    """k_j -> k_j + u for all j: out unchanged, lse_i += s q_i.u."""
    q, k, v = _qkv(1, 2, 20, 45, 8, 51)
    u = make_tensor((8,), 52)
    s = 0.5
    o1, l1 = attn(q, k, v, s)
    o2, l2 = attn(q, k.astype(np.float64) + u.astype(np.float64), v, s)
    assert _rel_err(o2, o1) < 1e-11
    shift = s * (q.astype(np.float64) @ u.astype(np.float64))
    assert _rel_err(l2, l1 + shift) < 1e-11


def pin_linear_in_v(attn, mrg):
    q, k, v1 = _qkv(1, 2, 20, 45, 8, 61)
    v2 = make_tensor(v1.shape, 64)
    beta = -1.75
    o1, _ = attn(q, k, v1, 0.5)
    o2, _ = attn(q, k, v2, 0.5)
    o3, _ = attn(q, k, v1.astype(np.float64) + beta * v2.astype(np.float64), 0.5)
    assert _rel_err(o3, o1 + beta * o2) < 1e-11


def pin_rows_sum_to_one(attn, mrg):
    """V = 1 everywhere gives out = 1 exactly when each softmax row sums to 1."""
    q, k, _ = _qkv(1, 3, 30, 70, 8, 71)
    ones = np.ones((1, 3, 70, 4))
    o, _ = attn(q, k, ones, 0.9)
    assert np.max(np.abs(o - 1.0)) < REL
    p = oracle.softmax_rows(q[0, 0], k[0, 0], 0.9)
    assert np.max(np.abs(p.sum(axis=1) - 1.0)) < REL


def pin_chunk_merge(attn, mrg):
    """Merging any chunking of KV by LSE equals the unchunked result."""
    q, k, v = _qkv(2, 2, 33, 90, 8, 81)
    o_full, l_full = attn(q, k, v, 0.4)
    chunkings = [chunk_bounds(90, 2), chunk_bounds(90, 4), [(0, 7), (7, 61), (61, 90)],
                 [(0, 0), (0, 45), (45, 45), (45, 90)], [(0, 90)]]
    for bounds in chunkings:
        parts = [attn(q, k, v, 0.4, a, b) for a, b in bounds]
        o, l = mrg([p[0] for p in parts], [p[1] for p in parts])
        assert _rel_err(o, o_full) < REL, bounds
        assert _rel_err(l, l_full) < REL, bounds


def pin_merge_grouping(attn, mrg):
    """merge(merge(a, b), c) = merge(a, merge(b, c)) = merge(a, b, c)."""
    q, k, v = _qkv(1, 2, 17, 60, 8, 91)
    pa, pb, pc = (attn(q, k, v, 0.6, a, b) for a, b in [(0, 13), (13, 40), (40, 60)])
    abc = mrg([pa[0], pb[0], pc[0]], [pa[1], pb[1], pc[1]])
    ab = mrg([pa[0], pb[0]], [pa[1], pb[1]])
    left = mrg([ab[0], pc[0]], [ab[1], pc[1]])
    bc = mrg([pb[0], pc[0]], [pb[1], pc[1]])
    right = mrg([pa[0], bc[0]], [pa[1], bc[1]])
    for o, l in (left, right):
        assert _rel_err(o, abc[0]) < REL and _rel_err(l, abc[1]) < REL


def pin_merge_empty(attn, mrg):
    """All chunks empty: out = 0, lse = -inf, no NaN; an empty chunk is ignored."""
    o = np.full((2, 3, 4), 5.0)
    l = np.full((2, 3), -np.inf)
    out, lse = mrg([o, o], [l, l])
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    l2 = np.random.default_rng(3).standard_normal((2, 3))
    o2 = np.random.default_rng(4).standard_normal((2, 3, 4))
    out, lse = mrg([o, o2], [l, l2])
    assert np.max(np.abs(out - o2)) < REL and np.max(np.abs(lse - l2)) < REL


PINS = [pin_brute_force, pin_library_sdpa, pin_equal_keys, pin_dominant_key, pin_single_key,
        pin_kv_permutation, pin_q_permutation, pin_key_shift, pin_linear_in_v,
        pin_rows_sum_to_one, pin_chunk_merge, pin_merge_grouping, pin_merge_empty]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(oracle.attention, oracle.merge)


# ----------------------------------------------------------------------------------------
# Planted mistakes: each mutant of the oracle must fail at least one pin.
# ----------------------------------------------------------------------------------------

def _blk_no_scale(qb, kk, vv, scale):
    return _REAL_BLOCK(qb, kk, vv, 1.0)


def _blk_wrong_sign(qb, kk, vv, scale):
    return _REAL_BLOCK(qb, kk, vv, -scale)


def _blk_k_for_v(qb, kk, vv, scale):
    o, l = _REAL_BLOCK(qb, kk, kk[:, :vv.shape[1]] if kk.shape[1] >= vv.shape[1] else vv, scale)
    return o, l


def _blk_lse_no_max(qb, kk, vv, scale):
    x = scale * (qb @ kk.T)
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    den = e.sum(axis=1, keepdims=True)
    return (e / den) @ vv, np.log(den)[:, 0]


def _blk_softmax_wrong_axis(qb, kk, vv, scale):
    x = scale * (qb @ kk.T)
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    den = e.sum(axis=1, keepdims=True)
    p = e / e.sum(axis=0, keepdims=True)
    return p @ vv, (m + np.log(den))[:, 0]


def _blk_drop_last_key(qb, kk, vv, scale):
    if kk.shape[0] > 1:
        kk, vv = kk[:-1], vv[:-1]
    return _REAL_BLOCK(qb, kk, vv, scale)


def _blk_transposed_q(qb, kk, vv, scale):
    # q rows and feature columns swapped where the shapes allow (square blocks)
    if qb.shape[0] == qb.shape[1]:
        qb = qb.T
    else:
        qb = qb[::-1]
    return _REAL_BLOCK(qb, kk, vv, scale)


_REAL_BLOCK = oatt._row_block

BLOCK_MUTANTS = [_blk_no_scale, _blk_wrong_sign, _blk_k_for_v, _blk_lse_no_max,
                 _blk_softmax_wrong_axis, _blk_drop_last_key, _blk_transposed_q]


def _merge_unnormalised(outs, lses):
    o, l = oracle.merge(outs, lses)
    L = np.stack([np.asarray(x, dtype=np.float64) for x in lses])
    M = np.max(L, axis=0)
    w = np.exp(L - np.where(np.isneginf(M), 0, M)).sum(axis=0)
    return o * np.where(np.isneginf(M), 1, w)[..., None], l


def _merge_lse_no_max(outs, lses):
    o, l = oracle.merge(outs, lses)
    M = np.max(np.stack([np.asarray(x, dtype=np.float64) for x in lses]), axis=0)
    return o, np.where(np.isneginf(M), l, l - M)


def _merge_first_only(outs, lses):
    return np.asarray(outs[0], dtype=np.float64), np.asarray(lses[0], dtype=np.float64)


MERGE_MUTANTS = [_merge_unnormalised, _merge_lse_no_max, _merge_first_only]


def _caught(attn, mrg):
    failures = 0
    for pin in PINS:
        try:
            pin(attn, mrg)
        except AssertionError:
            failures += 1
        except (ValueError, IndexError, FloatingPointError):
            failures += 1
    return failures


@pytest.mark.parametrize("mutant", BLOCK_MUTANTS, ids=[m.__name__ for m in BLOCK_MUTANTS])
def test_planted_block_mistake_is_caught(mutant, monkeypatch):
    monkeypatch.setattr(oatt, "_row_block", mutant)
    with np.errstate(all="ignore"):
        assert _caught(oatt.attention, oracle.merge) >= 1


@pytest.mark.parametrize("mutant", MERGE_MUTANTS, ids=[m.__name__ for m in MERGE_MUTANTS])
def test_planted_merge_mistake_is_caught(mutant):
    with np.errstate(all="ignore"):
        assert _caught(oracle.attention, mutant) >= 1


def test_planted_range_mistake_is_caught():
    def off_by_one(q, k, v, scale, k0=0, k1=None, rows=None):
        k1 = k.shape[2] if k1 is None else k1
        return oracle.attention(q, k, v, scale, min(k0 + 1, k1), k1, rows)
    assert _caught(off_by_one, oracle.merge) >= 1


# ----------------------------------------------------------------------------------------
# Row subsets and input layout
# ----------------------------------------------------------------------------------------

def test_row_subset_matches_full():
    q, k, v = _qkv(1, 2, 600, 300, 8, 5)
    o, l = oracle.attention(q, k, v, 0.3)
    rows = [0, 5, 255, 256, 257, 599]
    os_, ls = oracle.attention(q, k, v, 0.3, rows=rows)
    assert _rel_err(os_, o[:, :, rows]) < REL and _rel_err(ls, l[:, :, rows]) < REL


# ----------------------------------------------------------------------------------------
# E4M3 format pins
# ----------------------------------------------------------------------------------------

def test_e4m3_decode_closed_forms():
    vals = fp8.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert vals[0x00] == 0.0 and np.signbit(vals[0x80])
    assert vals[0x7E] == 448.0 and vals[0xFE] == -448.0          # largest finite
    assert vals[0x08] == 2.0 ** -6                                # smallest normal
    assert vals[0x01] == 2.0 ** -9                                # smallest subnormal
    assert vals[0x38] == 1.0 and vals[0x40] == 2.0 and vals[0xB8] == -1.0
    assert np.isnan(vals[0x7F]) and np.isnan(vals[0xFF])
    assert np.sum(np.isnan(vals)) == 2                            # no infinities
    pos = vals[:0x7F]
    assert np.all(np.diff(pos) > 0)                               # monotone in the code
    assert np.count_nonzero(pos) == 126


def test_e4m3_decode_matches_torch():
    import torch
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = fp8.e4m3_decode(np.arange(256, dtype=np.uint8))
    same = (ref == ours) | (np.isnan(ref) & np.isnan(ours))
    assert np.all(same)


def test_e4m3_encode_round_trip_and_ties():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = fp8.e4m3_decode(codes)
    assert np.array_equal(fp8.e4m3_encode(vals), codes)
    pos = fp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    got = fp8.e4m3_encode(mids)
    lo = np.arange(0x7E)
    want = np.where(lo % 2 == 0, lo, lo + 1)                      # ties to even code
    assert np.array_equal(got, want.astype(np.uint8))
    eps = 1e-9
    assert np.array_equal(fp8.e4m3_encode(mids * (1 + eps)), (lo + 1).astype(np.uint8))
    assert np.array_equal(fp8.e4m3_encode(mids * (1 - eps)), lo.astype(np.uint8))
    assert fp8.e4m3_encode(np.array([1e6]))[0] == 0x7E            # saturate
    assert fp8.e4m3_encode(np.array([-1e6]))[0] == 0xFE
    assert fp8.e4m3_encode(np.array([460.0]))[0] == 0x7E
    assert fp8.e4m3_encode(np.array([2.0 ** -10]))[0] == 0x00     # tie to zero (even)
    assert fp8.e4m3_encode(np.array([-0.0]))[0] == 0x80


def test_e4m3_encode_matches_torch_in_range():
    import torch
    x = np.random.default_rng(0).standard_normal(200000).astype(np.float32) * 60
    x = np.clip(x, -440, 440).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.e4m3_encode(x), ref)


def test_quantize_per_tensor():
    x = make_tensor((3, 1000), 9) * np.float32(3.0)
    codes, descale = fp8.quantize_per_tensor(x)
    amax = np.max(np.abs(x))
    assert descale == np.float32(amax / np.float32(448.0))
    deq = fp8.dequantize(codes, descale)
    # E4M3 relative step is 2^-3 for normals: error <= half a step of |x| (plus subnormal floor)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, descale * 2.0 ** -10)
    assert np.all(np.abs(deq - x) <= bound * (1 + 1e-12))
    assert np.max(np.abs(deq)) == pytest.approx(amax, rel=2 ** -4)
    zc, zd = fp8.quantize_per_tensor(np.zeros(10, dtype=np.float32))
    assert zd == 1.0 and np.all(zc == 0)


def test_quantize_per_block_constructed_scales():
    """Block i of each (b, h) holds E4M3-exact values times 2^i with 448 * 2^i present, so its
    descale is exactly 2^i and its codes are the plain encodings of the pattern; the ragged
    last block (S = 2 * 128 + 5) and an all-zero block follow the same rule."""
    rng = np.random.default_rng(3)
    B, H, S, D = 2, 3, 2 * 128 + 5, 16
    pos = fp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    pattern_codes = rng.integers(0, 0x7F, size=(B, H, S, D)).astype(np.uint8)
    pattern_codes |= (rng.integers(0, 2, size=pattern_codes.shape) << 7).astype(np.uint8)
    pattern_codes[:, :, ::128, 0] = 0x7E                  # 448 in every block
    x = fp8.e4m3_decode(pattern_codes)
    for i in range(3):
        x[:, :, i * 128:(i + 1) * 128] *= 2.0 ** i
    x[1, 2, 128:256] = 0.0                                 # one all-zero block
    codes, ds = fp8.quantize_per_block(x.astype(np.float32))
    want_ds = np.broadcast_to(np.array([1.0, 2.0, 4.0], dtype=np.float32), (B, H, 3)).copy()
    want_ds[1, 2, 1] = 0.0                                 # all-zero block: descale 0
    assert ds.dtype == np.float32 and np.array_equal(ds, want_ds)
    want_codes = pattern_codes.copy()
    want_codes[1, 2, 128:256] = np.where(np.signbit(x[1, 2, 128:256]), 0x80, 0x00)
    assert np.array_equal(codes, want_codes)
    assert np.array_equal(fp8.dequantize_per_block(codes, ds), x)
    assert np.all(np.isin(pos, pos))


def test_quantize_per_block_is_per_tensor_on_each_block():
    """Each block's codes and descale equal a per-tensor quantisation of that block alone, and
    one block covering all rows is the per-tensor quantiser itself."""
    x = make_tensor((1, 2, 300, 8), 11) * np.float32(5.0)
    x[0, 1, 150:170] *= np.float32(1e5)                     # an outlier run in block 1 of head 1
    codes, ds = fp8.quantize_per_block(x)
    assert ds.shape == (1, 2, 3)
    for h in range(2):
        for i, (a, b) in enumerate([(0, 128), (128, 256), (256, 300)]):
            c1, d1 = fp8.quantize_per_tensor(x[0, h, a:b])
            assert d1 == ds[0, h, i] and np.array_equal(c1, codes[0, h, a:b])
    z = np.zeros((1, 1, 130, 8), dtype=np.float32)
    z[0, 0, 0, 0] = -0.0
    zc, zd = fp8.quantize_per_block(z)
    assert np.array_equal(zd, np.zeros((1, 1, 2), dtype=np.float32))
    assert np.array_equal(zc, fp8.quantize_per_tensor(z)[0])      # codes of x / 1
    cw, dw = fp8.quantize_per_block(x[:, :1], block_rows=300)
    ct, dt = fp8.quantize_per_tensor(x[:, :1])
    assert dw[0, 0, 0] == dt and np.array_equal(cw, ct)
    # the outlier run pushes head 0 into the subnormal codes under one per-tensor scale; with
    # block scales head 0 keeps E4M3's relative step (rel-L2 about 2^-5)
    ct2, dt2 = fp8.quantize_per_tensor(x)

    def rel(a):
        return np.linalg.norm(a[0, 0] - x[0, 0]) / np.linalg.norm(x[0, 0])
    assert rel(fp8.dequantize_per_block(codes, ds)) < 0.05 and rel(fp8.dequantize(ct2, dt2)) > 0.2


# ------------------------------------------------------------------ neighborhood attention
from oracle import neighborhood as nbh  # noqa: E402


def test_window_start_is_the_nearest_k_positions():
    """The clamped window equals the K positions nearest to i (by brute force over the line;
    for odd K there is never a tie at the window's edge)."""
    for L in range(1, 13):
        for K in range(1, L + 1, 2):
            for i in range(L):
                order = sorted(range(L), key=lambda j: (abs(j - i), j))
                near = sorted(order[:K])
                assert abs(order[K - 1] - i) < abs(order[K] - i) if K < L else True
                st = nbh.window_start(i, K, L)
                assert near == list(range(st, st + K)), (L, K, i)
    with pytest.raises(ValueError):
        nbh.window_start(0, 4, 10)
    with pytest.raises(ValueError):
        nbh.window_start(0, 5, 3)


def _na_loops(q, k, v, grid, kernel, scale):
    """Pure-Python loops: key j is a neighbour of query i when, in every dimension, j's
    coordinate is among the K coordinates nearest to i's (the definition above, written
    without window_start)."""
    import math
    T, Y, X = grid
    B, H, S, D = q.shape

    def near(i, K, L):
        return set(sorted(range(L), key=lambda j: (abs(j - i), j))[:K])

    out = np.zeros((B, H, S, D))
    lse = np.zeros((B, H, S))
    for b in range(B):
        for h in range(H):
            for s in range(S):
                t, y, x = s // (Y * X), (s // X) % Y, s % X
                nt, ny, nx = near(t, kernel[0], T), near(y, kernel[1], Y), near(x, kernel[2], X)
                keys = [j for j in range(S) if j // (Y * X) in nt and (j // X) % Y in ny and j % X in nx]
                xs = [scale * sum(float(q[b, h, s, d]) * float(k[b, h, j, d]) for d in range(D)) for j in keys]
                m = max(xs)
                es = [math.exp(a - m) for a in xs]
                den = sum(es)
                for d in range(D):
                    out[b, h, s, d] = sum(e * float(v[b, h, j, d]) for e, j in zip(es, keys)) / den
                lse[b, h, s] = m + math.log(den)
    return out, lse


@pytest.mark.parametrize("grid,kernel", [((2, 3, 4), (1, 3, 3)), ((3, 4, 5), (3, 3, 1)), ((1, 5, 6), (1, 3, 5)),
                                         ((4, 2, 3), (3, 1, 3))])
def test_neighborhood_matches_loops(grid, kernel):
    S = int(np.prod(grid))
    q, k, v = (make_tensor((1, 2, S, 3), seed) for seed in (21, 22, 23))
    o, l = nbh.neighborhood_attention_3d(q, k, v, grid, kernel, 0.7)
    ro, rl = _na_loops(q, k, v, grid, kernel, 0.7)
    assert np.allclose(o, ro, rtol=0, atol=1e-12) and np.allclose(l, rl, rtol=0, atol=1e-12)


def test_neighborhood_full_window_is_full_attention():
    grid = (3, 5, 7)
    q, k, v = (make_tensor((2, 1, 105, 8), seed) for seed in (31, 32, 33))
    o, l = nbh.neighborhood_attention_3d(q, k, v, grid, grid, 0.3)
    ro, rl = oracle.attention(q, k, v, 0.3)
    assert np.allclose(o, ro, rtol=0, atol=1e-12) and np.allclose(l, rl, rtol=0, atol=1e-12)


def test_neighborhood_unit_window_is_self():
    grid = (2, 3, 4)
    q, k, v = (make_tensor((1, 2, 24, 4), seed) for seed in (41, 42, 43))
    o, l = nbh.neighborhood_attention_3d(q, k, v, grid, (1, 1, 1), 0.5)
    assert np.array_equal(o, v.astype(np.float64))
    assert np.allclose(l, 0.5 * np.einsum("bhsd,bhsd->bhs", q.astype(np.float64), k.astype(np.float64)),
                       rtol=0, atol=1e-12)


def test_neighborhood_rows_subset_and_counts():
    grid, kernel = (5, 6, 7), (3, 5, 3)
    q, k, v = (make_tensor((1, 1, 210, 4), seed) for seed in (51, 52, 53))
    o, l = nbh.neighborhood_attention_3d(q, k, v, grid, kernel, 0.4)
    rows = [0, 6, 41, 209, 100]
    os_, ls = nbh.neighborhood_attention_3d(q, k, v, grid, kernel, 0.4, rows=rows)
    assert np.array_equal(os_, o[:, :, rows]) and np.array_equal(ls, l[:, :, rows])
    for s in range(210):
        idx = nbh.neighbor_index(grid, kernel, s)
        assert len(set(idx.tolist())) == 45 and s in idx
