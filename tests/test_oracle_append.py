"""Pins of the oracle's cache-append step (the step before the decode: the
new token's rows are written into its paged slot).

- Rows appended token by token (and two at a time) into a pool with a random
  page permutation, read back with gather_paged, equal the rows in order.
- Slots no append touches keep their bytes.
- FP4 shared-latent appends, one token at a time, equal cache_write of the
  whole sequence byte for byte: the same RoPE position and quantiser.
- A page id outside the pool, or more new tokens than the length, raises.
"""
import numpy as np
import pytest

from oracle import mla as omla
from oracle import v41


def _pool_and_table(rng, lens, page_size, C, dtype):
    npages = [(int(L) + page_size - 1) // page_size for L in lens]
    perm = rng.permutation(sum(npages))
    bt = np.full((len(lens), max(npages)), -1, np.int32)
    k = 0
    for b, n in enumerate(npages):
        bt[b, :n] = perm[k:k + n]
        k += n
    pool = (rng.integers(0, 256, (sum(npages), page_size, C)).astype(dtype) if dtype == np.uint8
            else rng.standard_normal((sum(npages), page_size, C)).astype(dtype))
    return pool, bt


@pytest.mark.parametrize("Q", [1, 2])
def test_appends_read_back_in_order(Q):
    rng = np.random.Generator(np.random.PCG64(41))
    lens = np.array([130, 6, 64], np.int64)
    page, C = 64, 8
    pool, bt = _pool_and_table(rng, lens, page, C, np.float64)
    rows = rng.standard_normal((3, int(lens.max()), C))
    for b in range(3):                       # ragged: each sequence in chunks of up to Q tokens
        for t0 in range(0, int(lens[b]), Q):
            chunk = rows[b, t0:min(t0 + Q, int(lens[b]))]
            pool = omla.cache_append(pool, bt[b:b + 1], np.array([t0 + len(chunk)]), chunk[None], page)
    got = omla.gather_paged(pool, bt, lens, page)
    for b in range(3):
        np.testing.assert_array_equal(got[b, :lens[b]], rows[b, :lens[b]])


def test_batched_append_equals_per_sequence_appends():
    rng = np.random.Generator(np.random.PCG64(45))
    lens = np.array([65, 128, 1], np.int64)
    pool, bt = _pool_and_table(rng, lens, 64, 8, np.float64)
    new = rng.standard_normal((3, 1, 8))
    one = omla.cache_append(pool, bt, lens, new, 64)
    each = pool
    for b in range(3):
        each = omla.cache_append(each, bt[b:b + 1], lens[b:b + 1], new[b:b + 1], 64)
    np.testing.assert_array_equal(one, each)


def test_untouched_slots_keep_their_bytes():
    rng = np.random.Generator(np.random.PCG64(42))
    lens = np.array([70, 3], np.int64)
    pool, bt = _pool_and_table(rng, lens, 64, 288, np.uint8)
    before = pool.copy()
    new = rng.integers(0, 256, (2, 1, 288)).astype(np.uint8)
    after = omla.cache_append(pool, bt, lens, new, 64)
    changed = np.argwhere((after != before).any(axis=-1))
    slots = {(int(bt[b, (lens[b] - 1) // 64]), int((lens[b] - 1) % 64)) for b in range(2)}
    assert {tuple(map(int, c)) for c in changed} <= slots
    np.testing.assert_array_equal(pool, before)   # the input pool is not modified


def test_fp4_token_appends_equal_cache_write():
    rng = np.random.Generator(np.random.PCG64(43))
    B, Lk, D, page = 2, 100, 512, 64
    lat = rng.standard_normal((B, Lk, D))
    want = v41.cache_write(lat)
    lens = np.full(B, Lk, np.int64)
    pool, bt = _pool_and_table(rng, lens, page, 288, np.uint8)
    for t in range(Lk):
        pool = v41.fp4_cache_append(pool, bt, np.full(B, t + 1, np.int64), lat[:, t:t + 1], page)
    got = np.stack([np.stack([pool[bt[b, t // page], t % page] for t in range(Lk)]) for b in range(B)])
    np.testing.assert_array_equal(got, want)


def test_fp4_two_token_append_uses_both_positions():
    rng = np.random.Generator(np.random.PCG64(44))
    lat = rng.standard_normal((1, 2, 512))
    lens = np.array([9], np.int64)
    pool, bt = _pool_and_table(rng, lens, 64, 288, np.uint8)
    pool = v41.fp4_cache_append(pool, bt, lens, lat, 64)
    # tokens 7 and 8: the same bytes as cache_write rows 7 and 8 of a 9-token sequence
    full = np.zeros((1, 9, 512))
    full[0, 7:9] = lat[0]
    want = v41.cache_write(full)[0, 7:9]
    np.testing.assert_array_equal(pool[bt[0, 0], 7:9], want)


def test_bad_page_or_length_raises():
    pool = np.zeros((2, 64, 8))
    with pytest.raises(ValueError):
        omla.cache_append(pool, np.array([[5]]), np.array([1]), np.zeros((1, 1, 8)), 64)
    with pytest.raises(ValueError):
        omla.cache_append(pool, np.array([[0]]), np.array([1]), np.zeros((1, 2, 8)), 64)


def test_f32_decisions_agree_with_f64_away_from_ties():
    # both modes choose the same codes unless a quotient lies within float32
    # rounding of a nearest-even boundary; on N(0,1) latents that is rare
    rng = np.random.Generator(np.random.PCG64(46))
    lat = rng.standard_normal((4, 64, 512)).astype(np.float32).astype(np.float64)
    a = v41.fp4_quantize(lat)
    b = v41.fp4_quantize(lat, decide_in_f32=True)
    assert (a != b).mean() < 1e-4


def test_f32_decision_on_a_constructed_boundary():
    # amax = 6 * 2^-3 * (1 + 1/16): amax/6 sits exactly between the E4M3 values
    # 2^-3 and 2^-3 * (1 + 1/8); nearest-even picks the even mantissa (2^-3)
    x = np.zeros((1, 512))
    x[0, 0] = 6 * 0.125 * (1 + 1 / 16)
    for mode in (False, True):
        e = v41.fp4_quantize(x, decide_in_f32=mode)
        assert v41.e4m3_decode(e[0, 256:257])[0] == 0.125
