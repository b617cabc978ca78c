"""GPU parity of mla_cache_append (the step before the decode) against the oracle.

- bf16 and fp32 rows are copied bit for bit into their slots (paged and
  contiguous; Q = 1 and Q = 2), and no other slot changes.
- FP4 shared-latent entries (tail rotated at the token's position, then
  quantised) equal the oracle's entries byte for byte when the oracle takes
  the quantiser's decisions in float32, the kernel's precision.
- A page id outside the pool sets MLA_DEVICE_ERR_BLOCK_TABLE and that token
  is not written; the others are.
- A decode after the append sees the new token: it matches the oracle decode
  of the oracle-appended cache.
"""
import numpy as np
import pytest
import torch

from latent_kv_decode_b200 import workloads as wl
from oracle import mla as omla
from oracle import v41

from harness import (TOL_BF16, TOL_LSE_BF16, REL_L2_BF16, assert_close, dev, fp4_pool,
                     oracle_shared_latent)

pytestmark = pytest.mark.gpu


def _table(rng, lens, page):
    npages = [(int(L) + page - 1) // page for L in lens]
    perm = rng.permutation(sum(npages)).astype(np.int32)
    bt = np.full((len(lens), max(npages)), -1, np.int32)
    k = 0
    for b, n in enumerate(npages):
        bt[b, :n] = perm[k:k + n]
        k += n
    return bt, sum(npages)


def _bf16(a):
    return torch.from_numpy(wl.bf16_round(np.asarray(a, np.float32))).to(torch.bfloat16)


def _i32(a):
    return torch.from_numpy(np.asarray(a, np.int32)).cuda()


@pytest.mark.parametrize("Q", [1, 2])
def test_bf16_paged_append_bit_exact(Q):
    """Combined 576-wide pool rows: latent into [:512], rope into [512:]."""
    from latent_kv_decode_b200 import ops
    rng = np.random.Generator(np.random.PCG64(51))
    lens = np.array([130, 6, 64, 65], np.int64)
    bt, npg = _table(rng, lens, 64)
    pool = _bf16(rng.standard_normal((npg, 64, 576)))
    new = _bf16(rng.standard_normal((4, Q, 576)))
    want = omla.cache_append(pool.float().numpy(), bt, lens, new.float().numpy(), 64)
    dpool = pool.cuda()
    dnew = new.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.mla_cache_append(dnew[..., :512].contiguous(), dnew[..., 512:].contiguous(), dpool[..., :512],
                         dpool[..., 512:], _i32(lens), block_table=_i32(bt), err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(dpool.cpu(), torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16))


@pytest.mark.parametrize("Q", [1, 2])
def test_f32_contiguous_append_bit_exact(Q):
    """Separate (B, Lk, 512) latent and (B, Lk, 32) rope caches, float32."""
    from latent_kv_decode_b200 import ops
    rng = np.random.Generator(np.random.PCG64(53))
    B, Lk = 3, 40
    lens = np.array([40, 2, 17], np.int64)
    kv = rng.standard_normal((B, Lk, 512)).astype(np.float32)
    pe = rng.standard_normal((B, Lk, 32)).astype(np.float32)
    c_kv = rng.standard_normal((B, Q, 512)).astype(np.float32)
    k_pe = rng.standard_normal((B, Q, 32)).astype(np.float32)
    want_kv, want_pe = kv.copy(), pe.copy()
    for b in range(B):
        for i in range(Q):
            t = int(lens[b]) - Q + i
            want_kv[b, t], want_pe[b, t] = c_kv[b, i], k_pe[b, i]
    dkv, dpe = dev(kv), dev(pe)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.mla_cache_append(dev(c_kv), dev(k_pe), dkv, dpe, _i32(lens), err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(dkv.cpu().numpy(), want_kv)
    assert np.array_equal(dpe.cpu().numpy(), want_pe)


@pytest.mark.parametrize("src", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("Q", [1, 2])
def test_fp4_paged_append_matches_oracle_f32_decisions(src, Q):
    from latent_kv_decode_b200 import ops
    rng = np.random.Generator(np.random.PCG64(52 + Q))
    lens = np.array([100, 7, 64, 8191], np.int64)   # the last one rotates at a large position
    bt, npg = _table(rng, lens, 64)
    pool = rng.integers(0, 256, (npg, 64, 288)).astype(np.uint8)
    lat = torch.from_numpy(rng.standard_normal((4, Q, 512)).astype(np.float32)).to(src)
    want = v41.fp4_cache_append(pool, bt, lens, lat.float().numpy().astype(np.float64), 64,
                                decide_in_f32=True)
    dpool = torch.from_numpy(pool).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.mla_cache_append(lat.cuda(), None, dpool, None, _i32(lens), block_table=_i32(bt),
                         rope_tail=64, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = dpool.cpu().numpy()
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[:4].tolist()}"


def test_fp4_contiguous_append_without_rope():
    """Contiguous (B, Lk, 288) entries, rope_tail = 0: the latent is quantised as is."""
    from latent_kv_decode_b200 import ops
    rng = np.random.Generator(np.random.PCG64(54))
    B, Lk = 2, 96
    lens = np.array([96, 33], np.int64)
    cache = rng.integers(0, 256, (B, Lk, 288)).astype(np.uint8)
    lat = rng.standard_normal((B, 1, 512)).astype(np.float32)
    ent = v41.fp4_quantize(lat.astype(np.float64), 512, decide_in_f32=True)
    want = cache.copy()
    for b in range(B):
        want[b, int(lens[b]) - 1] = ent[b, 0]
    dcache = dev(cache)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.mla_cache_append(dev(lat), None, dcache, None, _i32(lens), rope_tail=0, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(dcache.cpu().numpy(), want)


@pytest.mark.parametrize("fp4", [False, True])
def test_bad_page_id_sets_flag_and_writes_nothing_for_that_token(fp4):
    from latent_kv_decode_b200 import ops
    rng = np.random.Generator(np.random.PCG64(55))
    lens = np.array([70, 130], np.int64)
    bt, npg = _table(rng, lens, 64)
    bad = bt.copy()
    bad[0, 1] = npg + 5                       # token 69 of sequence 0 has no valid page
    if fp4:
        pool = rng.integers(0, 256, (npg, 64, 288)).astype(np.uint8)
        lat = rng.standard_normal((2, 1, 512)).astype(np.float32)
        want = v41.fp4_cache_append(pool, bt[1:], lens[1:], lat[1:].astype(np.float64), 64,
                                    decide_in_f32=True)
        dpool = dev(pool)
        args = (dev(lat), None, dpool, None)
        kw = dict(rope_tail=64)
    else:
        pool = _bf16(rng.standard_normal((npg, 64, 512)))
        new = _bf16(rng.standard_normal((2, 1, 512)))
        want = omla.cache_append(pool.float().numpy(), bt[1:], lens[1:], new[1:].float().numpy(), 64)
        dpool = pool.cuda()
        args = (new.cuda(), None, dpool, None)
        kw = {}
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.mla_cache_append(*args, _i32(lens), block_table=_i32(bad), err_flag=err, **kw)
    torch.cuda.synchronize()
    assert int(err.item()) & 1
    got = dpool.cpu()
    if fp4:
        assert np.array_equal(got.numpy(), want)
    else:
        assert torch.equal(got, torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16))


def test_bf16_append_then_decode_sees_the_new_token():
    """Decode a paged bf16 cache whose last token was written by mla_cache_append."""
    from latent_kv_decode_b200 import ops
    w = wl.make_mla(3, 128, 1, 128, 64, 128, 512, 0, dtype="bf16", seed=56, seq_lens=[200, 64, 129],
                    paged=True)
    rng = np.random.Generator(np.random.PCG64(57))
    new_kv = wl.bf16_round(rng.standard_normal((3, 1, 512)).astype(np.float32))
    new_pe = wl.bf16_round(rng.standard_normal((3, 1, 64)).astype(np.float32))
    lens = w.lens()
    kv_pool = omla.cache_append(w.kv_pool, w.block_table, lens, new_kv, 64)
    pe_pool = omla.cache_append(w.pe_pool, w.block_table, lens, new_pe, 64)
    # the device pools start from the workload's pools; the append writes the new rows
    dkv, dpe = dev(w.kv_pool, torch.bfloat16), dev(w.pe_pool, torch.bfloat16)
    bt, sl = dev(w.block_table), dev(w.seq_lens)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.mla_cache_append(dev(new_kv, torch.bfloat16), dev(new_pe, torch.bfloat16), dkv, dpe, sl,
                         block_table=bt, err_flag=err)
    q_lat = ops.mla_absorb_q(dev(w.q_nope, torch.bfloat16), dev(w.wkv_b, torch.bfloat16))
    x, lse = ops.decode(q_lat, dev(w.q_pe, torch.bfloat16), dkv, dpe, w.softmax_scale, seq_lens=sl,
                        block_table=bt, num_splits=2, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    gq = q_lat.float().cpu().numpy().astype(np.float64)
    kv = omla.gather_paged(kv_pool, w.block_table, lens, 64)
    pe = omla.gather_paged(pe_pool, w.block_table, lens, 64)
    vis = omla.visibility(3, 1, kv.shape[1], w.seq_lens)
    xo, _, lo = omla.latent_attention(gq, w.q_pe, kv, pe, w.softmax_scale, vis)
    assert_close(x.float().cpu().numpy(), xo, TOL_BF16, "x", REL_L2_BF16)
    assert_close(lse.cpu().numpy(), lo, TOL_LSE_BF16, "lse")


def test_fp4_append_then_decode_sees_the_new_token():
    """Shared-latent FP4: the last token of each sequence appended on the GPU, then decoded."""
    from latent_kv_decode_b200 import ops
    w = wl.make_shared_latent(3, 64, 1, 300, seed=58, seq_lens=[300, 65, 130], paged=True)
    full = v41.cache_write(w.latent, w.rope_tail, w.rope_theta)          # oracle entries, all tokens
    lens = w.lens()
    pool = fp4_pool(w, full)
    stale = pool.copy()
    for b in range(w.B):                                                # the slot of the last token
        t = int(lens[b]) - 1                                            # holds garbage before the append
        stale[w.block_table[b, t // 64], t % 64] = 0xFF
    last = np.stack([w.latent[b, int(lens[b]) - 1] for b in range(w.B)])[:, None, :]
    dpool = dev(stale)
    bt, sl = dev(w.block_table), dev(w.seq_lens)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.mla_cache_append(dev(last.astype(np.float32)), None, dpool, None, sl, block_table=bt,
                         rope_tail=w.rope_tail, rope_theta=w.rope_theta, err_flag=err)
    call = ops.mla_decode(dev(w.q, torch.bfloat16), None, dpool, None, w.softmax_scale, seq_lens=sl,
                          block_table=bt, sinks=dev(w.sinks.astype(np.float32)),
                          rope_tail=w.rope_tail, rope_theta=w.rope_theta, num_splits=2, err_flag=err)
    ops.mla_combine(call)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # the device-written entries are the oracle's float32-decision entries
    want = v41.fp4_cache_append(stale, w.block_table, lens, last.astype(np.float64), 64,
                                w.rope_tail, w.rope_theta, decide_in_f32=True)
    assert np.array_equal(dpool.cpu().numpy(), want)
    ent = np.zeros((w.B, w.Lk, 288), np.uint8)
    for b in range(w.B):
        for t in range(int(lens[b])):
            ent[b, t] = want[w.block_table[b, t // 64], t % 64]
    ref = oracle_shared_latent(w, ent)
    assert_close(call.x.float().cpu().numpy(), ref["x"], TOL_BF16, "x", REL_L2_BF16)
    assert_close(call.lse.cpu().numpy(), ref["lse"], TOL_LSE_BF16, "lse")
