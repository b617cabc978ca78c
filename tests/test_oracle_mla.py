"""Pins of the absorbed-MLA oracle against facts that do not come from the oracle itself.

CPU only. Every test here would fail for a plausible mistake in oracle/mla.py
(a dropped score term, a wrong weight slice, a transposed operand, a missing
scale, a wrong causal offset, a wrong merge weight).
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import mla
from latent_kv_decode_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _tiny(seed=0, B=2, H=3, Q=2, Dn=4, Dr=3, Vd=5, Ckv=6, Lk=7):
    r = _rng(seed)
    return dict(q_nope=r.standard_normal((B, H, Q, Dn)), q_pe=r.standard_normal((B, H, Q, Dr)),
                kv_cache=r.standard_normal((B, Lk, Ckv)), pe_cache=r.standard_normal((B, Lk, Dr)),
                wkv_b=r.standard_normal((H, Dn + Vd, Ckv)), softmax_scale=1.0 / math.sqrt(Dn + Dr))


def test_demo_output_shape_matches_printed_shape():
    g = json.load(open(os.path.join(GOLDEN, "demo_output_shape.json")))
    w = wl.demo_fp32()
    assert (w.B, w.H, w.Q, w.Dn, w.Dr, w.Vd, w.Lk, w.Ckv) == tuple(
        g["inputs"][k] for k in ("B", "H", "Q", "Dn", "Dr", "Vd", "Lk", "Ckv"))
    out = mla.mla_decode_step(w.q_nope, w.q_pe, w.kv_cache, w.pe_cache, w.wkv_b,
                              w.softmax_scale, w.causal_mask)
    assert list(out.shape) == g["out_shape"]
    assert np.all(np.isfinite(out))


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("causal", [False, True])
def test_absorbed_equals_naive_decompressed(seed, causal):
    t = _tiny(seed)
    B, H, Q, Dn = t["q_nope"].shape
    Lk = t["kv_cache"].shape[1]
    seq_lens = np.array([Lk, Lk - 2])
    mask = np.ones(Lk, np.uint8)
    mask[1] = 0
    vis = mla.visibility(B, Q, Lk, seq_lens, mask, causal)
    naive = mla.naive_decompressed_mha(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"],
                                       t["wkv_b"], t["softmax_scale"], vis)
    absorbed = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                                   t["softmax_scale"], mask, seq_lens, causal)
    assert np.allclose(absorbed, naive, rtol=1e-10, atol=1e-12)


def test_absorbed_equals_naive_on_demo_workload():
    w = wl.demo_fp32()
    vis = mla.visibility(w.B, w.Q, w.Lk, None, w.causal_mask, False)
    naive = mla.naive_decompressed_mha(w.q_nope, w.q_pe, w.kv_cache, w.pe_cache, w.wkv_b,
                                       w.softmax_scale, vis)
    absorbed = mla.mla_decode_step(w.q_nope, w.q_pe, w.kv_cache, w.pe_cache, w.wkv_b,
                                   w.softmax_scale, w.causal_mask)
    assert np.allclose(absorbed, naive, rtol=1e-10, atol=1e-10)


def test_softmax_rows_sum_to_one_and_masked_weights_are_zero():
    t = _tiny(3, Lk=9)
    B, H, Q, _ = t["q_nope"].shape
    mask = np.array([1, 0, 1, 1, 0, 1, 1, 1, 1], np.uint8)
    r = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                            t["softmax_scale"], mask, np.array([9, 6]), True, return_all=True)
    attn, vis = r["attn"], r["vis"]
    assert np.allclose(attn.sum(-1), 1.0, atol=1e-12)
    hidden = ~np.broadcast_to(vis[:, None], attn.shape)
    assert np.all(attn[hidden] == 0.0)
    assert np.all(attn[~hidden] > 0.0)


def test_single_visible_token_returns_that_row_exactly():
    t = _tiny(4, Lk=8)
    mask = np.zeros(8, np.uint8)
    mask[5] = 1
    r = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                            t["softmax_scale"], mask, return_all=True)
    x = r["x"]
    for b in range(x.shape[0]):
        assert np.array_equal(x[b], np.broadcast_to(t["kv_cache"][b, 5], x[b].shape))


def test_zero_query_gives_mean_of_visible_rows():
    t = _tiny(5, Lk=8)
    t["q_nope"][:] = 0
    t["q_pe"][:] = 0
    seq_lens = np.array([8, 5])
    r = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                            t["softmax_scale"], None, seq_lens, return_all=True)
    for b, L in enumerate(seq_lens):
        mean = t["kv_cache"][b, :L].mean(axis=0)
        assert np.allclose(r["x"][b], mean, atol=1e-14)


def test_single_token_cache_closed_form():
    """Lk = 1: the softmax is 1, so out[b,h] = W_UV[h] @ kv[b,0] whatever q is."""
    t = _tiny(6, Lk=1)
    out = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                              t["softmax_scale"])
    Dn = t["q_nope"].shape[-1]
    W = t["wkv_b"]
    for b in range(out.shape[0]):
        for h in range(out.shape[1]):
            expect = W[h, Dn:] @ t["kv_cache"][b, 0]
            assert np.allclose(out[b, h], expect[None, :], atol=1e-13)


def test_weight_split_rows():
    """Rows [0,Dn) of wkv_b act only on scores, the last Vd rows only on the output.

    Zeroing W_UK and q_pe leaves uniform weights (out = W_UV @ mean kv);
    zeroing W_UV zeroes the output; changing W_UK changes the output.
    """
    t = _tiny(7, Lk=6)
    Dn = t["q_nope"].shape[-1]
    w = t["wkv_b"].copy()
    w[:, :Dn] = 0
    qpe0 = np.zeros_like(t["q_pe"])
    out = mla.mla_decode_step(t["q_nope"], qpe0, t["kv_cache"], t["pe_cache"], w, t["softmax_scale"])
    for b in range(out.shape[0]):
        for h in range(out.shape[1]):
            assert np.allclose(out[b, h], (w[h, Dn:] @ t["kv_cache"][b].mean(0))[None], atol=1e-13)
    w2 = t["wkv_b"].copy()
    w2[:, Dn:] = 0
    out2 = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], w2,
                               t["softmax_scale"])
    assert np.all(out2 == 0)


def test_scale_multiplies_the_merged_score():
    """With one visible pair of tokens the weight ratio is exp(scale * (s0 - s1))."""
    t = _tiny(8, Lk=2)
    r = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                            t["softmax_scale"], return_all=True)
    # raw scores by explicit loops over the projected query, independent of einsum
    Dn = t["q_nope"].shape[-1]
    b, h, q = 1, 2, 1
    Wk = t["wkv_b"][h, :Dn]
    ql = sum(t["q_nope"][b, h, q, d] * Wk[d] for d in range(Dn))
    s = [float(ql @ t["kv_cache"][b, j] + t["q_pe"][b, h, q] @ t["pe_cache"][b, j]) for j in range(2)]
    a = r["attn"][b, h, q]
    assert math.isclose(a[0] / a[1], math.exp(t["softmax_scale"] * (s[0] - s[1])), rel_tol=1e-12)


def test_causal_query_zero_equals_shorter_single_query_decode():
    t = _tiny(9, Q=2, Lk=9)
    seq_lens = np.array([9, 7])
    r2 = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                             t["softmax_scale"], None, seq_lens, causal=True)
    r1 = mla.mla_decode_step(t["q_nope"][:, :, :1], t["q_pe"][:, :, :1], t["kv_cache"],
                             t["pe_cache"], t["wkv_b"], t["softmax_scale"], None, seq_lens - 1)
    assert np.allclose(r2[:, :, 0], r1[:, :, 0], rtol=1e-12, atol=1e-14)
    r_last = mla.mla_decode_step(t["q_nope"][:, :, 1:], t["q_pe"][:, :, 1:], t["kv_cache"],
                                 t["pe_cache"], t["wkv_b"], t["softmax_scale"], None, seq_lens)
    assert np.allclose(r2[:, :, 1], r_last[:, :, 0], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("bounds", [[(0, 11)], [(0, 4), (4, 11)], [(0, 3), (3, 3), (3, 8), (8, 11)],
                                    [(0, 5), (5, 11), (11, 11)]])
def test_split_merge_invariance(bounds):
    t = _tiny(10, Q=2, Lk=11)
    B, H, Q, _ = t["q_nope"].shape
    seq_lens = np.array([11, 4])       # second sequence leaves later splits empty
    vis = mla.visibility(B, Q, 11, seq_lens, None, True)
    ql = mla.absorb_q(t["q_nope"], t["wkv_b"])
    full, _, lse_full = mla.latent_attention(ql, t["q_pe"], t["kv_cache"], t["pe_cache"],
                                             t["softmax_scale"], vis)
    O, lse = mla.split_partials(ql, t["q_pe"], t["kv_cache"], t["pe_cache"], t["softmax_scale"],
                                vis, bounds)
    x, L = mla.combine_partials(O, lse)
    assert np.allclose(x, full, rtol=1e-12, atol=1e-14)
    assert np.allclose(L, lse_full, rtol=1e-12)


def test_combine_two_splits_by_hand():
    """Two splits with lse a and b merge with weights e^a/(e^a+e^b) and e^b/(e^a+e^b)."""
    O = np.stack([np.full((1, 1, 1, 3), 2.0), np.full((1, 1, 1, 3), -1.0)])
    lse = np.array([math.log(3.0), math.log(1.0)]).reshape(2, 1, 1, 1)
    x, L = mla.combine_partials(O, lse)
    assert np.allclose(x, 0.75 * 2.0 + 0.25 * -1.0)
    assert math.isclose(float(L.ravel()[0]), math.log(4.0))


def test_paged_gather_equals_contiguous():
    w = wl.make_mla(3, 2, 2, 4, 3, 5, 6, 0, dtype="f32", seed=11, lk_range=(1, 150), paged=True,
                    causal=True)
    # rebuild the contiguous cache row by row from (page, offset) coordinates
    ps = w.page_size
    L = w.lens()
    kv = mla.gather_paged(w.kv_pool, w.block_table, L, ps)
    for b in range(w.B):
        for t in (0, int(L[b]) - 1, int(L[b]) // 2):
            page = w.block_table[b, t // ps]
            assert np.array_equal(kv[b, t], w.kv_pool[page, t % ps])
    used = np.concatenate([w.block_table[b, :(int(L[b]) + ps - 1) // ps] for b in range(w.B)])
    assert sorted(used.tolist()) == list(range(w.kv_pool.shape[0]))


def test_fully_masked_row_is_zero():
    t = _tiny(12, Lk=4)
    mask = np.zeros(4, np.uint8)
    r = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                            t["softmax_scale"], mask, return_all=True)
    assert np.all(r["out"] == 0) and np.all(np.isneginf(r["lse"]))


def test_lse_is_log_of_denominator():
    t = _tiny(13, Lk=5)
    r = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                            t["softmax_scale"], return_all=True)
    ql = r["q_lat"]
    b, h, q = 0, 1, 0
    logits = [t["softmax_scale"] * float(ql[b, h, q] @ t["kv_cache"][b, j] +
                                         t["q_pe"][b, h, q] @ t["pe_cache"][b, j]) for j in range(5)]
    assert math.isclose(float(r["lse"][b, h, q]), math.log(sum(math.exp(v) for v in logits)),
                        rel_tol=1e-12)
