"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each case monkeypatches one oracle function with a plausible bug and checks
that an independent pin from test_oracle_mla / test_oracle_v41 now fails.
"""
import math

import numpy as np
import pytest

from oracle import mla, v41


def _tiny(seed=0, B=2, H=3, Q=2, Dn=4, Dr=3, Vd=5, Ckv=6, Lk=7):
    r = np.random.default_rng(seed)
    return dict(q_nope=r.standard_normal((B, H, Q, Dn)), q_pe=r.standard_normal((B, H, Q, Dr)),
                kv_cache=r.standard_normal((B, Lk, Ckv)), pe_cache=r.standard_normal((B, Lk, Dr)),
                wkv_b=r.standard_normal((H, Dn + Vd, Ckv)), softmax_scale=1.0 / math.sqrt(Dn + Dr))


def _absorbed_vs_naive(t, causal=True):
    B, H, Q, _ = t["q_nope"].shape
    Lk = t["kv_cache"].shape[1]
    seq_lens = np.array([Lk, Lk - 2])
    vis = mla.visibility(B, Q, Lk, seq_lens, None, causal)
    naive = mla.naive_decompressed_mha(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"],
                                       t["wkv_b"], t["softmax_scale"], vis)
    ab = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                             t["softmax_scale"], None, seq_lens, causal)
    return np.allclose(ab, naive, rtol=1e-10, atol=1e-12)


def test_unmutated_oracle_passes():
    assert _absorbed_vs_naive(_tiny())


def test_dropped_position_term_is_caught(monkeypatch):
    orig = mla.latent_scores
    monkeypatch.setattr(mla, "latent_scores", lambda ql, qp, kv, pe: orig(ql, None, kv, pe))
    assert not _absorbed_vs_naive(_tiny())


def test_wrong_weight_slice_is_caught(monkeypatch):
    def bad_split(wkv_b, Dn):
        w = np.asarray(wkv_b, float)
        Vd = w.shape[1] - Dn
        return w[:, :Dn, :], w[:, :Vd, :]          # W_UV taken from the first rows
    monkeypatch.setattr(mla, "split_wkv_b", bad_split)
    assert not _absorbed_vs_naive(_tiny())


def test_transposed_up_projection_is_caught(monkeypatch):
    # square per-head weights so that the transposed contraction is shape-valid
    t = _tiny(Dn=4, Vd=6, Ckv=6)

    def bad_up(x, wkv_b, Dn):
        _, w_uv = mla.split_wkv_b(wkv_b, Dn)
        return np.einsum("bhqc,hcv->bhqv", np.asarray(x, float), w_uv)
    monkeypatch.setattr(mla, "up_proj", bad_up)
    assert not _absorbed_vs_naive(t)


def test_missing_scale_is_caught(monkeypatch):
    orig = mla.latent_attention
    monkeypatch.setattr(mla, "latent_attention",
                        lambda ql, qp, kv, pe, sc, vis, sinks=None: orig(ql, qp, kv, pe, 1.0, vis, sinks))
    assert not _absorbed_vs_naive(_tiny())


def test_causal_off_by_one_is_caught(monkeypatch):
    orig = mla.visibility

    def bad_vis(B, Q, Lk, seq_lens=None, causal_mask=None, causal=False):
        v = orig(B, Q, Lk, seq_lens, causal_mask, False)
        if causal:
            t = np.arange(Lk)
            L = np.full(B, Lk) if seq_lens is None else np.asarray(seq_lens)
            last = L[:, None] - Q + np.arange(Q)[None, :] - 1       # one too few
            v &= t[None, None, :] <= last[:, :, None]
        return v
    t = _tiny(Lk=9)
    seq_lens = np.array([9, 7])
    good = mla.mla_decode_step(t["q_nope"][:, :, 1:], t["q_pe"][:, :, 1:], t["kv_cache"],
                               t["pe_cache"], t["wkv_b"], t["softmax_scale"], None, seq_lens)
    monkeypatch.setattr(mla, "visibility", bad_vis)
    r2 = mla.mla_decode_step(t["q_nope"], t["q_pe"], t["kv_cache"], t["pe_cache"], t["wkv_b"],
                             t["softmax_scale"], None, seq_lens, causal=True)
    assert not np.allclose(r2[:, :, 1], good[:, :, 0], rtol=1e-12, atol=1e-14)


def test_unnormalised_merge_is_caught():
    O = np.stack([np.full((1, 1, 1, 3), 2.0), np.full((1, 1, 1, 3), -1.0)])
    lse = np.array([math.log(3.0), 0.0]).reshape(2, 1, 1, 1)
    w = np.exp(lse)                                   # forgetting to divide by e^L
    bad = (w[..., None] * O).sum(0)
    good, _ = mla.combine_partials(O, lse)
    assert not np.allclose(bad, good)


def test_swapped_nibbles_are_caught():
    """Reading channel 2i from the high nibble decodes a different vector."""
    ent = np.zeros(v41.ENTRY_BYTES, np.uint8)
    ent[0] = 0x3 | (0xA << 4)
    ent[256] = 0x38
    good = v41.fp4_dequant(ent)
    swapped = ent.copy()
    swapped[0] = 0xA | (0x3 << 4)
    assert not np.array_equal(v41.fp4_dequant(swapped), good)
    assert good[0] == 1.5 and good[1] == -1.0


def test_wrong_rope_frequency_is_caught():
    x = np.random.default_rng(2).standard_normal((1, 512))
    pos = np.array([7.0])
    j = np.arange(32)
    z = (x[:, 448::2] + 1j * x[:, 449::2]) * np.exp(1j * pos[:, None] * 10000.0 ** (-j / 32.0))
    bad = v41.rope_tail(x, pos, theta=500000.0)
    assert not np.allclose(bad[:, 448::2], z.real, atol=1e-12)


def _fp4_appends_match_cache_write(append):
    r = np.random.default_rng(5)
    lat = r.standard_normal((1, 12, 512))
    bt = np.array([[1, 0]], np.int32)
    pool = np.zeros((2, 64, 288), np.uint8)
    for t in range(12):
        pool = append(pool, bt, np.array([t + 1]), lat[:, t:t + 1], 64)
    return np.array_equal(pool[1, :12], v41.cache_write(lat)[0])


def test_unmutated_fp4_append_passes():
    assert _fp4_appends_match_cache_write(v41.fp4_cache_append)


def test_append_position_off_by_one_is_caught():
    def bad_append(pool, block_table, seq_lens, latent_new, page_size=64, tail=64, theta=10000.0):
        lat = np.asarray(latent_new, float)
        B, Q, D = lat.shape
        pos = np.asarray(seq_lens)[:, None] - Q + np.arange(Q)[None, :] + 1   # the slot's position + 1
        ent = v41.fp4_quantize(v41.rope_tail(lat, pos.astype(float), tail, theta), D)
        return mla.cache_append(pool, block_table, seq_lens, ent, page_size)
    assert not _fp4_appends_match_cache_write(bad_append)


def test_append_slot_off_by_one_is_caught(monkeypatch):
    def bad_cache_append(pool, block_table, seq_lens, rows, page_size):
        out = np.array(pool, copy=True)
        r = np.asarray(rows)
        for b in range(r.shape[0]):
            for i in range(r.shape[1]):
                t = int(seq_lens[b]) - r.shape[1] + i + 1          # writes one slot late
                out[int(block_table[b][t // page_size]), t % page_size] = r[b, i]
        return out
    monkeypatch.setattr(mla, "cache_append", bad_cache_append)
    assert not _fp4_appends_match_cache_write(v41.fp4_cache_append)


def test_interleaved_head_groups_are_caught(monkeypatch):
    # heads assigned to groups round-robin (h mod G) instead of in contiguous runs
    from test_oracle_v41 import _wo_case, wo_dense_reference
    orig = v41.grouped_wo

    def bad(x, wo_a, wo_b=None):
        G = np.asarray(wo_a).shape[0]
        H = np.asarray(x).shape[1]
        perm = np.concatenate([np.arange(g, H, G) for g in range(G)])
        return orig(np.asarray(x)[:, perm], wo_a, wo_b)
    monkeypatch.setattr(v41, "grouped_wo", bad)
    x, wa, wb = _wo_case(G=4)
    assert not np.allclose(v41.grouped_wo(x, wa, wb), wo_dense_reference(x, wa, wb))


def test_query_major_stacking_is_caught(monkeypatch):
    # a group's heads stacked dim-major (c, h) instead of head-major (h, c)
    from test_oracle_v41 import _wo_case, wo_dense_reference

    def bad(x, wo_a, wo_b=None):
        xx = np.asarray(x, float)
        B, H, Q, C = xx.shape
        wa = np.asarray(wo_a, float)
        G, R, K = wa.shape
        z = np.zeros((B, Q, G * R))
        for g in range(G):
            u = np.transpose(xx[:, g * (H // G):(g + 1) * (H // G)], (0, 2, 3, 1)).reshape(B, Q, K)
            z[:, :, g * R:(g + 1) * R] = u @ wa[g].T
        return z if wo_b is None else z @ np.asarray(wo_b, float).T
    monkeypatch.setattr(v41, "grouped_wo", bad)
    x, wa, wb = _wo_case(G=2)
    assert not np.allclose(v41.grouped_wo(x, wa, wb), wo_dense_reference(x, wa, wb))
