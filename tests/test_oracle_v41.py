"""Pins of the shared-latent (V4.1) oracle: FP4/E4M3 formats, quantiser, RoPE, sink.

CPU only. The E4M3 table is checked against torch's float8_e4m3fn
conversion (a library routine), the E2M1 table against the OCP MX value set,
RoPE against complex multiplication, and the sink against a closed form.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import mla, v41
from latent_kv_decode_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e4m3_all_256_codes_match_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ours = v41.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.all(both_nan | (ours == ref))
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF]) and ours[0x7E] == 448.0


def test_e2m1_all_16_codes_match_ocp_table():
    g = json.load(open(os.path.join(GOLDEN, "e2m1_values.json")))
    ours = v41.e2m1_decode(np.arange(16))
    assert np.array_equal(ours, np.array(g["values"]))
    assert np.array_equal(np.signbit(ours), np.signbit(np.array(g["values"])))


def test_e2m1_quantiser_nearest_even_ties_and_saturation():
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 100.0, -0.26, -2.6, 0.0])
    vals = v41.e2m1_decode(v41.e2m1_quantize(x))
    assert np.array_equal(vals, [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, -0.5, -3.0, 0.0])


def test_e4m3_quantiser_roundtrips_every_finite_code():
    codes = np.arange(0x7F, dtype=np.uint8)
    assert np.array_equal(v41.e4m3_quantize(v41.e4m3_decode(codes)), codes)
    assert v41.e4m3_quantize(np.array([1e6]))[0] == 0x7E


def test_entry_layout_nibbles_and_scales():
    g = json.load(open(os.path.join(GOLDEN, "fp4_entry_bytes.json")))
    D = g["latent_dims"]
    assert g["entry_bytes"] == D // 2 + D // g["channels_per_scale"] == v41.ENTRY_BYTES
    ent = np.zeros(v41.ENTRY_BYTES, np.uint8)
    ent[0] = 0x3 | (0xA << 4)          # channel 0 -> code 3 (1.5), channel 1 -> code 10 (-1.0)
    ent[255] = 0x7 << 4                 # channel 511 -> code 7 (6.0)
    ent[256] = 0x38                     # scale of channels 0..15 = 1.0
    ent[256 + 31] = 0x40                # scale of channels 496..511 = 2.0
    v = v41.fp4_dequant(ent)
    assert v[0] == 1.5 and v[1] == -1.0 and v[511] == 12.0
    assert np.all(v[2:511] == 0.0)


def test_cache_bytes_do_not_depend_on_head_count():
    lat = np.random.default_rng(0).standard_normal((2, 16, 512))
    entries = v41.cache_write(lat)
    assert entries.nbytes == 2 * 16 * 288
    for H in (8, 64, 128):
        w = wl.make_shared_latent(2, H, 1, 16, seed=1)
        assert v41.cache_write(w.latent).nbytes == entries.nbytes


def test_fp4_roundtrip_within_format_bound():
    """|dequant(quant(x)) - x| <= half the E2M1 spacing at |x|, times the group scale, plus scale rounding."""
    lat = np.random.default_rng(1).standard_normal((64, 512))
    deq = v41.fp4_dequant(v41.fp4_quantize(lat))
    g = lat.reshape(64, 32, 16)
    amax = np.abs(g).max(-1, keepdims=True)
    # the E4M3 scale is within 1/16 relative of amax/6; E2M1's largest gap (4->6) is 2
    bound = np.broadcast_to(1.0 * amax / 6.0 * (1 + 1 / 16), g.shape).reshape(64, 512) + 1e-12
    err = np.abs(deq - lat)
    assert np.all(err <= bound)
    rel = np.linalg.norm(deq - lat) / np.linalg.norm(lat)
    assert rel < 0.2


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 512))
    pos = np.array([0, 1, 7, 1000, 8191], float)
    y = v41.rope_tail(x, pos)
    j = np.arange(32)
    z = (x[:, 448::2] + 1j * x[:, 449::2]) * np.exp(1j * pos[:, None] * 10000.0 ** (-j / 32.0))
    assert np.allclose(y[:, 448::2], z.real, atol=1e-12)
    assert np.allclose(y[:, 449::2], z.imag, atol=1e-12)
    assert np.array_equal(y[:, :448], x[:, :448])
    assert np.array_equal(y[0], x[0])


def test_rope_roundtrip_and_relative_position():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal((2, 512))
    for m, n in [(5, 2), (100, 37), (8191, 0)]:
        lhs = v41.rope_tail(q, np.array(m)) @ v41.rope_tail(k, np.array(n))
        rhs = v41.rope_tail(q, np.array(m - n)) @ k
        assert math.isclose(lhs, rhs, rel_tol=1e-10, abs_tol=1e-10)
    x = rng.standard_normal((3, 512))
    p = np.array([3.0, 999.0, 8191.0])
    back = v41.rope_tail(v41.rope_tail(x, p), p, inverse=True)
    assert np.allclose(back, x, atol=1e-12)


def test_sink_closed_form_with_uniform_logits():
    """q = 0: all n visible logits are 0, so p_sink = e^s/(e^s+n) and x = (n/(e^s+n)) * mean."""
    w = wl.make_shared_latent(2, 4, 1, 16, seed=5, seq_lens=[16, 9])
    q = np.zeros_like(w.q)
    ent = v41.cache_write(w.latent)
    lat = v41.fp4_dequant(ent)
    r = v41.shared_latent_decode(q, ent, w.sinks, w.softmax_scale, w.seq_lens, tail=0,
                                 return_all=True)
    for b, n in enumerate([16, 9]):
        mean = lat[b, :n].mean(0)
        for h in range(4):
            es = math.exp(float(w.sinks[h]))
            assert np.allclose(r["x"][b, h, 0], n / (es + n) * mean, atol=1e-13)
            assert math.isclose(r["attn"][b, h, 0, :n].sum(), n / (es + n), rel_tol=1e-12)
            assert math.isclose(float(r["lse"][b, h, 0]), math.log(es + n), rel_tol=1e-12)


def test_shared_latent_decode_inverse_rope_position():
    """A single visible token t = L-1 gives x = inverse-RoPE(v_t, L-1) = dequantised unrotated tail."""
    w = wl.make_shared_latent(1, 2, 1, 12, seed=6)
    ent = v41.cache_write(w.latent)
    mask = np.zeros(12, np.uint8)
    mask[11] = 1
    x = v41.shared_latent_decode(w.q, ent, None, w.softmax_scale, causal_mask=mask)
    v = v41.fp4_dequant(ent[0, 11])
    expect = v41.rope_tail(v, np.array(11.0), inverse=True)
    assert np.allclose(x[0, 0, 0], expect, atol=1e-13)
    # the dequantised, un-rotated tail is close to the raw latent (FP4 error only)
    assert np.linalg.norm(expect - w.latent[0, 11]) / np.linalg.norm(w.latent[0, 11]) < 0.2


def test_shared_latent_paged_equals_contiguous():
    lens = np.array([70, 129, 5])
    w = wl.make_shared_latent(3, 4, 1, 129, seed=7, seq_lens=lens, paged=True)
    ent = v41.cache_write(w.latent)
    ps = w.page_size
    pool = np.zeros((w.block_table.max() + 1, ps, 288), np.uint8)
    for b in range(3):
        for t in range(lens[b]):
            pool[w.block_table[b, t // ps], t % ps] = ent[b, t]
    a = v41.shared_latent_decode(w.q, ent, w.sinks, w.softmax_scale, lens)
    p = v41.shared_latent_decode(w.q, pool, w.sinks, w.softmax_scale, lens,
                                 block_table=w.block_table, page_size=ps)
    assert np.allclose(a, p, atol=1e-14)


def test_sink_enters_split_merge_once():
    rng = np.random.default_rng(8)
    O = rng.standard_normal((3, 1, 2, 1, 4))
    lse = rng.standard_normal((3, 1, 2, 1))
    sinks = np.array([0.5, -1.0])
    x, L = mla.combine_partials(O, lse, sinks)
    for h in range(2):
        den = np.exp(lse[:, 0, h, 0]).sum() + math.exp(sinks[h])
        expect = (np.exp(lse[:, 0, h, 0])[:, None] * O[:, 0, h, 0]).sum(0) / den
        assert np.allclose(x[0, h, 0], expect, atol=1e-14)
        assert math.isclose(float(L[0, h, 0]), math.log(den), rel_tol=1e-12)


def test_e2m1_quantize_keeps_the_sign_of_a_value_rounding_to_zero():
    # a conversion rounds the magnitude and keeps the sign: -0.1 -> -0 (code 8)
    assert list(v41.e2m1_quantize(np.array([-0.1, 0.1, -0.0, 0.0]))) == [8, 0, 8, 0]


# ----------------------------------------------------------------------------- grouped W_O
def _wo_case(seed=0, B=2, H=8, Q=2, C=6, G=4, R=3, D=5):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B, H, Q, C)), r.standard_normal((G, R, (H // G) * C)),
            r.standard_normal((D, G * R)))


def _block_diag(blocks):
    rows = sum(b.shape[0] for b in blocks)
    cols = sum(b.shape[1] for b in blocks)
    out = np.zeros((rows, cols))
    i = j = 0
    for b in blocks:
        out[i:i + b.shape[0], j:j + b.shape[1]] = b
        i += b.shape[0]
        j += b.shape[1]
    return out


def wo_dense_reference(x, wo_a, wo_b):
    """The grouped factors as one dense map on the heads laid side by side."""
    B, H, Q, C = x.shape
    W = _block_diag(list(wo_a))                        # (G*R, H*C), group g on heads gH/G..
    if wo_b is not None:
        W = wo_b @ W
    flat = np.transpose(x, (0, 2, 1, 3)).reshape(B, Q, H * C)
    return flat @ W.T


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_grouped_wo_equals_dense_blockdiag_map(G):
    x, wa, wb = _wo_case(G=G, R=3)
    assert np.allclose(v41.grouped_wo(x, wa, wb), wo_dense_reference(x, wa, wb), rtol=1e-12, atol=1e-12)
    assert np.allclose(v41.grouped_wo(x, wa), wo_dense_reference(x, wa, None), rtol=1e-12, atol=1e-12)


def test_grouped_wo_one_hot_selects_the_weight_column():
    # a single nonzero x[b, h, q, c] = 1 picks column (h mod H/G)*C + c of group h // (H/G)
    B, H, Q, C, G, R, D = 2, 8, 2, 6, 4, 3, 5
    _, wa, wb = _wo_case(B=B, H=H, Q=Q, C=C, G=G, R=R, D=D)
    for (b, h, q, c) in [(0, 0, 0, 0), (1, 5, 1, 4), (0, 7, 1, 5), (1, 2, 0, 3)]:
        x = np.zeros((B, H, Q, C))
        x[b, h, q, c] = 1.0
        g, j = h // (H // G), h % (H // G)
        z = np.zeros(G * R)
        z[g * R:(g + 1) * R] = wa[g][:, j * C + c]
        y = v41.grouped_wo(x, wa, wb)
        others = np.ones((B, Q), bool)
        others[b, q] = False
        assert np.all(y[others] == 0.0)                          # exactly: no other (b, q) is touched
        assert np.allclose(y[b, q], wb @ z, rtol=1e-14, atol=1e-14)
        assert np.array_equal(v41.grouped_wo(x, wa)[b, q], z)   # the selected column itself


def test_grouped_wo_groups_are_isolated():
    x, wa, _ = _wo_case()
    H, G, R = x.shape[1], wa.shape[0], wa.shape[1]
    x2 = x.copy()
    x2[:, 2 * (H // G):3 * (H // G)] += 1.0            # only group 2's heads change
    z1, z2 = v41.grouped_wo(x, wa), v41.grouped_wo(x2, wa)
    changed = np.any(z1 != z2, axis=(0, 1))
    assert np.all(changed[2 * R:3 * R]) and not np.any(np.delete(changed, np.s_[2 * R:3 * R]))


def test_grouped_wo_special_cases():
    # one group: a plain low-rank product of the flattened heads
    x, wa, wb = _wo_case(G=1, R=4)
    flat = np.transpose(x, (0, 2, 1, 3)).reshape(x.shape[0], x.shape[2], -1)
    assert np.allclose(v41.grouped_wo(x, wa, wb), (flat @ wa[0].T) @ wb.T, rtol=1e-12, atol=1e-12)
    # one head per group: z_h = wo_a[h] x_h, per head
    x, wa, _ = _wo_case(H=4, G=4, R=3)
    z = v41.grouped_wo(x, wa)
    for h in range(4):
        assert np.allclose(z[:, :, 3 * h:3 * h + 3], np.einsum("rc,bqc->bqr", wa[h], x[:, h]),
                           rtol=1e-12, atol=1e-12)
