"""fp64 oracle of the shared-latent MLA variant (test infrastructure only).

Source: openarchlab DeepSeek-V4.1-Flash course page "4A · Multi-head Latent
Attention · latent K/V dùng chung, RoPE nửa sau và W_O nhóm":

- §1 Định nghĩa: every head reads one shared 512-dim latent per cache entry,
  which serves as both K and V; RoPE rotates only the tail of the latent; an
  entry takes 288 B of K/V in the FP4 budget.
- §2 Luồng: 64 query heads of 512 dims against the single latent, sparse
  attention with an attn_sink score column, inverse RoPE on the output, then
  the grouped output projection "Group-LoRA W_O (8 nhóm × 1024)" back to
  [B, T, D_model] (``grouped_wo``);
- §3 W_O nhóm: the output projection works per group of heads: each group
  merges its own heads' outputs with its own small matrix, and the groups'
  results are put side by side, instead of one large matrix.
- §4 Profiling: FP4 latent with one E4M3 scale per 16 channels checked
  against the fp32 latent; RoPE on the tail checked by hand and undone by the
  inverse; cache bytes independent of the number of query heads.

Readings where the pages leave a step open:

- entry layout, 288 B = 256 B of E2M1 codes + 32 E4M3 scales: byte i holds
  channel 2i in its low nibble and channel 2i+1 in its high nibble; byte
  256+g is the scale of channels 16g..16g+15;
- E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0;
  E4M3 (the "fn" variant): sign bit 7, exponent bits 6..3 (bias 7),
  mantissa bits 2..0, S.1111.111 = NaN, no infinities, max 448;
- quantiser of the cache-write step (input preparation; decode parity does
  not depend on it): scale_g = E4M3(amax_g / 6) rounded to nearest-even,
  code = E2M1(x / scale_g) rounded to nearest-even with saturation at 6
  and x's sign kept (-0 for a small negative x), zero codes when scale_g = 0;
- RoPE on the last ``tail`` = 64 dims as interleaved pairs (D-tail+2j,
  D-tail+2j+1), j = 0..tail/2-1, angle = pos * theta^(-2j/tail), theta =
  10000; cache rows are rotated at their token position before
  quantisation; q arrives already rotated; the output's tail is rotated back
  by the query position L_b - Q + i;
- softmax_scale = 1/sqrt(512); the sink is a raw logit (not scaled) that
  enters each (b,h,q) denominator once and contributes no value;
- grouped W_O ("8 nhóm × 1024", the group shapes are garbled on the page):
  G = 8 groups of H/G consecutive heads; group g stacks its heads' inverse-
  rotated outputs head-major into u_g of (H/G)*512 values and applies its own
  low-rank factor wo_a[g] (R x (H/G)*512, R = 1024) to give z_g; the z_g are
  concatenated g-major into z of G*R values ("ghép lại"), and the shared
  factor wo_b (D x G*R) maps z to the model width D ("phân rã", "về lại
  [B, T, D_model]"). D_model is not on the pages (4096 is the synthetic
  choice); without wo_b the output is z itself.

Pins (tests/test_oracle_v41.py): the grouped W_O against one dense matrix
wo_b . blockdiag(wo_a[0..G-1]) on the flattened heads, one-hot inputs
against the selected weight columns, group isolation, and the one-group
and one-head-per-group special cases; all 256 E4M3 codes against torch's
float8_e4m3fn conversion; the 16 E2M1 codes against the OCP MX E2M1 value
set (tests/golden/e2m1_values.json); nearest-even ties of the quantiser;
FP4 round-trip error bound on N(0,1) latents; 288 B per entry and cache
bytes independent of H; RoPE against complex multiplication by
e^{i pos theta_j}, relative-position property, identity at pos 0, round trip
and untouched head dims; the sink's closed form with uniform logits;
token-by-token FP4 appends equal cache_write of the whole sequence.
"""
from __future__ import annotations

import numpy as np

from . import mla as _mla

F64 = np.float64
ENTRY_BYTES = 288          # 512 x 4-bit codes + 32 E4M3 scales
GROUP = 16                 # channels per E4M3 scale


def e2m1_decode(codes):
    """Value of each 4-bit E2M1 code (0..15) as float64."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = (c & 0x1).astype(F64)
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2((e - 1).astype(F64)))
    return sign * mag


def e4m3_decode(b):
    """Value of each E4M3 (fn) byte as float64 (0x7F / 0xFF -> NaN)."""
    c = np.asarray(b, dtype=np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(F64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(F64)))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def fp4_dequant(entries, D: int = 512):
    """Decode (..., 288) uint8 entries to (..., 512) float64: v[c] = E2M1(code[c]) * E4M3(scale[c//16])."""
    ent = np.asarray(entries, dtype=np.uint8)
    nb = D // 2
    codes = ent[..., :nb]
    lo = e2m1_decode(codes & 0xF)
    hi = e2m1_decode(codes >> 4)
    vals = np.empty(ent.shape[:-1] + (D,))
    vals[..., 0::2] = lo
    vals[..., 1::2] = hi
    sc = e4m3_decode(ent[..., nb:nb + D // GROUP])
    return vals * np.repeat(sc, GROUP, axis=-1)


def _nearest_even(x, grid_vals, grid_codes):
    """Index into a sorted grid of the nearest value; ties go to the even code."""
    x = np.asarray(x, F64)
    idx = np.searchsorted(grid_vals, x)
    idx = np.clip(idx, 1, len(grid_vals) - 1)
    lo, hi = grid_vals[idx - 1], grid_vals[idx]
    dlo, dhi = x - lo, hi - x
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (grid_codes[idx] % 2 == 0))
    out = np.where(pick_hi, idx, idx - 1)
    out = np.where(x <= grid_vals[0], 0, out)
    out = np.where(x >= grid_vals[-1], len(grid_vals) - 1, out)
    return out


def e4m3_quantize(x):
    """Non-negative float64 -> E4M3 byte, nearest-even, saturating at 448."""
    codes = np.arange(0x7F)                       # 0x00..0x7E: all finite non-negative codes
    vals = e4m3_decode(codes)
    return codes[_nearest_even(x, vals, codes)].astype(np.uint8)


def e2m1_quantize(x):
    """float64 -> 4-bit E2M1 code, nearest-even on the magnitude, saturating at 6.

    The sign bit is x's sign, also when the magnitude rounds to 0 (a negative
    value below 0.25 becomes -0), as a floating-point conversion keeps it.
    """
    x = np.asarray(x, F64)
    codes = np.arange(8)
    vals = e2m1_decode(codes)
    mag = codes[_nearest_even(np.abs(x), vals, codes)]
    return np.where(np.signbit(x), mag | 0x8, mag).astype(np.uint8)


def fp4_quantize(latent, D: int = 512, decide_in_f32: bool = False):
    """Cache-write quantiser: (..., 512) float -> (..., 288) uint8 entries.

    scale_g = E4M3(amax_g / 6), code = E2M1(x / scale_g); zero codes where
    scale_g decodes to 0. The pages do not fix the precision of the two
    quotients whose rounding picks the codes; ``decide_in_f32`` takes them
    the way a float32 implementation does: the input rounded to float32, then
    amax / 6 and x / scale_g each correctly rounded in float32 before the
    nearest-even choice (the float64 default rounds only at the choice).
    """
    x = np.asarray(latent, F64)
    if decide_in_f32:
        x = x.astype(np.float32).astype(F64)
    g = x.reshape(x.shape[:-1] + (D // GROUP, GROUP))
    amax = np.abs(g).max(axis=-1)
    if decide_in_f32:
        sbytes = e4m3_quantize((amax.astype(np.float32) / np.float32(6.0)).astype(F64))
    else:
        sbytes = e4m3_quantize(amax / 6.0)
    s = e4m3_decode(sbytes)
    safe = np.where(s > 0, s, 1.0)
    if decide_in_f32:
        q = (g.astype(np.float32) / safe[..., None].astype(np.float32)).astype(F64)
    else:
        q = g / safe[..., None]
    codes = e2m1_quantize(q)
    codes = np.where((s > 0)[..., None], codes, 0).reshape(x.shape).astype(np.uint8)
    out = np.empty(x.shape[:-1] + (ENTRY_BYTES,), np.uint8)
    out[..., :D // 2] = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    out[..., D // 2:] = sbytes
    return out


def rope_tail(x, pos, tail: int = 64, theta: float = 10000.0, inverse: bool = False):
    """Rotate the last ``tail`` dims of x (..., D) by position ``pos`` (broadcast over x[..., 0]).

    Pair j = (D-tail+2j, D-tail+2j+1) turns by angle pos * theta^(-2j/tail)
    (by minus that angle when ``inverse``); the first D-tail dims are copied.
    """
    x = np.asarray(x, F64)
    D = x.shape[-1]
    j = np.arange(tail // 2, dtype=F64)
    freq = theta ** (-2.0 * j / tail)
    ang = np.asarray(pos, F64)[..., None] * freq
    if inverse:
        ang = -ang
    c, s = np.cos(ang), np.sin(ang)
    out = x.copy()
    a = x[..., D - tail + 0::2]
    b = x[..., D - tail + 1::2]
    out[..., D - tail + 0::2] = a * c - b * s
    out[..., D - tail + 1::2] = a * s + b * c
    return out


def cache_write(latent, tail: int = 64, theta: float = 10000.0):
    """Cache-append reference for a (B, Lk, 512) latent: RoPE at positions 0..Lk-1, then FP4."""
    lat = np.asarray(latent, F64)
    Lk = lat.shape[1]
    pos = np.broadcast_to(np.arange(Lk, dtype=F64)[None, :], lat.shape[:2])
    return fp4_quantize(rope_tail(lat, pos, tail, theta))


def fp4_cache_append(pool, block_table, seq_lens, latent_new, page_size: int = 64, tail: int = 64,
                     theta: float = 10000.0, decide_in_f32: bool = False):
    """Shared-latent cache append into a paged pool of 288-byte entries.

    latent_new (B, Q, 512): the new tokens' latents; seq_lens: lengths after
    the append. Each new token's tail is rotated at its position
    seq_lens[b] - Q + i, quantised to an FP4 entry (``decide_in_f32`` as in
    fp4_quantize), and written to its slot (mla.cache_append's addressing):
    the per-token form of cache_write.
    """
    lat = np.asarray(latent_new, F64)
    B, Q, D = lat.shape
    pos = np.asarray(seq_lens, np.int64)[:, None] - Q + np.arange(Q)[None, :]
    ent = fp4_quantize(rope_tail(lat, pos.astype(F64), tail, theta), D, decide_in_f32)
    return _mla.cache_append(pool, block_table, seq_lens, ent, page_size)


def shared_latent_decode(q, entries, sinks, softmax_scale, seq_lens=None, causal: bool = False,
                         causal_mask=None, tail: int = 64, theta: float = 10000.0,
                         block_table=None, page_size: int = 64, return_all: bool = False):
    """Decode with K = V = dequantised shared latent, a sink per head and inverse RoPE.

    q (B,H,Q,512) already rotated; entries (B,Lk,288) uint8, or a paged pool
    (num_pages, page_size, 288) with ``block_table``. Logits q . k_t *
    softmax_scale; the softmax denominator adds exp(sink_h); x = sum_t p_t v_t;
    then x's tail is rotated back by the query position L_b - Q + i.
    """
    qq = np.asarray(q, F64)
    B, H, Q, D = qq.shape
    if block_table is not None:
        lens = np.asarray(seq_lens, np.int64)
        lat = _mla.gather_paged(fp4_dequant(entries, D), block_table, lens, page_size)
    else:
        lat = fp4_dequant(entries, D)
    Lk = lat.shape[1]
    vis = _mla.visibility(B, Q, Lk, seq_lens, causal_mask, causal)
    x, attn, lse = _mla.latent_attention(qq, None, lat, None, softmax_scale, vis, sinks)
    L = np.full(B, Lk, np.int64) if seq_lens is None else np.asarray(seq_lens, np.int64)
    pos = (L[:, None] - Q + np.arange(Q)[None, :])                 # (B,Q)
    pos = np.broadcast_to(pos[:, None, :], (B, H, Q))
    if tail:
        x = rope_tail(x, pos, tail, theta, inverse=True)
    if return_all:
        return dict(x=x, attn=attn, lse=lse, latent=lat, vis=vis)
    return x


def grouped_wo(x, wo_a, wo_b=None):
    """Grouped low-rank output projection (4A §2 Luồng, §3 W_O nhóm).

    x (B,H,Q,C) inverse-rotated attention output; wo_a (G,R,(H/G)*C): group
    g's own factor; wo_b (D,G*R) or None. Returns (B,Q,D), or (B,Q,G*R) when
    wo_b is None: for every (b,q), u_g = x[b, gH/G:(g+1)H/G, q, :] flattened
    head-major, z_g = wo_a[g] u_g, z = [z_0, ..., z_{G-1}], y = wo_b z.
    """
    xx = np.asarray(x, F64)
    wa = np.asarray(wo_a, F64)
    B, H, Q, C = xx.shape
    G, R, K = wa.shape
    assert H % G == 0 and K == (H // G) * C
    z = np.zeros((B, Q, G * R), F64)
    for g in range(G):
        heads = xx[:, g * (H // G):(g + 1) * (H // G), :, :]          # (B,H/G,Q,C)
        u = np.transpose(heads, (0, 2, 1, 3)).reshape(B, Q, K)        # head-major
        z[:, :, g * R:(g + 1) * R] = u @ wa[g].T
    if wo_b is None:
        return z
    return z @ np.asarray(wo_b, F64).T
