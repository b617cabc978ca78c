"""fp64 oracle of absorbed MLA single-step decode (test infrastructure only).

Source of the method: the exam question "MLA 单步解码" on 6547.cn, whose
``mla_decode_step(q_nope, q_pe, kv_cache, pe_cache, wkv_b, softmax_scale,
causal_mask)`` fixes the shapes and leaves five blanks:

  [1] project q_nope through each head's W_UK slice into the latent space,
  [2] correlate the projected query with kv_cache (scores_nope),
  [3] add the position scores and scale,
  [4] set invisible positions to -inf,
  [5] map the softmax-weighted latent back through each head's W_UV slice.

The blanks are read from the shape comments beside them and the question's
prose (content part projected through head-dependent weights, position part
dotted directly with the position cache, scores merged then scaled, future
positions masked, result mapped back to each head's value space). The same
absorbed score, q_absorbed . c_kv + q_rope . k_rope, is written out in the
comments of ``MultiHeadLatentAttention.forward_inference`` on the neuronix
page "DeepSeek-V3/R1 架构深度全景解析".

Readings where the pages leave a step open:

- weight split: rows [0,Dn) of wkv_b are W_UK and the last Vd rows W_UV,
  Vd = wkv_b.shape[1] - Dn (the question's dimension-preparation lines);
- mask: 1 = visible, 0 = hidden; visible(b,q,t) = mask[t] and t < L_b and,
  for causal speculative decoding with Q new tokens (already appended as the
  last Q cache rows), t <= L_b - Q + q;
- a row with no visible position gets all-zero weights, x = 0, lse = -inf;
- split-KV partials store the normalised partial output O_s and
  lse_s = log sum_t exp(logit_t); they merge by weights exp(lse_s - L) with
  L = log sum_s exp(lse_s) (plus the sink logit when there is one).

Pins (tests/test_oracle_mla.py): demo output shape (2,8,1,128) printed by the
question's demo; equality with the naive decompressed MHA (the
CacheDecompressed form of the ackingliu.top "DeepSeek MLA projection
absorption" article) on tiny inputs; rows of the softmax sum to 1; masked
weights are exactly 0; single-visible-token and zero-query closed forms;
Lk = 1 closed form; W_UK/W_UV row-split closed forms; Q=2 causal prefix
property; split-merge invariance; paged == contiguous. Cache append
(tests/test_oracle_append.py): token-by-token appends read back by
gather_paged equal the rows in order; untouched slots keep their bytes.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def _f64(x):
    return None if x is None else np.asarray(x, dtype=F64)


def split_wkv_b(wkv_b, Dn: int):
    """W_UK = wkv_b[:, :Dn, :] (H,Dn,Ckv), W_UV = wkv_b[:, -Vd:, :] (H,Vd,Ckv).

    "MLA 单步解码" question, mla_decode_step, dimension preparation and weight
    split (k_nope_w, v_w).
    """
    w = _f64(wkv_b)
    Vd = w.shape[1] - Dn
    return w[:, :Dn, :], w[:, w.shape[1] - Vd:, :]


def absorb_q(q_nope, wkv_b):
    """Blank [1]: q_lat[b,h,q,c] = sum_d q_nope[b,h,q,d] * W_UK[h,d,c] -> (B,H,Q,Ckv).

    "MLA 单步解码" question, mla_decode_step step 1); the absorption of W_UK on
    the query side is the associativity step in the comments of
    MultiHeadLatentAttention.forward_inference (neuronix DeepSeek-V3/R1 page).
    """
    q = _f64(q_nope)
    w_uk, _ = split_wkv_b(wkv_b, q.shape[-1])
    return np.einsum("bhqd,hdc->bhqc", q, w_uk)


def visibility(B: int, Q: int, Lk: int, seq_lens=None, causal_mask=None, causal: bool = False):
    """Boolean (B,Q,Lk): position t of sequence b is visible to query q.

    mask[t] != 0 (the question's (1,1,1,Lk) causal_mask, 1 = visible) and
    t < L_b and, when ``causal``, t <= L_b - Q + q (the Q new tokens are the
    last Q rows; each sees itself and everything before it, the question's
    "only the current and earlier positions").
    """
    t = np.arange(Lk)
    L = np.full(B, Lk, dtype=np.int64) if seq_lens is None else np.asarray(seq_lens, np.int64)
    vis = np.broadcast_to(t[None, None, :] < L[:, None, None], (B, Q, Lk)).copy()
    if causal_mask is not None:
        m = np.asarray(causal_mask).reshape(-1)[:Lk] != 0
        vis &= m[None, None, :]
    if causal:
        qi = np.arange(Q)
        last = L[:, None] - Q + qi[None, :]          # (B,Q)
        vis &= t[None, None, :] <= last[:, :, None]
    return vis


def latent_scores(q_lat, q_pe, kv_cache, pe_cache):
    """Blanks [2] and the position part: s = q_lat . kv[t] + q_pe . pe[t] -> (B,H,Q,Lk).

    "MLA 单步解码" question, steps 2) and 3): scores_nope = einsum(bhqc,btc),
    scores_pe = einsum(bhqr,btr), merged by addition.
    """
    s = np.einsum("bhqc,btc->bhqt", _f64(q_lat), _f64(kv_cache))
    if q_pe is not None:
        s = s + np.einsum("bhqr,btr->bhqt", _f64(q_pe), _f64(pe_cache))
    return s


def masked_softmax(logits, vis, sinks=None):
    """Softmax over the last axis with invisible positions at -inf (blank [4]).

    ``sinks`` (H,) adds one extra logit per head to the denominator only (it
    carries no value), as the attn_sink score column of the DeepSeek-V4.1-Flash
    4A page (§2 Luồng). Returns (attn (B,H,Q,Lk), lse (B,H,Q)) where lse is the
    natural log of the full denominator. Rows with nothing visible (and no
    sink) get zero weights and lse = -inf.
    """
    lg = np.where(vis[:, None, :, :], _f64(logits), -np.inf)
    m = lg.max(axis=-1)                                       # (B,H,Q)
    if sinks is not None:
        sk = _f64(sinks)[None, :, None]
        m = np.maximum(m, sk)
    m0 = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(lg - m0[..., None])
    den = e.sum(axis=-1)
    if sinks is not None:
        den = den + np.exp(sk - m0)
    attn = np.zeros_like(e)
    ok = den > 0
    attn[ok] = e[ok] / den[ok][:, None]
    lse = np.full(den.shape, -np.inf)
    lse[ok] = m0[ok] + np.log(den[ok])
    return attn, lse


def latent_attention(q_lat, q_pe, kv_cache, pe_cache, softmax_scale, vis, sinks=None):
    """Scores, scale, mask, softmax and latent aggregation.

    logits = (scores_nope + scores_pe) * softmax_scale (blank [3]); invisible
    -> -inf (blank [4]); attn = softmax; x = einsum(bhqt,btc) over kv_cache
    (step 5) of the "MLA 单步解码" question). Returns (x (B,H,Q,Ckv), attn, lse).
    """
    logits = latent_scores(q_lat, q_pe, kv_cache, pe_cache) * float(softmax_scale)
    attn, lse = masked_softmax(logits, vis, sinks)
    x = np.einsum("bhqt,btc->bhqc", attn, _f64(kv_cache))
    return x, attn, lse


def up_proj(x, wkv_b, Dn: int):
    """Blank [5]: out[b,h,q,v] = sum_c x[b,h,q,c] * W_UV[h,v,c] -> (B,H,Q,Vd)."""
    _, w_uv = split_wkv_b(wkv_b, Dn)
    return np.einsum("bhqc,hvc->bhqv", _f64(x), w_uv)


def mla_decode_step(q_nope, q_pe, kv_cache, pe_cache, wkv_b, softmax_scale, causal_mask=None,
                    seq_lens=None, causal: bool = False, return_all: bool = False):
    """The whole absorbed step of the "MLA 单步解码" question -> out (B,H,Q,Vd).

    With ``return_all`` also returns q_lat, x, attn and lse.
    """
    qn = _f64(q_nope)
    B, H, Q, Dn = qn.shape
    Lk = np.asarray(kv_cache).shape[1]
    vis = visibility(B, Q, Lk, seq_lens, causal_mask, causal)
    q_lat = absorb_q(qn, wkv_b)
    x, attn, lse = latent_attention(q_lat, q_pe, kv_cache, pe_cache, softmax_scale, vis)
    out = up_proj(x, wkv_b, Dn)
    if return_all:
        return dict(out=out, q_lat=q_lat, x=x, attn=attn, lse=lse, vis=vis)
    return out


def naive_decompressed_mha(q_nope, q_pe, kv_cache, pe_cache, wkv_b, softmax_scale, vis):
    """Standard attention over decompressed per-head K and V (no absorption).

    The CacheDecompressed form of the ackingliu.top article "DeepSeek MLA
    projection absorption": every cached latent c_t is up-projected per head,
    k_nope = W_UK[h] c_t (Dn) and v = W_UV[h] c_t (Vd); the key is k_nope
    concatenated with the shared rope key pe_t; the query is q_nope
    concatenated with q_pe. Written independently of the absorbed functions
    above (own weight slicing, own softmax) so that it can pin them.
    """
    qn, qp, kv, pe, w = (_f64(a) for a in (q_nope, q_pe, kv_cache, pe_cache, wkv_b))
    B, H, Q, Dn = qn.shape
    Lk = kv.shape[1]
    Dr = qp.shape[-1]
    Vd = w.shape[1] - Dn
    out = np.zeros((B, H, Q, Vd))
    for b in range(B):
        for h in range(H):
            Wk = w[h, 0:Dn, :]
            Wv = w[h, Dn:Dn + Vd, :]
            k = np.empty((Lk, Dn + Dr))
            k[:, :Dn] = kv[b] @ Wk.T
            k[:, Dn:] = pe[b]
            v = kv[b] @ Wv.T                                  # (Lk, Vd)
            for q in range(Q):
                qq = np.concatenate([qn[b, h, q], qp[b, h, q]])
                s = (k @ qq) * float(softmax_scale)
                seen = vis[b, q]
                if not seen.any():
                    continue
                smax = s[seen].max()
                p = np.where(seen, np.exp(s - smax), 0.0)
                p /= p.sum()
                out[b, h, q] = p @ v
    return out


def gather_paged(pool, block_table, seq_lens, page_size: int, Lk: int | None = None):
    """Rebuild contiguous (B, Lk, C) rows from a paged pool.

    Token t of sequence b lives in row t mod page_size of pool page
    block_table[b][t div page_size]: the paged form of the per-token slot
    offsets of the neuronix page's LatentKVCachePool::allocate_slot. Rows at
    or beyond seq_lens[b] are zero.
    """
    pool = _f64(pool)
    bt = np.asarray(block_table)
    L = np.asarray(seq_lens, np.int64)
    B = bt.shape[0]
    if Lk is None:
        Lk = int(L.max())
    out = np.zeros((B, Lk, pool.shape[-1]))
    for b in range(B):
        for t in range(int(L[b])):
            out[b, t] = pool[bt[b, t // page_size], t % page_size]
    return out


def cache_append(pool, block_table, seq_lens, rows, page_size: int):
    """Write each sequence's Q new cache rows into their paged slots.

    rows (B, Q, C) are the new tokens' rows (latent, rope part, combined row
    or FP4 entry); seq_lens are the lengths after the append, so new token i
    of sequence b sits at position t = seq_lens[b] - Q + i and goes to row
    t mod page_size of page block_table[b][t div page_size] -- the slot
    addressing read back by gather_paged (the neuronix page appends the new
    token's latent to the LatentKVCachePool before attending). Returns a new
    pool of the input's dtype; a page id outside [0, num_pages) raises.
    """
    out = np.array(pool, copy=True)
    bt = np.asarray(block_table)
    L = np.asarray(seq_lens, np.int64)
    r = np.asarray(rows)
    B, Q = r.shape[0], r.shape[1]
    for b in range(B):
        for i in range(Q):
            t = int(L[b]) - Q + i
            if t < 0:
                raise ValueError(f"sequence {b}: length {int(L[b])} shorter than the {Q} new tokens")
            page = int(bt[b, t // page_size])
            if not 0 <= page < out.shape[0]:
                raise ValueError(f"sequence {b}, token {t}: page id {page} outside the pool")
            out[page, t % page_size] = r[b, i]
    return out


def split_partials(q_lat, q_pe, kv_cache, pe_cache, softmax_scale, vis, bounds):
    """Per-split partial results over token ranges ``bounds = [(t0, t1), ...]``.

    For split s: O_s = softmax over visible t in [t0,t1) applied to kv rows,
    and lse_s = log sum exp of those logits (-inf when none is visible).
    Returns O (S,B,H,Q,Ckv), lse (S,B,H,Q).
    """
    Os, lses = [], []
    for (t0, t1) in bounds:
        v = np.zeros_like(vis)
        v[:, :, t0:t1] = vis[:, :, t0:t1]
        x, _, lse = latent_attention(q_lat, q_pe, kv_cache, pe_cache, softmax_scale, v)
        Os.append(x)
        lses.append(lse)
    return np.stack(Os), np.stack(lses)


def combine_partials(O, lse, sinks=None):
    """Merge split partials: L = log(sum_s e^{lse_s} [+ e^{sink_h}]), x = sum_s e^{lse_s-L} O_s.

    The flash-attention rescaling the CANN ops-nn MLA article refers to as the
    usual FlashAttention softmax update (§二, ComputeChunk Stage 3), applied
    across splits instead of across 64-token chunks. Returns (x, L).
    """
    O = _f64(O)
    lse = _f64(lse)
    terms = lse
    if sinks is not None:
        sk = np.broadcast_to(_f64(sinks)[None, None, :, None], (1,) + lse.shape[1:])
        terms = np.concatenate([lse, sk], axis=0)
    m = terms.max(axis=0)
    m0 = np.where(np.isfinite(m), m, 0.0)
    den = np.exp(terms - m0[None]).sum(axis=0)
    L = np.full(den.shape, -np.inf)
    ok = den > 0
    L[ok] = m0[ok] + np.log(den[ok])
    Lsafe = np.where(ok, L, 0.0)
    w = np.where(np.isfinite(lse), np.exp(lse - Lsafe[None]), 0.0)
    x = (w[..., None] * O).sum(axis=0)
    return x, L
