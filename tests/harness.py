"""Shared helpers of the parity tests: upload workloads, run the library, run the oracle, compare.

The GPU side goes through latent_kv_decode_b200.ops (the C ABI); the
expected values come from oracle/ on the same seeded inputs.
"""
from __future__ import annotations

import numpy as np
import torch

from latent_kv_decode_b200 import workloads as wl
from oracle import mla as omla
from oracle import v41 as ov41

# tolerances: |g - o| <= atol + rtol*|o|
TOL_F32 = dict(rtol=1e-4, atol=1e-4)
TOL_BF16 = dict(rtol=2e-2, atol=2e-2)
REL_L2_BF16 = 1e-2   # extra gate: ||g-o|| / ||o|| for bf16 outputs
# lse is what mla_combine weights the splits by: an absolute bound of its own.
# The GPU forms it in float32 from the same bf16 operands the oracle reads, so
# only accumulation order and the exp2 approximation separate the two.
TOL_LSE_BF16 = dict(rtol=0.0, atol=1e-2)
TOL_LSE_F32 = dict(rtol=0.0, atol=1e-4)


def tdt(w: wl.Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def dev(a, dtype=None):
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def upload(w: wl.Workload, combined: bool = False) -> dict:
    """Device tensors of a workload. ``combined`` stores latent+rope as one 576-wide row."""
    dt = tdt(w)
    d = dict(q_nope=dev(w.q_nope, dt), q_pe=dev(w.q_pe, dt), wkv_b=dev(w.wkv_b, dt))
    if w.block_table is not None:
        if combined:
            pool = torch.cat([dev(w.kv_pool, dt), dev(w.pe_pool, dt)], dim=-1).contiguous()
            d["kv"], d["pe"] = pool[..., :w.Ckv], pool[..., w.Ckv:]
        else:
            d["kv"], d["pe"] = dev(w.kv_pool, dt), dev(w.pe_pool, dt)
        d["block_table"] = dev(w.block_table)
    else:
        if combined:
            cat = torch.cat([dev(w.kv_cache, dt), dev(w.pe_cache, dt)], dim=-1).contiguous()
            d["kv"], d["pe"] = cat[..., :w.Ckv], cat[..., w.Ckv:]
        else:
            d["kv"], d["pe"] = dev(w.kv_cache, dt), dev(w.pe_cache, dt)
        d["block_table"] = None
    d["seq_lens"] = dev(w.seq_lens) if w.seq_lens is not None else None
    d["mask"] = dev(w.causal_mask) if w.causal_mask is not None else None
    return d


def gpu_step(w: wl.Workload, d: dict, num_splits: int = 0, err_flag=None):
    """absorb -> decode -> combine -> up_proj through the C ABI; returns numpy dict."""
    from latent_kv_decode_b200 import ops
    own_flag = err_flag is None
    if own_flag:
        err_flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_lat = ops.mla_absorb_q(d["q_nope"], d["wkv_b"])
    call = ops.mla_decode(q_lat, d["q_pe"], d["kv"], d["pe"], w.softmax_scale,
                          seq_lens=d["seq_lens"], block_table=d["block_table"],
                          page_size=w.page_size, causal_mask=d["mask"], causal=w.causal,
                          num_splits=num_splits, err_flag=err_flag,
                          Lk=w.Lk if d["block_table"] is None else None)
    ops.mla_combine(call)
    out = ops.mla_up_proj(call.x, d["wkv_b"], w.Dn)
    torch.cuda.synchronize()
    if own_flag:
        assert int(err_flag.item()) == 0, f"kernel reported device error bits {int(err_flag.item())}"
    f = lambda t: t.float().cpu().numpy().astype(np.float64)
    return dict(q_lat=f(q_lat), x=f(call.x), lse=f(call.lse), out=f(out), splits=call.num_splits)


def contiguous_cache(w: wl.Workload, batch=None):
    """(B', Lk, C) caches of the selected sequences (all when ``batch`` is None)."""
    sel = slice(None) if batch is None else np.asarray(batch)
    if w.block_table is None:
        return w.kv_cache[sel], w.pe_cache[sel]
    L = w.lens()[sel]
    bt = w.block_table[sel]
    return (omla.gather_paged(w.kv_pool, bt, L, w.page_size, w.Lk),
            omla.gather_paged(w.pe_pool, bt, L, w.page_size, w.Lk))


def oracle_step(w: wl.Workload, batch=None, q_lat=None, x=None):
    """Oracle of the whole step (optionally on a subset of sequences).

    ``q_lat`` / ``x``: when given (the GPU's rounded intermediates), the
    later stages start from them, so each ABI call is checked on its own.
    """
    kv, pe = contiguous_cache(w, batch)
    sel = slice(None) if batch is None else np.asarray(batch)
    qn, qp = w.q_nope[sel], w.q_pe[sel]
    lens = None if w.seq_lens is None else w.seq_lens[sel]
    B = qn.shape[0]
    vis = omla.visibility(B, w.Q, kv.shape[1], lens, w.causal_mask, w.causal)
    ql = omla.absorb_q(qn, w.wkv_b)
    if x is not None:
        # only the up-projection of the given latent output is asked for
        return dict(q_lat=ql, x=None, lse=None, out=omla.up_proj(x, w.wkv_b, w.Dn))
    ql_in = ql if q_lat is None else q_lat
    xo, attn, lse = omla.latent_attention(ql_in, qp, kv, pe, w.softmax_scale, vis)
    out = omla.up_proj(xo, w.wkv_b, w.Dn)
    return dict(q_lat=ql, x=xo, lse=lse, out=out)


def assert_close(g, o, tol, name="", rel_l2=None):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    assert g.shape == o.shape, (name, g.shape, o.shape)
    fin = np.isfinite(o)
    assert np.array_equal(np.isfinite(g), fin), f"{name}: finite pattern differs"
    err = np.abs(g[fin] - o[fin])
    lim = tol["atol"] + tol["rtol"] * np.abs(o[fin])
    bad = err > lim
    if bad.any():
        i = np.argmax(err - lim)
        raise AssertionError(f"{name}: {bad.sum()} of {bad.size} outside tolerance; worst "
                             f"|g-o|={err[i]:.3e} at |o|={abs(o[fin][i]):.3e}")
    if not np.array_equal(g[~fin], o[~fin]):
        raise AssertionError(f"{name}: non-finite values differ")
    if rel_l2 is not None and fin.any():
        num = np.linalg.norm(g[fin] - o[fin])
        den = np.linalg.norm(o[fin])
        if den > 0:
            assert num / den <= rel_l2, f"{name}: relative L2 error {num / den:.3e} > {rel_l2}"


# --- shared-latent (FP4) variant ---------------------------------------------

def fp4_entries(w: wl.Workload) -> np.ndarray:
    """FP4 cache entries of a shared-latent workload (the oracle's cache-write step)."""
    return ov41.cache_write(w.latent, w.rope_tail, w.rope_theta)


def fp4_pool(w: wl.Workload, entries: np.ndarray) -> np.ndarray:
    ps = w.page_size
    L = w.lens()
    pool = np.zeros((int(w.block_table.max()) + 1, ps, ov41.ENTRY_BYTES), np.uint8)
    for b in range(w.B):
        for t in range(int(L[b])):
            pool[w.block_table[b, t // ps], t % ps] = entries[b, t]
    return pool


def gpu_shared_latent(w: wl.Workload, entries: np.ndarray, num_splits: int = 0, paged=False,
                      row_bytes: int = 288):
    """The shared-latent decode through the C ABI. ``row_bytes`` > 288 stores
    each 288-byte entry at the start of a wider (padded) cache row."""
    from latent_kv_decode_b200 import ops
    q = dev(w.q, torch.bfloat16)
    store = fp4_pool(w, entries) if paged else entries
    if row_bytes != ov41.ENTRY_BYTES:
        wide = np.zeros(store.shape[:-1] + (row_bytes,), np.uint8)
        wide[..., :ov41.ENTRY_BYTES] = store
        kv = dev(wide)[..., :ov41.ENTRY_BYTES]
    else:
        kv = dev(store)
    bt = dev(w.block_table) if paged else None
    sinks = dev(w.sinks.astype(np.float32)) if w.sinks is not None else None
    err_flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    call = ops.mla_decode(q, None, kv, None, w.softmax_scale,
                          seq_lens=dev(w.seq_lens) if w.seq_lens is not None else None,
                          block_table=bt, page_size=w.page_size, causal=w.causal, sinks=sinks,
                          causal_mask=dev(w.causal_mask) if w.causal_mask is not None else None,
                          rope_tail=w.rope_tail, rope_theta=w.rope_theta, num_splits=num_splits,
                          Lk=w.Lk if bt is None else None, err_flag=err_flag)
    ops.mla_combine(call)
    torch.cuda.synchronize()
    assert int(err_flag.item()) == 0, f"kernel reported device error bits {int(err_flag.item())}"
    return dict(x=call.x.float().cpu().numpy().astype(np.float64),
                lse=call.lse.cpu().numpy().astype(np.float64), splits=call.num_splits)


def oracle_shared_latent(w: wl.Workload, entries: np.ndarray, batch=None):
    sel = slice(None) if batch is None else np.asarray(batch)
    r = ov41.shared_latent_decode(w.q[sel], entries[sel], w.sinks, w.softmax_scale,
                                  None if w.seq_lens is None else w.seq_lens[sel], w.causal,
                                  causal_mask=w.causal_mask, tail=w.rope_tail,
                                  theta=w.rope_theta, return_all=True)
    return dict(x=r["x"], lse=r["lse"])
