"""GPU parity: libmla through its C ABI vs the fp64 oracle on the same seeded inputs.

Each ABI call is checked on its own (the oracle stage is fed the GPU's
previous output) and end to end. Small cases span several 64-token tiles and
a ragged tail; full-size workloads are checked on sampled sequences.
"""
import numpy as np
import pytest
import torch

from latent_kv_decode_b200 import workloads as wl
from oracle import mla as omla

from harness import (TOL_BF16, TOL_F32, TOL_LSE_BF16, TOL_LSE_F32, REL_L2_BF16, assert_close, dev,
                     fp4_entries, gpu_shared_latent, gpu_step, oracle_shared_latent, oracle_step,
                     upload)

pytestmark = pytest.mark.gpu


def _check_step(w, g, batch=None, tol=None, rel=None):
    tol = tol or (TOL_F32 if w.dtype == "f32" else TOL_BF16)
    tol_lse = TOL_LSE_F32 if w.dtype == "f32" else TOL_LSE_BF16
    rel = rel if rel is not None else (None if w.dtype == "f32" else REL_L2_BF16)
    sel = slice(None) if batch is None else np.asarray(batch)
    ref = oracle_step(w, batch)
    assert_close(g["q_lat"][sel], ref["q_lat"], tol, "q_lat", rel)
    # decode on the GPU's own q_lat, up-projection on the GPU's own x
    ref_x = oracle_step(w, batch, q_lat=g["q_lat"][sel])
    assert_close(g["x"][sel], ref_x["x"], tol, "x", rel)
    assert_close(g["lse"][sel], ref_x["lse"], tol_lse, "lse")
    ref_o = oracle_step(w, batch, x=g["x"][sel])
    assert_close(g["out"][sel], ref_o["out"], tol, "out(up_proj)", rel)
    assert_close(g["out"][sel], ref["out"], tol, "out(end to end)", rel)


@pytest.mark.parametrize("B,Q,Dn", [(70, 1, 128), (33, 2, 128), (5, 4, 64), (1, 1, 128)])
def test_projections_row_blocks(B, Q, Dn):
    """Both projections on their own: query rows in blocks of 64 with a ragged
    last block (70, 66, 20 and 1 rows), Q > 1 and Dn = 64. up_proj is fed the
    GPU's q_lat as its latent input."""
    from latent_kv_decode_b200 import ops
    w = wl.make_mla(B=B, H=8, Q=Q, Dn=Dn, Dr=64, Vd=128, Ckv=512, Lk=8, dtype="bf16", seed=11)
    d = upload(w)
    q_lat = ops.mla_absorb_q(d["q_nope"], d["wkv_b"])
    out = ops.mla_up_proj(q_lat, d["wkv_b"], Dn)
    torch.cuda.synchronize()
    g_lat = q_lat.float().cpu().numpy().astype(np.float64)
    g_out = out.float().cpu().numpy().astype(np.float64)
    assert_close(g_lat, omla.absorb_q(w.q_nope, w.wkv_b), TOL_BF16, "q_lat", REL_L2_BF16)
    assert_close(g_out, omla.up_proj(g_lat, w.wkv_b, Dn), TOL_BF16, "out", REL_L2_BF16)


@pytest.mark.parametrize("splits", [0, 1, 3])
def test_demo_fp32(splits):
    w = wl.demo_fp32()
    g = gpu_step(w, upload(w), num_splits=splits)
    assert g["out"].shape == (2, 8, 1, 128)
    _check_step(w, g)


@pytest.mark.parametrize("splits", [1, 2, 5, 0])
@pytest.mark.parametrize("combined", [False, True])
def test_dsv3_small_ragged_tail(splits, combined):
    w = wl.dsv3(B=3, Lk=333, seed=11)
    _check_step(w, gpu_step(w, upload(w, combined), num_splits=splits))


def test_fp32_dsv3_dims():
    w = wl.make_mla(2, 16, 1, 128, 64, 128, 512, 150, dtype="f32", seed=12)
    _check_step(w, gpu_step(w, upload(w), num_splits=2))


@pytest.mark.parametrize("splits", [1, 4])
def test_seq_lens_mask_and_causal_q2(splits):
    mask = np.ones(300, np.uint8)
    mask[[0, 17, 64, 65, 299]] = 0
    w = wl.make_mla(4, 128, 2, 128, 64, 128, 512, 300, dtype="bf16", seed=13,
                    seq_lens=[300, 1, 65, 129], causal=True, causal_mask=mask)
    _check_step(w, gpu_step(w, upload(w), num_splits=splits))


@pytest.mark.parametrize("combined", [False, True])
def test_paged_ragged_q2(combined):
    w = wl.make_mla(5, 128, 2, 128, 64, 128, 512, 0, dtype="bf16", seed=14, lk_range=(2, 700),
                    paged=True, causal=True)
    _check_step(w, gpu_step(w, upload(w, combined), num_splits=0))


def test_more_splits_than_tiles_leaves_empty_splits():
    w = wl.dsv3(B=2, Lk=100, seed=15)
    _check_step(w, gpu_step(w, upload(w), num_splits=7))


def test_single_token_cache():
    w = wl.dsv3(B=2, Lk=1, seed=16)
    _check_step(w, gpu_step(w, upload(w), num_splits=1))


def test_fully_masked_rows_are_zero():
    mask = np.zeros(70, np.uint8)
    w = wl.make_mla(2, 8, 1, 64, 32, 128, 512, 70, dtype="f32", seed=17, causal_mask=mask)
    g = gpu_step(w, upload(w), num_splits=2)
    assert np.all(g["x"] == 0) and np.all(g["out"] == 0) and np.all(np.isneginf(g["lse"]))


def test_bad_block_table_entry_sets_flag_and_skips_page():
    w = wl.make_mla(2, 8, 1, 64, 32, 128, 512, 0, dtype="f32", seed=18, seq_lens=[200, 130],
                    paged=True)
    d = upload(w)
    bt = w.block_table.copy()
    bt[0, 1] = 10_000                      # page 1 of sequence 0 is out of range
    d["block_table"] = dev(bt)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = gpu_step(w, d, num_splits=2, err_flag=flag)
    assert int(flag.item()) & 1
    # expected: the same decode with tokens 64..127 of sequence 0 invisible
    mask_w = wl.make_mla(2, 8, 1, 64, 32, 128, 512, 0, dtype="f32", seed=18, seq_lens=[200, 130],
                         paged=True)
    kv = omla.gather_paged(mask_w.kv_pool, mask_w.block_table, mask_w.lens(), 64)
    pe = omla.gather_paged(mask_w.pe_pool, mask_w.block_table, mask_w.lens(), 64)
    vis = omla.visibility(2, 1, kv.shape[1], mask_w.seq_lens)
    vis[0, :, 64:128] = False
    x, _, _ = omla.latent_attention(g["q_lat"], w.q_pe, kv, pe, w.softmax_scale, vis)
    assert_close(g["x"], x, TOL_F32, "x with skipped page")


# --- shapes the tensor-core kernels do not take (generic CUDA-core decode) ----

@pytest.mark.parametrize("H,Q,splits", [(8, 1, 1), (64, 1, 3), (24, 2, 0), (40, 1, 2)])
def test_bf16_generic_decode_rows_not_multiple_of_128(H, Q, splits):
    """bf16 caches whose H*Q is not a multiple of 128 run the generic decode:
    parity with the oracle, ragged lengths ending mid-tile, causal for Q > 1."""
    w = wl.make_mla(3, H, Q, 128, 64, 128, 512, 0, dtype="bf16", seed=40 + H + Q,
                    seq_lens=[333, 70, 129], causal=Q > 1)
    _check_step(w, gpu_step(w, upload(w), num_splits=splits))


def test_bf16_generic_decode_dr32_dn64():
    """Dr = 32 (not the tensor-core kernel's 64) on bf16, Dn = 64."""
    w = wl.make_mla(2, 128, 1, 64, 32, 128, 512, 200, dtype="bf16", seed=45)
    _check_step(w, gpu_step(w, upload(w), num_splits=2))


@pytest.mark.parametrize("H,Q,splits", [(40, 1, 1), (8, 2, 3), (24, 1, 0)])
def test_shared_latent_fp4_generic_rows(H, Q, splits):
    """FP4 caches with H*Q not a multiple of 64 run the generic decode."""
    w = wl.make_shared_latent(2, H, Q, 150, seed=46 + H, seq_lens=[150, 77], causal=Q > 1)
    ent = fp4_entries(w)
    g = gpu_shared_latent(w, ent, num_splits=splits)
    ref = oracle_shared_latent(w, ent)
    assert_close(g["x"], ref["x"], TOL_BF16, "x", REL_L2_BF16)
    assert_close(g["lse"], ref["lse"], TOL_LSE_BF16, "lse")


@pytest.mark.parametrize("paged", [False, True])
def test_shared_latent_fp4_padded_rows(paged):
    """288-byte entries at the start of 304-byte cache rows (a row stride the
    tensor-core FP4 kernel does not take): the generic decode reads them."""
    w = wl.make_shared_latent(3, 64, 1, 200, seed=49, seq_lens=[200, 65, 3], paged=paged)
    ent = fp4_entries(w)
    g = gpu_shared_latent(w, ent, num_splits=2, paged=paged, row_bytes=304)
    ref = oracle_shared_latent(w, ent)
    assert_close(g["x"], ref["x"], TOL_BF16, "x", REL_L2_BF16)
    assert_close(g["lse"], ref["lse"], TOL_LSE_BF16, "lse")


# --- shared-latent FP4 variant ----------------------------------------------

@pytest.mark.parametrize("splits", [1, 3, 0])
def test_shared_latent_fp4_small(splits):
    w = wl.make_shared_latent(3, 64, 1, 333, seed=21, seq_lens=[333, 64, 200])
    ent = fp4_entries(w)
    g = gpu_shared_latent(w, ent, num_splits=splits)
    ref = oracle_shared_latent(w, ent)
    assert_close(g["x"], ref["x"], TOL_BF16, "x", REL_L2_BF16)
    assert_close(g["lse"], ref["lse"], TOL_LSE_BF16, "lse")


def test_shared_latent_fp4_causal_q2():
    """Q = 2 causal rows (row = head * Q + query): 32 heads x 2 queries fill one
    64-row block; ragged lengths end mid-tile."""
    w = wl.make_shared_latent(2, 32, 2, 150, seed=23, seq_lens=[150, 97], causal=True)
    ent = fp4_entries(w)
    g = gpu_shared_latent(w, ent, num_splits=2)
    ref = oracle_shared_latent(w, ent)
    assert_close(g["x"], ref["x"], TOL_BF16, "x", REL_L2_BF16)
    assert_close(g["lse"], ref["lse"], TOL_LSE_BF16, "lse")


@pytest.mark.parametrize("splits", [1, 3])
def test_shared_latent_fp4_question_mask(splits):
    """The question's (Lk) mask on top of causal Q = 2 rows and ragged lengths:
    hidden tokens sit inside tiles, at tile edges and in whole 32-token runs."""
    w = wl.make_shared_latent(2, 32, 2, 200, seed=24, seq_lens=[200, 131], causal=True)
    rng = np.random.Generator(np.random.PCG64(24))
    mask = (rng.random(200) > 0.3).astype(np.uint8)
    mask[[0, 31, 32, 63, 64]] = 0
    mask[96:128] = 0
    w.causal_mask = mask
    ent = fp4_entries(w)
    g = gpu_shared_latent(w, ent, num_splits=splits)
    ref = oracle_shared_latent(w, ent)
    assert_close(g["x"], ref["x"], TOL_BF16, "x", REL_L2_BF16)
    assert_close(g["lse"], ref["lse"], TOL_LSE_BF16, "lse")


def test_shared_latent_fp4_paged():
    w = wl.make_shared_latent(3, 64, 1, 260, seed=22, seq_lens=[260, 65, 3], paged=True)
    ent = fp4_entries(w)
    g = gpu_shared_latent(w, ent, num_splits=2, paged=True)
    ref = oracle_shared_latent(w, ent)
    assert_close(g["x"], ref["x"], TOL_BF16, "x", REL_L2_BF16)
    assert_close(g["lse"], ref["lse"], TOL_LSE_BF16, "lse")


# --- full-size workloads, sampled sequences ----------------------------------

@pytest.mark.slow
def test_full_dsv3_b64_lk4096():
    w = wl.dsv3()
    g = gpu_step(w, upload(w))
    _check_step(w, g)                      # every one of the 64 sequences


@pytest.mark.slow
def test_full_longctx_b4_lk131072():
    w = wl.longctx()
    g = gpu_step(w, upload(w))
    assert g["splits"] > 1
    _check_step(w, g, batch=[0, 3])


@pytest.mark.slow
def test_full_ragged_paged_b128_q2():
    w = wl.ragged_paged()
    g = gpu_step(w, upload(w))
    L = w.lens()
    # the shortest and the longest sequence, and 14 more spread over the batch
    order = np.argsort(L, kind="stable")
    batch = sorted({int(order[0]), int(order[-1])} |
                   {int(order[i]) for i in np.linspace(1, w.B - 2, 14).astype(int)})
    assert len(batch) == 16
    _check_step(w, g, batch=batch)


@pytest.mark.slow
def test_full_v41_fp4_sink_h64():
    w = wl.v41_shared_latent()
    ent = fp4_entries(w)
    g = gpu_shared_latent(w, ent)
    ref = oracle_shared_latent(w, ent)     # every one of the 32 sequences
    assert_close(g["x"], ref["x"], TOL_BF16, "x", REL_L2_BF16)
    assert_close(g["lse"], ref["lse"], TOL_LSE_BF16, "lse")
