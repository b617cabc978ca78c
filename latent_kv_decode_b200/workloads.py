"""Seeded synthetic inputs for single-step MLA decode.

This module draws random inputs and lays them out; it holds none of the
decode arithmetic. Both the CUDA path's tests/bench and the CPU oracle take
their inputs from here, so the two sides see bit-identical values.

Every array is returned as NumPy. Floating-point inputs are float32 arrays
whose values are exactly representable in the storage dtype of the workload
(bf16 values are rounded once, round-to-nearest-even, at generation time);
``bf16_bits`` gives the raw 16-bit patterns that are uploaded to the GPU.

Workloads (shapes follow ``mla_decode_step`` of the "MLA 单步解码" exam
question on 6547.cn: q_nope (B,H,Q,Dn), q_pe (B,H,Q,Dr), kv_cache (B,Lk,Ckv),
pe_cache (B,Lk,Dr), wkv_b (H,Dn+Vd,Ckv)):

- ``demo_fp32``: the question's ``demo_mla_step`` shape, fp32, all N(0,1).
- ``dsv3_b64_lk4096``: DeepSeek-V3 decode shape, bf16 storage, B=64, Lk=4096.
- ``ragged_paged_b128_q2``: B=128, Lk_b ~ U[512, 16384], 64-token pages with
  a random page permutation, Q=2 causal speculative tokens.
- ``longctx_b4_lk131072``: B=4, Lk=131072.
- ``v41_fp4_sink_h64``: the DeepSeek-V4.1-Flash shared-latent variant, H=64,
  B=32, Lk=8192; this module only draws the raw latent, sinks and q; the FP4
  cache entries are made from the latent by the cache-write step.

Draw order per workload (NumPy PCG64, one generator per workload): seq_lens,
q_nope, q_pe, kv_cache, pe_cache, wkv_b, sinks, block-table permutation.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

PAGE_SIZE = 64


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); float32 out."""
    return bf16_from_bits(bf16_bits(x))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of the bf16 nearest to each float32 (RNE)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_from_bits(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Workload:
    """One decode step's inputs. ``None`` fields are absent for the workload."""

    name: str
    B: int
    H: int
    Q: int
    Dn: int
    Dr: int
    Vd: int
    Ckv: int
    Lk: int                       # cache rows per sequence (max over sequences when ragged)
    dtype: str                    # storage dtype of q / cache / weights: "f32" or "bf16"
    softmax_scale: float
    q_nope: Optional[np.ndarray]  # (B,H,Q,Dn)
    q_pe: Optional[np.ndarray]    # (B,H,Q,Dr)
    kv_cache: Optional[np.ndarray]  # (B,Lk,Ckv) contiguous, or None when paged
    pe_cache: Optional[np.ndarray]  # (B,Lk,Dr)
    wkv_b: Optional[np.ndarray]   # (H,Dn+Vd,Ckv)
    causal_mask: Optional[np.ndarray] = None  # (Lk,) uint8, 1 = visible
    seq_lens: Optional[np.ndarray] = None     # (B,) int32
    causal: bool = False                      # Q>1: query i sees t <= len-Q+i
    # paged layout: pools hold num_pages pages of PAGE_SIZE rows
    kv_pool: Optional[np.ndarray] = None      # (num_pages, page, Ckv)
    pe_pool: Optional[np.ndarray] = None      # (num_pages, page, Dr)
    block_table: Optional[np.ndarray] = None  # (B, max_pages) int32
    page_size: int = PAGE_SIZE
    # shared-latent (V4.1) variant
    q: Optional[np.ndarray] = None            # (B,H,Q,Ckv) query in latent space, RoPE'd tail
    latent: Optional[np.ndarray] = None       # (B,Lk,Ckv) raw latent before RoPE/quantisation
    sinks: Optional[np.ndarray] = None        # (H,) float32 sink logits
    rope_tail: int = 0
    rope_theta: float = 10000.0
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        """Query tokens decoded by one step: B*Q."""
        return self.B * self.Q

    def lens(self) -> np.ndarray:
        return (np.full(self.B, self.Lk, np.int64) if self.seq_lens is None
                else self.seq_lens.astype(np.int64))


def _normal(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    return x if dtype == "f32" else bf16_round(x)


def make_mla(B: int, H: int, Q: int, Dn: int, Dr: int, Vd: int, Ckv: int, Lk: int,
             dtype: str = "bf16", seed: int = 0, wkv_scale: Optional[float] = None,
             softmax_scale: Optional[float] = None, seq_lens=None, lk_range=None,
             paged: bool = False, causal: bool = False, causal_mask=None,
             name: str = "custom") -> Workload:
    """General absorbed-MLA workload (q_nope/q_pe/kv/pe/wkv_b).

    ``wkv_scale``: multiplier of the N(0,1) wkv_b draw (None = 1/sqrt(Ckv),
    the fan-in of the latent-to-head projection). ``lk_range=(lo,hi)`` draws
    per-sequence lengths uniformly in [lo,hi]; ``seq_lens`` fixes them.
    ``paged`` lays the cache out in 64-token pages with a random permutation.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    if lk_range is not None:
        lo, hi = lk_range
        seq_lens = rng.integers(lo, hi, size=B, endpoint=True).astype(np.int32)
    if seq_lens is not None:
        seq_lens = np.asarray(seq_lens, np.int32)
        Lk = int(max(Lk, seq_lens.max())) if Lk else int(seq_lens.max())
    if wkv_scale is None:
        wkv_scale = 1.0 / math.sqrt(Ckv)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(Dn + Dr)
    q_nope = _store(_normal(rng, (B, H, Q, Dn)), dtype)
    q_pe = _store(_normal(rng, (B, H, Q, Dr)), dtype)
    w = Workload(name=name, B=B, H=H, Q=Q, Dn=Dn, Dr=Dr, Vd=Vd, Ckv=Ckv, Lk=Lk, dtype=dtype,
                 softmax_scale=float(softmax_scale), q_nope=q_nope, q_pe=q_pe,
                 kv_cache=None, pe_cache=None, wkv_b=None, seq_lens=seq_lens, causal=causal,
                 causal_mask=None if causal_mask is None else np.asarray(causal_mask, np.uint8))
    if not paged:
        w.kv_cache = _store(_normal(rng, (B, Lk, Ckv)), dtype)
        w.pe_cache = _store(_normal(rng, (B, Lk, Dr)), dtype)
        w.wkv_b = _store(_normal(rng, (H, Dn + Vd, Ckv), wkv_scale), dtype)
        return w
    # Paged: each sequence's L_b rows are drawn in order (all kv rows, then
    # all pe rows), then scattered into 64-token pages of one pool whose page
    # ids are a random permutation. Unused table slots hold -1; unused rows of
    # a last page are zero.
    ps = w.page_size
    lens = w.lens()
    npages = [(int(L) + ps - 1) // ps for L in lens]
    total = int(sum(npages))
    kv_pool = np.zeros((total, ps, Ckv), np.float32)
    pe_pool = np.zeros((total, ps, Dr), np.float32)
    kv_rows = [_store(_normal(rng, (int(L), Ckv)), dtype) for L in lens]
    pe_rows = [_store(_normal(rng, (int(L), Dr)), dtype) for L in lens]
    w.wkv_b = _store(_normal(rng, (H, Dn + Vd, Ckv), wkv_scale), dtype)
    perm = rng.permutation(total).astype(np.int32)
    bt = np.full((B, max(npages)), -1, np.int32)
    k = 0
    for b in range(B):
        L = int(lens[b])
        for j in range(npages[b]):
            p = perm[k]
            k += 1
            bt[b, j] = p
            n = min(ps, L - j * ps)
            kv_pool[p, :n] = kv_rows[b][j * ps:j * ps + n]
            pe_pool[p, :n] = pe_rows[b][j * ps:j * ps + n]
        kv_rows[b] = pe_rows[b] = None
    w.kv_pool, w.pe_pool, w.block_table = kv_pool, pe_pool, bt
    return w


def make_shared_latent(B: int, H: int, Q: int, Lk: int, Ckv: int = 512, seed: int = 4,
                       rope_tail: int = 64, rope_theta: float = 10000.0, seq_lens=None,
                       causal: bool = False, paged: bool = False,
                       name: str = "custom_shared_latent") -> Workload:
    """Inputs of the shared-latent (K = V = latent) variant.

    Draws q (B,H,Q,Ckv) as bf16 N(0,1), the raw latent (B,Lk,Ckv) N(0,1) in
    float32 and one N(0,1) sink logit per head. The FP4 entries are made by
    the cache-write step (RoPE at the token's position, then quantisation),
    which is outside this module.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    if seq_lens is not None:
        seq_lens = np.asarray(seq_lens, np.int32)
    q = bf16_round(_normal(rng, (B, H, Q, Ckv)))
    latent = _normal(rng, (B, Lk, Ckv))
    sinks = _normal(rng, (H,))
    w = Workload(name=name, B=B, H=H, Q=Q, Dn=0, Dr=0, Vd=0, Ckv=Ckv, Lk=Lk, dtype="bf16",
                 softmax_scale=1.0 / math.sqrt(Ckv), q_nope=None, q_pe=None, kv_cache=None,
                 pe_cache=None, wkv_b=None, seq_lens=seq_lens, causal=causal, q=q,
                 latent=latent, sinks=sinks, rope_tail=rope_tail, rope_theta=rope_theta)
    if paged:
        lens = w.lens()
        ps = w.page_size
        npages = [(int(L) + ps - 1) // ps for L in lens]
        perm = rng.permutation(int(sum(npages))).astype(np.int32)
        bt = np.full((B, max(npages)), -1, np.int32)
        k = 0
        for b in range(B):
            for j in range(npages[b]):
                bt[b, j] = perm[k]
                k += 1
        w.block_table = bt
    return w


# --- the five named workloads -------------------------------------------------

def demo_fp32(seed: int = 0) -> Workload:
    """``demo_mla_step``: B,H,Dn,Dr,Vd,Lk,Ckv = 2,8,64,32,128,10,512, fp32, all
    N(0,1) (wkv_b unscaled, as the demo draws it), scale 1/sqrt(Dn+Dr), mask
    all ones."""
    return make_mla(2, 8, 1, 64, 32, 128, 512, 10, dtype="f32", seed=seed, wkv_scale=1.0,
                    causal_mask=np.ones(10, np.uint8), name="demo_fp32")


def dsv3(B: int = 64, Lk: int = 4096, seed: int = 1, Q: int = 1) -> Workload:
    """DeepSeek-V3 decode shape: H=128, Dn=128, Dr=64, Vd=128, Ckv=512, bf16,
    wkv_b N(0,1)/sqrt(512), scale 1/sqrt(192), contiguous cache."""
    return make_mla(B, 128, Q, 128, 64, 128, 512, Lk, dtype="bf16", seed=seed,
                    name=f"dsv3_b{B}_lk{Lk}")


def ragged_paged(B: int = 128, lk_range=(512, 16384), seed: int = 2) -> Workload:
    """Ragged paged batch: per-sequence Lk ~ U[512,16384], 64-token pages in a
    randomly permuted block table, Q=2 speculative tokens causal among
    themselves."""
    w = make_mla(B, 128, 2, 128, 64, 128, 512, 0, dtype="bf16", seed=seed, lk_range=lk_range,
                 paged=True, causal=True, name=f"ragged_paged_b{B}_q2")
    return w


def longctx(B: int = 4, Lk: int = 131072, seed: int = 3) -> Workload:
    """Long-context split-KV case: B=4, Lk=131072, H=128, Q=1."""
    return make_mla(B, 128, 1, 128, 64, 128, 512, Lk, dtype="bf16", seed=seed,
                    name=f"longctx_b{B}_lk{Lk}")


def v41_shared_latent(B: int = 32, Lk: int = 8192, H: int = 64, seed: int = 4) -> Workload:
    """DeepSeek-V4.1-Flash-style shared latent: H=64, Q=1, B=32, Lk=8192."""
    return make_shared_latent(B, H, 1, Lk, seed=seed, name=f"v41_fp4_sink_h{H}")


def fp4_random_entries(B: int, Lk: int, Ckv: int = 512, seed: int = 5) -> np.ndarray:
    """(B, Lk, Ckv/2 + Ckv/16) uint8 cache entries for timing: Ckv/2 bytes of
    uniformly random E2M1 code pairs, then Ckv/16 random positive E4M3 scale
    bytes in [0.125, 0.94) (exponent field 4..6), the range a per-16 amax/6
    scale takes for N(0,1) latents. Valid entries with no encoding step;
    parity tests use the cache-write step's entries instead."""
    rng = np.random.Generator(np.random.PCG64(seed))
    codes = rng.integers(0, 256, size=(B, Lk, Ckv // 2), dtype=np.uint8)
    exp = rng.integers(4, 7, size=(B, Lk, Ckv // 16), dtype=np.uint8)
    mant = rng.integers(0, 8, size=(B, Lk, Ckv // 16), dtype=np.uint8)
    scales = (exp << 3) | mant
    return np.concatenate([codes, scales], axis=-1)


def group_wo_inputs(B: int, H: int, Q: int, Ckv: int = 512, G: int = 8, R: int = 1024, D: int = 4096,
                    seed: int = 6, with_wo_b: bool = True) -> dict:
    """Inputs of the grouped output projection: x (B,H,Q,Ckv) N(0,1); wo_a
    (G,R,(H/G)*Ckv) and wo_b (D,G*R) N(0,1)/sqrt(fan-in); all bf16-rounded."""
    rng = np.random.Generator(np.random.PCG64(seed))
    K1 = (H // G) * Ckv
    out = dict(x=_store(_normal(rng, (B, H, Q, Ckv)), "bf16"),
               wo_a=_store(_normal(rng, (G, R, K1), 1.0 / np.sqrt(K1)), "bf16"))
    out["wo_b"] = _store(_normal(rng, (D, G * R), 1.0 / np.sqrt(G * R)), "bf16") if with_wo_b else None
    return out


def layout_only(name: str, seed: int) -> Workload:
    """The named workload's shapes, lengths and page table without its large
    arrays (q, caches, weights are None): for timing runs that draw those
    arrays on the device. Lengths come from the workload's own first draw;
    the page permutation is drawn right after them (the full workload draws
    it after the arrays, so the two tables differ)."""
    B, H, Q, Lk = {"dsv3_b64_lk4096": (64, 128, 1, 4096), "ragged_paged_b128_q2": (128, 128, 2, 0),
                   "longctx_b4_lk131072": (4, 128, 1, 131072),
                   "v41_fp4_sink_h64": (32, 64, 1, 8192)}[name]
    rng = np.random.Generator(np.random.PCG64(seed))
    w = Workload(name=name, B=B, H=H, Q=Q, Dn=128, Dr=64, Vd=128, Ckv=512, Lk=Lk, dtype="bf16",
                 softmax_scale=1.0 / math.sqrt(192), q_nope=None, q_pe=None, kv_cache=None,
                 pe_cache=None, wkv_b=None)
    if name == "ragged_paged_b128_q2":
        w.seq_lens = rng.integers(512, 16384, size=B, endpoint=True).astype(np.int32)
        w.Lk = int(w.seq_lens.max())
        w.causal = True
        npages = [(int(L) + PAGE_SIZE - 1) // PAGE_SIZE for L in w.seq_lens]
        perm = rng.permutation(int(sum(npages))).astype(np.int32)
        bt = np.full((B, max(npages)), -1, np.int32)
        k = 0
        for b in range(B):
            bt[b, :npages[b]] = perm[k:k + npages[b]]
            k += npages[b]
        w.block_table = bt
    if name == "v41_fp4_sink_h64":
        w.Dn = w.Dr = w.Vd = 0
        w.softmax_scale = 1.0 / math.sqrt(512)
        w.rope_tail = 64
        w.extra["shared_latent"] = True
    return w


WORKLOADS = {
    "demo_fp32": demo_fp32,
    "dsv3_b64_lk4096": dsv3,
    "ragged_paged_b128_q2": ragged_paged,
    "longctx_b4_lk131072": longctx,
    "v41_fp4_sink_h64": v41_shared_latent,
}
