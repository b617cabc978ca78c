"""mla_decode_static_scratch: decode + combine with the library's own scratch array.

This entry point is for callers that may not allocate device memory when
they decode -- a serving engine that reserved nearly all of HBM for its KV
cache at start-up, or a plugin hook that is not allowed to allocate. It takes
no workspace; its split-KV partials live in one library-owned array per GPU.

The test calls it through the C ABI twice in a row, on different inputs,
and compares each result with the existing mla_decode + mla_combine (caller
workspace). Both run the same kernels with the same split count, so the
results must be bit-identical, not merely within the parity tolerance. The
cases cover the bf16 tensor-core decode (contiguous, and paged causal Q = 2),
the generic float32 decode (the question's demo shape with 3 splits) and the
shared-latent FP4 decode with sinks and the inverse-RoPE tail in the merge.
It also checks that the size limit is reported as MLA_ERR_WORKSPACE. The
file sorts last so that a run stopping at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from latent_kv_decode_b200 import workloads as wl

from harness import dev, fp4_entries, upload

pytestmark = pytest.mark.gpu


def _call(w, d, q_lat, splits):
    from latent_kv_decode_b200 import ops
    return ops.make_decode_args(q_lat, d["q_pe"], d["kv"], d["pe"], w.softmax_scale,
                                seq_lens=d["seq_lens"], block_table=d["block_table"],
                                page_size=w.page_size, causal=w.causal, num_splits=splits,
                                causal_mask=d["mask"],
                                Lk=w.Lk if d["block_table"] is None else None)


def _absorbed_case(w, splits):
    """(reference call, static-scratch call) of one absorbed-MLA workload."""
    from latent_kv_decode_b200 import ops
    d = upload(w)
    q_lat = ops.mla_absorb_q(d["q_nope"], d["wkv_b"])
    return _call(w, d, q_lat, splits), _call(w, d, q_lat, splits)


def _shared_latent_case(w, splits):
    from latent_kv_decode_b200 import ops
    q = dev(w.q, torch.bfloat16)
    kv = dev(fp4_entries(w))
    sinks = dev(w.sinks.astype(np.float32))
    mk = lambda: ops.make_decode_args(q, None, kv, None, w.softmax_scale, seq_lens=dev(w.seq_lens),
                                      sinks=sinks, rope_tail=w.rope_tail, rope_theta=w.rope_theta,
                                      num_splits=splits, Lk=w.Lk)
    return mk(), mk()


def test_static_scratch_matches_workspace_path_on_two_calls_in_a_row():
    from latent_kv_decode_b200 import ops
    cases = [
        ("bf16 contiguous", lambda: _absorbed_case(wl.dsv3(B=3, Lk=333, seed=31), 5)),
        ("bf16 paged causal Q=2", lambda: _absorbed_case(
            wl.make_mla(4, 128, 2, 128, 64, 128, 512, 0, dtype="bf16", seed=32, lk_range=(2, 700),
                        paged=True, causal=True), 5)),
        ("fp32 demo", lambda: _absorbed_case(wl.demo_fp32(), 3)),
        ("fp4 shared latent, sinks, rope tail", lambda: _shared_latent_case(
            wl.make_shared_latent(3, 64, 1, 333, seed=34, seq_lens=[333, 64, 200]), 3)),
    ]
    for name, make in cases:
        ref, got = make()
        assert ref.num_splits > 1 and ops.workspace_bytes(ref) > 0   # the scratch is in use
        ops.launch_decode(ref)
        ops.mla_combine(ref)
        ops.mla_decode_static_scratch(got)
        torch.cuda.synchronize()
        assert torch.equal(got.x, ref.x), f"{name}: x differs from the workspace path"
        assert torch.equal(got.lse, ref.lse), f"{name}: lse differs from the workspace path"


def test_static_scratch_rejects_sizes_beyond_its_array():
    from latent_kv_decode_b200 import ops
    w = wl.dsv3(B=1, Lk=64, seed=33)
    d = upload(w)
    q_lat = ops.mla_absorb_q(d["q_nope"], d["wkv_b"])
    call = _call(w, d, q_lat, splits=256)             # 256 splits x 128 rows x 2052 B > 32 MiB
    assert ops.workspace_bytes(call) > (32 << 20)
    L = ops.lib()
    assert L.mla_decode_static_scratch(ctypes.byref(call.args), None) == 3   # MLA_ERR_WORKSPACE
    one = _call(w, d, q_lat, splits=1)                # a single split needs no scratch
    ops.mla_decode_static_scratch(one)
    ref = _call(w, d, q_lat, splits=1)
    ops.launch_decode(ref)
    torch.cuda.synchronize()
    assert torch.equal(one.x, ref.x) and torch.equal(one.lse, ref.lse)
