"""mla_decode_static_scratch: decode + combine with the library's own scratch array.

This entry point is for callers that may not allocate device memory when
they decode -- a serving engine that reserved nearly all of HBM for its KV
cache at start-up, or a plugin hook that is not allowed to allocate. It takes
no workspace; its split-KV partials live in one library-owned array per GPU.

The test calls it through the C ABI twice in a row, on two different inputs,
and compares each result with the existing mla_decode + mla_combine (caller
workspace) within the bf16 tolerance of the parity tests. It also checks the
size limit is reported as MLA_ERR_WORKSPACE. The file sorts last so that a
run stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from latent_kv_decode_b200 import workloads as wl

from harness import TOL_BF16, REL_L2_BF16, assert_close, upload

pytestmark = pytest.mark.gpu


def _call(w, d, q_lat, splits):
    from latent_kv_decode_b200 import ops
    return ops.make_decode_args(q_lat, d["q_pe"], d["kv"], d["pe"], w.softmax_scale,
                                seq_lens=d["seq_lens"], block_table=d["block_table"],
                                page_size=w.page_size, causal=w.causal, num_splits=splits,
                                Lk=w.Lk if d["block_table"] is None else None)


def _f(t):
    return t.float().cpu().numpy().astype(np.float64)


def test_static_scratch_matches_workspace_path_on_two_calls_in_a_row():
    from latent_kv_decode_b200 import ops
    cases = [wl.dsv3(B=3, Lk=333, seed=31),
             wl.make_mla(4, 128, 2, 128, 64, 128, 512, 0, dtype="bf16", seed=32, lk_range=(2, 700),
                         paged=True, causal=True)]
    for w in cases:
        d = upload(w)
        q_lat = ops.mla_absorb_q(d["q_nope"], d["wkv_b"])
        ref = _call(w, d, q_lat, splits=5)
        assert ref.num_splits == 5 and ops.workspace_bytes(ref) > 0   # the scratch is in use
        ops.launch_decode(ref)
        ops.mla_combine(ref)
        got = _call(w, d, q_lat, splits=5)
        ops.mla_decode_static_scratch(got)
        torch.cuda.synchronize()
        assert_close(_f(got.x), _f(ref.x), TOL_BF16, f"{w.name} x", REL_L2_BF16)
        assert_close(_f(got.lse), _f(ref.lse), TOL_BF16, f"{w.name} lse")


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
    assert_close(_f(one.x), _f(ref.x), TOL_BF16, "x, one split")
