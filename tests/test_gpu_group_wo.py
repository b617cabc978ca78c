"""GPU parity of mla_group_wo (the grouped low-rank W_O after the inverse RoPE)
against the fp64 oracle, through the C ABI. z is rounded to bf16 between the
two factors on the GPU; the oracle keeps fp64, so the bf16 tolerance applies."""
import numpy as np
import pytest
import torch

from latent_kv_decode_b200 import workloads as wl
from oracle import v41 as ov41

from harness import REL_L2_BF16, TOL_BF16, assert_close, dev, fp4_entries, gpu_shared_latent

pytestmark = pytest.mark.gpu


def _run(inp, **kw):
    from latent_kv_decode_b200 import ops
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = dev(inp["x"], torch.bfloat16)
    wa = dev(inp["wo_a"], torch.bfloat16)
    wb = dev(inp["wo_b"], torch.bfloat16) if inp["wo_b"] is not None else None
    y = ops.mla_group_wo(x, wa, wb, err_flag=err, **kw)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return y.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("B,H,Q,C,G,R,D", [
    (3, 16, 2, 128, 4, 128, 256),      # several groups, Q = 2, six tokens
    (5, 8, 1, 64, 8, 256, 128),        # one head per group
    (2, 8, 3, 64, 1, 128, 384),        # one group, Q = 3 (token blocks of 48 rows)
])
def test_group_wo_small(B, H, Q, C, G, R, D):
    inp = wl.group_wo_inputs(B, H, Q, C, G, R, D, seed=31)
    y = _run(inp)
    ref = ov41.grouped_wo(inp["x"], inp["wo_a"], inp["wo_b"])
    assert_close(y, ref, TOL_BF16, "y", REL_L2_BF16)


def test_group_wo_without_shared_factor():
    inp = wl.group_wo_inputs(4, 16, 1, 128, 4, 256, 0, seed=32, with_wo_b=False)
    y = _run(inp)
    ref = ov41.grouped_wo(inp["x"], inp["wo_a"])
    assert y.shape == (4, 1, 4 * 256)
    assert_close(y, ref, TOL_BF16, "z", REL_L2_BF16)


def test_group_wo_token_blocks_with_ragged_tail():
    # 300 tokens: two blocks of up to 256, the second read past the end (zero fill)
    inp = wl.group_wo_inputs(300, 8, 1, 64, 2, 128, 128, seed=33)
    y = _run(inp)
    ref = ov41.grouped_wo(inp["x"], inp["wo_a"], inp["wo_b"])
    assert_close(y, ref, TOL_BF16, "y", REL_L2_BF16)


def test_group_wo_full_size_v41():
    """The V4.1-Flash shape: B = 32 tokens, H = 64, Ckv = 512, 8 groups x 1024, D = 4096."""
    inp = wl.group_wo_inputs(32, 64, 1, 512, 8, 1024, 4096, seed=34)
    y = _run(inp)
    ref = ov41.grouped_wo(inp["x"], inp["wo_a"], inp["wo_b"])
    assert_close(y, ref, TOL_BF16, "y", REL_L2_BF16)


def test_group_wo_after_shared_latent_decode():
    """The path's tail: FP4 shared-latent decode (sink, inverse RoPE) then the grouped W_O."""
    w = wl.make_shared_latent(2, 64, 1, 300, seed=35, seq_lens=[300, 177])
    ent = fp4_entries(w)
    g = gpu_shared_latent(w, ent, num_splits=1)
    ref_x = ov41.shared_latent_decode(w.q, ent, w.sinks, w.softmax_scale, w.seq_lens, w.causal,
                                      tail=w.rope_tail, theta=w.rope_theta)
    inp = wl.group_wo_inputs(2, 64, 1, 512, 8, 1024, 512, seed=36)
    inp["x"] = wl.bf16_round(g["x"])                  # the GPU's decode output, as the next step sees it
    y = _run(inp)
    ref = ov41.grouped_wo(ref_x, inp["wo_a"], inp["wo_b"])
    assert_close(y, ref, TOL_BF16, "y", REL_L2_BF16)
