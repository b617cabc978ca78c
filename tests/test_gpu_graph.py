"""A whole step captured in a CUDA graph and replayed gives bit-identical
results to the eagerly launched step (same kernels, same inputs)."""
import os
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


@pytest.mark.parametrize("name,splits", [("dsv3_b8_lk1024", 0), ("dsv3_b4_lk700", 3)])
def test_graph_replay_equals_eager_step(name, splits):
    import bench
    dev = torch.device("cuda", 0)
    w = bench.layout_workload(name, 0)
    r = bench.StepRunner(w, dev, seed=7, num_splits=splits)
    st = torch.cuda.current_stream()
    r.step(st)
    torch.cuda.synchronize()
    eager_out = r.slots[0]["out"].clone()
    eager_x = r.slots[0]["call"].x.clone()
    r.slots[0]["out"].zero_()
    r.slots[0]["call"].x.zero_()
    g = bench.capture_step(r, st)
    r.slots[0]["out"].zero_()
    r.slots[0]["call"].x.zero_()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(r.slots[0]["call"].x, eager_x)
    assert torch.equal(r.slots[0]["out"], eager_out)
    assert r.num_splits == (splits if splits else r.num_splits)
