"""The C-ABI launches under CUDA graph capture: the small launch-bound
configs (RMSNorm f32 4x128x1024, LayerNorm f32 1x1024x768, dual q/k head
RMSNorm at one decode token, "norm_fusion.rs": decode is bound by launches
per token) captured into one graph give the eager calls' bits on replay, and
read their input buffers' current contents on every replay."""
import pytest
import torch

import transformer_row_normalization_b200 as rn
from transformer_row_normalization_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _calls():
    ins = {n: wl.make_inputs(wl.WORKLOADS[n], device="cuda") for n in wl.SMALL_SUITE}
    a, b, d = (ins[n] for n in wl.SMALL_SUITE)
    y1 = torch.empty_like(a["x"])
    y2 = torch.empty_like(b["x"])
    yq, yk = torch.empty_like(d["q"]), torch.empty_like(d["k"])
    e1, e2, ed = (wl.WORKLOADS[n].eps for n in wl.SMALL_SUITE)

    def run():
        rn.rms_norm(a["x"], a["w"], e1, out=y1)
        rn.layer_norm(b["x"], b["w"], b["b"], e2, out=y2)
        rn.dual_head_rms_norm(d["q"], d["k"], d["wq"], d["wk"], ed, out_q=yq, out_k=yk)

    return (a, b, d), (y1, y2, yq, yk), run


def test_graph_replay_matches_eager_bits():
    (a, b, d), outs, run = _calls()
    run()
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    for o in outs:
        o.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for _ in range(2):
        for o in outs:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for o, e in zip(outs, eager):
            assert torch.equal(o, e)
    # new inputs in the same buffers: the replay normalizes them
    gen = torch.Generator(device="cuda").manual_seed(7)
    for t in (a["x"], b["x"], d["q"], d["k"]):
        t.copy_(torch.randn(t.shape, generator=gen, device="cuda").to(t.dtype))
    g.replay()
    torch.cuda.synchronize()
    replayed = [o.clone() for o in outs]
    run()
    torch.cuda.synchronize()
    for o, r in zip(outs, replayed):
        assert torch.equal(o, r)
    del g
