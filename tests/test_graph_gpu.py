"""The decode step can be captured in a CUDA graph (its side-stream fork and join
included) and replayed with the same bits as eager steps."""
import pytest
import torch

from linear_attention_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wa():
    from linear_attention_paged_b200 import build
    build.build()
    from linear_attention_paged_b200 import wa as mod
    return mod


def test_step_graph_replay_matches_eager(wa):
    cfg = W.HSAConfig("graph_small", H=2, d=128, T_p=1280, n_c=6, Nq=520, K_p=3, B=64, r=128,
                      dtype="bf16", seed=35, recipe="offset")
    inp = W.make_inputs(cfg, device="cuda")
    step = wa.HSAStep(inp["q"], inp["k_pool"], inp["v_pool"], inp["chunk_pages"], inp["e_k"], inp["e_v"],
                      inp["tau"].cuda(), inp["gate"], cfg.K_p, cfg.B)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step(s)                                   # creates the library's side stream eagerly
    torch.cuda.synchronize()
    ref = step.out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    step.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(step.out, ref)
    # new inputs in the same buffers flow through the replay
    inp["q"].copy_(torch.flip(inp["q"], dims=[0]))
    with torch.cuda.stream(s):
        eager = step(s).clone()
    torch.cuda.synchronize()
    step.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(step.out, eager) and not torch.equal(eager, ref)
    assert wa.wa_device_error() == 0
