"""The public calls inside a CUDA graph: a captured prefill and decode step
replay to the same bits as the same calls made one by one, and the kernel
timer reports the replayed kernels when its events were captured too."""
import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_sequence_02_b200 as lib
    from linear_recurrent_sequence_02_b200.build import build
    build()
    lib.load_library()
    return lib


def _inputs(seed, B=2, n=768, H=3, d=256):
    q, k, v, g = wl.make_prefill_inputs(B, H, n, d, "bf16", 1.0 / 16.0, seed, hidden=256)
    return [torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (q, k, v, g)]


def test_captured_prefill_and_step_replay_bit_exact(rn):
    q, k, v, g = _inputs(71)
    B, n, H, d = q.shape
    gam = rn.retnet_default_gammas(H)
    rng = np.random.default_rng(72)
    qd, kd, vd = (torch.from_numpy(rng.standard_normal((B, H, d)).astype(np.float32) / 16)
                  .to(torch.bfloat16).cuda() for _ in range(3))
    wsb = rn.retnet_chunkwise_workspace_size(B, H, n, d, d, torch.bfloat16, 256, "auto")
    ws = rn.retnet_workspace(wsb, "cuda")

    def run(y, st, o):
        rn.retnet_retention_chunkwise(q, k, v, gam, 256, state_out=st, gate=g, out=y,
                                      workspace=ws)
        rn.retnet_retention_step(qd, kd, vd, gam, st, n, out=o)

    y0 = torch.empty_like(q)
    s0 = torch.empty(B, H, d, d, device="cuda")
    o0 = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
    run(y0, s0, o0)
    torch.cuda.synchronize()

    y1 = torch.full_like(y0, float("nan"))
    s1 = torch.full_like(s0, float("nan"))
    o1 = torch.full_like(o0, float("nan"))
    rn.retnet_profiler_reset()
    rn.retnet_profiler_select("tc_output")
    rn.retnet_profiler_enable(True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run(y1, s1, o1)
    rn.retnet_profiler_enable(False)
    rn.retnet_profiler_select(None)
    graph.replay()
    torch.cuda.synchronize()
    rn.retnet_check_device_errors()
    kern = rn.retnet_profiler_read()
    del graph

    assert torch.equal(y0, y1)
    assert torch.equal(s0, s1)
    assert torch.equal(o0, o1)
    assert set(kern) == {"tc_output"}
    ms, launches = kern["tc_output"]
    assert launches == 1 and ms > 0.0
