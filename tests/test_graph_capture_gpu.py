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


@pytest.mark.parametrize("chunk", [128, 64])
def test_captured_short_chunk_prefill_chain_replays_bit_exact(rn, chunk):
    """The 200M-layer prefill at chunk 128 (and 64, computed with 128-token
    chunks) as a chain of steps, each continuing the previous step's state,
    captured once and replayed three times: every replay gives the bits of
    the same calls made one by one.  One output work item per chunk makes
    every item end on the cross-chunk product, right before the next item
    copies its queries into tensor memory."""
    w = wl.WORKLOADS["layer200m"]
    B, n, H, d = w.batch, w.seqlen, w.heads, w.d
    gam = rn.retnet_default_gammas(H)
    sets = []
    for i in range(3):
        q, k, v = wl.make_prefill_inputs_device(B, H, n, d, w.scale, w.seed + 13 * i, "cuda")
        gen = torch.Generator(device="cuda")
        gen.manual_seed(w.seed + 13 * i + 1)
        g = (torch.randn(B, n, H, d, generator=gen, device="cuda") * 0.6).to(torch.bfloat16)
        sets.append((q, k, v, g))
    steps = 4
    wsb = rn.retnet_chunkwise_workspace_size(B, H, n, d, d, torch.bfloat16, chunk, "tensor")
    ws = rn.retnet_workspace(wsb, "cuda")

    def chain(ys, states):
        for i in range(steps):
            q, k, v, g = sets[i % 3]
            rn.retnet_retention_chunkwise(q, k, v, gam, chunk, pos0=i * n,
                                          state_in=None if i == 0 else states[i - 1],
                                          state_out=states[i], gate=g, out=ys[i], workspace=ws,
                                          algo="tensor")

    def buffers(fill):
        ys = [torch.full((B, n, H, d), fill, dtype=torch.bfloat16, device="cuda")
              for _ in range(steps)]
        sts = [torch.full((B, H, d, d), fill, device="cuda") for _ in range(steps)]
        return ys, sts

    ye, se = buffers(0.0)
    chain(ye, se)
    torch.cuda.synchronize()
    rn.retnet_check_device_errors()

    yg, sg = buffers(float("nan"))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        chain(yg, sg)
    for _ in range(3):
        for t in yg + sg:
            t.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        rn.retnet_check_device_errors()
        for a, b in zip(ye + se, yg + sg):
            assert torch.equal(a, b)
    del graph
