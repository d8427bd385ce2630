"""Programmatic launch overlap changes only when kernels start, never what
they compute: chains of calls that reuse one workspace and hand the state
from call to call give the same bits with the overlap on and off, eagerly
and replayed from a CUDA graph."""
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
    yield lib
    lib.retnet_set_launch_overlap(True)


B, N, H, D = 2, 1024, 3, 256


def _sets(seed):
    out = []
    for s in range(2):
        q, k, v, g = wl.make_prefill_inputs(B, H, N, D, "bf16", 1.0 / 16.0, seed + s, hidden=256)
        out.append([torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (q, k, v, g)])
    qd, kd, vd = wl.make_decode_inputs(B, H, 4, D, "bf16", 1.0 / 16.0, seed + 9)
    dec = [[torch.from_numpy(x[s]).to(torch.bfloat16).cuda() for x in (qd, kd, vd)]
           for s in range(4)]
    return out, dec


def _chain(rn, sets, dec, ws, ys, states, outs):
    """Four prefills sharing one workspace, each continuing the previous
    call's state through two state buffers, each followed by a decode step."""
    gam = rn.retnet_default_gammas(H)
    for i in range(4):
        q, k, v, g = sets[i % 2]
        sin = None if i == 0 else states[(i - 1) % 2]
        rn.retnet_retention_chunkwise(q, k, v, gam, 512, pos0=i * (N + 1), state_in=sin,
                                      state_out=states[i % 2], gate=g, out=ys[i], workspace=ws)
        qd, kd, vd = dec[i]
        rn.retnet_retention_step(qd, kd, vd, gam, states[i % 2], (i + 1) * (N + 1) - 1,
                                 out=outs[i])


def _buffers():
    ys = [torch.full((B, N, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
          for _ in range(4)]
    states = [torch.full((B, H, D, D), float("nan"), device="cuda") for _ in range(2)]
    outs = [torch.full((B, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
            for _ in range(4)]
    return ys, states, outs


def test_chunkwise_chain_same_bits_with_and_without_overlap(rn):
    sets, dec = _sets(301)
    wsb = rn.retnet_chunkwise_workspace_size(B, H, N, D, D, torch.bfloat16, 512, "tensor")
    ws = rn.retnet_workspace(wsb, "cuda")
    results = []
    for overlap, graphed in ((False, False), (True, False), (True, True)):
        rn.retnet_set_launch_overlap(overlap)
        bufs = _buffers()
        if graphed:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                _chain(rn, sets, dec, ws, *bufs)
            graph.replay()
            torch.cuda.synchronize()
            del graph
        else:
            _chain(rn, sets, dec, ws, *bufs)
            torch.cuda.synchronize()
        rn.retnet_check_device_errors()
        results.append(bufs)
    rn.retnet_set_launch_overlap(True)
    ref = results[0]
    for other in results[1:]:
        for a, b in zip(ref, other):
            for x, y in zip(a, b):
                assert not torch.isnan(x.float()).any()
                assert torch.equal(x, y)


def test_parallel_chain_same_bits_with_and_without_overlap(rn):
    sets, _ = _sets(311)
    gam = rn.retnet_default_gammas(H)
    ws = rn.retnet_workspace(rn.retnet_parallel_workspace_size(B, H, N, D, D, torch.bfloat16),
                             "cuda")
    results = []
    for overlap in (False, True):
        rn.retnet_set_launch_overlap(overlap)
        ys = [torch.empty(B, N, H, D, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
        for i in range(4):
            q, k, v, g = sets[i % 2]
            rn.retnet_retention_parallel(q, k, v, gam, gate=g, out=ys[i], workspace=ws)
        torch.cuda.synchronize()
        rn.retnet_check_device_errors()
        results.append(ys)
    rn.retnet_set_launch_overlap(True)
    for x, y in zip(*results):
        assert torch.equal(x, y)


def test_set_launch_overlap_validates(rn):
    assert rn.load_library().retnet_set_launch_overlap(2) == 1
    assert rn.load_library().retnet_set_launch_overlap(1) == 0
