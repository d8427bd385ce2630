"""GPU parity of the recurrent form over a run of tokens
(retnet_retention_recurrent: multi-token decode / continuing a sequence by a
short chunk) against the oracle's token-by-token recurrence, plus exact
agreement with the same tokens fed one decode step at a time.

Error measure: worst (batch, head) slice of max|gpu - oracle| / max|oracle|;
bounds 1e-4 for float32 inputs and 2e-2 for bfloat16 inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import slice_rel_err

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def rn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_sequence_02_b200 as lib
    from linear_recurrent_sequence_02_b200.build import build
    build()
    lib.load_library()
    return lib


def dev(x, dtype):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(TORCH_DT[dtype]).cuda()


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def want(q, k, v, gam, S0, pos0, rotate=True):
    if rotate:
        q, k = oracle.xpos_rotate(q, pos0), oracle.xpos_rotate(k, pos0)
    return oracle.retention_recurrent(q, k, v, np.float32(gam), S0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv,T", [(64, 64, 13), (128, 64, 5), (256, 256, 16), (256, 128, 1)])
def test_recurrent_tokens_against_oracle(rn, dtype, dk, dv, T):
    B, H, pos0 = 3, 4, 2049
    rng = np.random.default_rng(dk + dv + T)
    q = wl.normal(rng, (B, T, H, dk), 1.0 / np.sqrt(dk), dtype)
    k = wl.normal(rng, (B, T, H, dk), 1.0 / np.sqrt(dk), dtype)
    v = wl.normal(rng, (B, T, H, dv), 1.0 / np.sqrt(dk), dtype)
    S0 = rng.standard_normal((B, H, dk, dv)).astype(np.float32) * 0.05
    gam = rn.retnet_default_gammas(H)
    S = torch.from_numpy(S0).cuda()
    out = rn.retnet_retention_recurrent(dev(q, dtype), dev(k, dtype), dev(v, dtype), gam, S, pos0)
    torch.cuda.synchronize()
    rn.retnet_check_device_errors()
    o_ref, S_ref = want(q, k, v, gam, S0, pos0)
    assert slice_rel_err(host(out), o_ref) < TOL[dtype]
    assert slice_rel_err(S.cpu().numpy(), S_ref, head_axis=1) < 1e-5


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_recurrent_equals_single_steps_bitwise(rn, dtype):
    B, H, d, T, pos0 = 2, 3, 256, 9, 77
    rng = np.random.default_rng(5)
    q, k, v = (wl.normal(rng, (B, T, H, d), 1.0 / 16.0, dtype) for _ in range(3))
    S0 = torch.from_numpy(rng.standard_normal((B, H, d, d)).astype(np.float32) * 0.05).cuda()
    gam = rn.retnet_default_gammas(H)
    qd, kd, vd = dev(q, dtype), dev(k, dtype), dev(v, dtype)
    Sa = S0.clone()
    out = rn.retnet_retention_recurrent(qd, kd, vd, gam, Sa, pos0)
    Sb = S0.clone()
    steps = [rn.retnet_retention_step(qd[:, t].contiguous(), kd[:, t].contiguous(),
                                      vd[:, t].contiguous(), gam, Sb, pos0 + t)
             for t in range(T)]
    torch.cuda.synchronize()
    assert torch.equal(out, torch.stack(steps, dim=1))
    assert torch.equal(Sa, Sb)


@pytest.mark.parametrize("d,T", [(256, 30), (64, 100)])
def test_recurrent_runs_longer_than_one_launch(rn, d, T):
    """A launch carries the rotation of 3072 / (d/2) tokens (24 at d = 256,
    96 at 64); longer runs take several launches with the state carried in
    memory between them."""
    B, H, pos0 = 2, 2, 300
    rng = np.random.default_rng(d + T)
    q, k, v = (wl.normal(rng, (B, T, H, d), 1.0 / np.sqrt(d), "bf16") for _ in range(3))
    S0 = rng.standard_normal((B, H, d, d)).astype(np.float32) * 0.05
    gam = rn.retnet_default_gammas(H)
    qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    Sa = torch.from_numpy(S0).cuda()
    out = rn.retnet_retention_recurrent(qd, kd, vd, gam, Sa, pos0)
    Sb = torch.from_numpy(S0).cuda()
    steps = [rn.retnet_retention_step(qd[:, t].contiguous(), kd[:, t].contiguous(),
                                      vd[:, t].contiguous(), gam, Sb, pos0 + t)
             for t in range(T)]
    torch.cuda.synchronize()
    assert torch.equal(out, torch.stack(steps, dim=1))
    assert torch.equal(Sa, Sb)
    o_ref, S_ref = want(q, k, v, gam, S0, pos0)
    assert slice_rel_err(host(out), o_ref) < TOL["bf16"]
    assert slice_rel_err(Sa.cpu().numpy(), S_ref, head_axis=1) < 1e-5


def test_prefill_then_recurrent_continuation(rn):
    """A 1000-token chunkwise prefill continued by 24 tokens of the recurrent
    form equals the 1024-token prefill (outputs of the last 24 tokens and
    the final state)."""
    B, H, d, n, T = 2, 4, 256, 1000, 24
    q, k, v, _ = wl.make_prefill_inputs(B, H, n + T, d, "bf16", 1.0 / 16.0, 404)
    gam = rn.retnet_default_gammas(H)
    qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    S_full = torch.empty(B, H, d, d, device="cuda")
    full = rn.retnet_retention_chunkwise(qd, kd, vd, gam, 512, state_out=S_full)
    S = torch.empty(B, H, d, d, device="cuda")
    rn.retnet_retention_chunkwise(qd[:, :n].contiguous(), kd[:, :n].contiguous(),
                                  vd[:, :n].contiguous(), gam, 512, state_out=S)
    tail = rn.retnet_retention_recurrent(qd[:, n:].contiguous(), kd[:, n:].contiguous(),
                                         vd[:, n:].contiguous(), gam, S, n)
    torch.cuda.synchronize()
    assert slice_rel_err(host(tail), host(full[:, n:])) < TOL["bf16"]
    assert slice_rel_err(S.cpu().numpy(), S_full.cpu().numpy(), head_axis=1) < TOL["bf16"]


def test_recurrent_without_rotation_and_edge_decays(rn):
    B, H, d, T = 2, 2, 64, 6
    rng = np.random.default_rng(6)
    q, k, v = (rng.standard_normal((B, T, H, d)).astype(np.float32) for _ in range(3))
    S = torch.zeros(B, H, d, d, device="cuda")
    out = rn.retnet_retention_recurrent(dev(q, "f32"), dev(k, "f32"), dev(v, "f32"), [0.0, 1.0],
                                        S, 0, rotate=False)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.retention_recurrent(q, k, v, [0.0, 1.0], np.zeros((B, H, d, d)))
    assert slice_rel_err(host(out), o_ref) < 1e-5
    assert slice_rel_err(S.cpu().numpy(), S_ref, head_axis=1) < 1e-6


def test_recurrent_more_rows_than_one_grid(rn):
    # 4097 sequences x 16 heads = 65552 (sequence, head) rows, 3 tokens each
    B, H, d, T, pos = 4097, 16, 64, 3, 11
    g = torch.Generator(device="cuda")
    g.manual_seed(12)
    q, k, v = ((torch.randn(B, T, H, d, generator=g, device="cuda") / 8).to(torch.bfloat16)
               for _ in range(3))
    S = torch.randn(B, H, d, d, generator=g, device="cuda") * 0.1
    picks = [0, 2048, 4095, 4096]
    S0 = S[picks].cpu().numpy().astype(np.float64)
    gam = rn.retnet_default_gammas(H)
    o = rn.retnet_retention_recurrent(q, k, v, gam, S, pos)
    torch.cuda.synchronize()
    o_ref, S_ref = want(host(q[picks]), host(k[picks]), host(v[picks]), gam, S0, pos)
    assert slice_rel_err(host(o[picks]), o_ref) < TOL["bf16"]
    assert slice_rel_err(S[picks].cpu().numpy(), S_ref, head_axis=1) < 1e-5


def test_recurrent_empty_run_is_a_no_op(rn):
    S = torch.full((1, 2, 64, 64), 3.0, device="cuda")
    q = torch.empty(1, 0, 2, 64, device="cuda")
    out = rn.retnet_retention_recurrent(q, q, q, [0.9, 0.9], S, 5)
    torch.cuda.synchronize()
    assert out.shape == (1, 0, 2, 64)
    assert bool((S == 3.0).all())
