"""GPU parity: the CUDA library against the CPU oracle on seeded inputs.

Error measure: worst (batch, head) slice of max|gpu - oracle| / max|oracle|
(norm-wise relative error).  Bounds: 1e-4 for float32 inputs, 2e-2 for
bfloat16 inputs with float32 accumulation.
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


# ----------------------------------------------------------------- rotation
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d,pos0", [(8, 0), (64, 5), (256, 8000)])
def test_rotation(rn, dtype, d, pos0):
    B, n, H = 2, 37, 3
    x = wl.normal(np.random.default_rng(1), (B, n, H, d), 1.0, dtype)
    want = oracle.xpos_rotate(x, pos0)
    got = host(rn.retnet_xpos_rotate(dev(x, dtype), pos0))
    tol = 1e-5 if dtype == "f32" else 8e-3     # bf16 output rounding is 2^-9 relative
    assert slice_rel_err(got, want) < tol
    # in place
    t = dev(x, dtype)
    rn.retnet_xpos_rotate(t, pos0, out=t)
    assert np.array_equal(host(t), got)


# ----------------------------------------------------------------- epilogue
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dv", [64, 256, 1024])
@pytest.mark.parametrize("affine", [False, True])
def test_groupnorm_swish(rn, dtype, dv, affine):
    rng = np.random.default_rng(2)
    rows, H = 257, 3
    o = wl.normal(rng, (rows, H, dv), 0.3, dtype) + wl.to_dtype(np.float32(0.1), dtype)
    g = wl.normal(rng, (rows, H, dv), 2.0, dtype)
    w = rng.standard_normal(H * dv).astype(np.float32) if affine else None
    b = rng.standard_normal(H * dv).astype(np.float32) if affine else None
    want = oracle.groupnorm_swish(o, g, None if w is None else w.reshape(H, dv),
                                  None if b is None else b.reshape(H, dv), 1e-5)
    tw = None if w is None else torch.from_numpy(w).cuda()
    tb = None if b is None else torch.from_numpy(b).cuda()
    got = host(rn.retnet_groupnorm_swish(dev(o, dtype), dev(g, dtype), tw, tb, 1e-5))
    err = slice_rel_err(got.reshape(1, rows, H, dv), want.reshape(1, rows, H, dv))
    assert err < (1e-5 if dtype == "f32" else 1e-2), err


# ----------------------------------------------------------------- decode
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("batch", [1, 3])
def test_decode_steps(rn, dtype, d, batch):
    H, steps, pos = 4, 5, 1000
    rng = np.random.default_rng(3)
    q, k, v = (wl.normal(rng, (steps, batch, H, d), 1.0 / np.sqrt(d), dtype) for _ in range(3))
    S0 = rng.standard_normal((batch, H, d, d)).astype(np.float32) * 0.1
    gam = rn.retnet_default_gammas(H)
    S_ref = S0.astype(np.float64)
    S_dev = torch.from_numpy(S0).cuda()
    for s in range(steps):
        qr = oracle.xpos_rotate(q[s][:, None], pos + s)[:, 0]
        kr = oracle.xpos_rotate(k[s][:, None], pos + s)[:, 0]
        o_ref, S_ref = oracle.retention_step(qr, kr, v[s], np.float32(gam), S_ref)
        o = rn.retnet_retention_step(dev(q[s], dtype), dev(k[s], dtype), dev(v[s], dtype), gam,
                                     S_dev, pos + s)
        err = slice_rel_err(host(o)[:, None], o_ref[:, None])
        assert err < TOL[dtype], (s, err)
    serr = slice_rel_err(S_dev.cpu().numpy(), S_ref, head_axis=1)
    assert serr < 1e-5, serr


def test_decode_more_rows_than_one_grid(rn):
    # 4097 sequences x 16 heads = 65552 (sequence, head) rows: more than one
    # launch's grid holds; rows on both sides of the split are checked.
    B, H, d, pos = 4097, 16, 64, 7
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    q, k, v = ((torch.randn(B, H, d, generator=g, device="cuda") / 8).to(torch.bfloat16)
               for _ in range(3))
    S = torch.randn(B, H, d, d, generator=g, device="cuda") * 0.1
    picks = [0, 2048, 4095, 4096]
    S0 = S[picks].cpu().numpy().astype(np.float64)
    gam = rn.retnet_default_gammas(H)
    o = rn.retnet_retention_step(q, k, v, gam, S, pos)
    torch.cuda.synchronize()
    qs, ks, vs = (host(x[picks]) for x in (q, k, v))
    qr = oracle.xpos_rotate(qs[:, None], pos)[:, 0]
    kr = oracle.xpos_rotate(ks[:, None], pos)[:, 0]
    o_ref, S_ref = oracle.retention_step(qr, kr, vs, np.float32(gam), S0)
    assert slice_rel_err(host(o[picks])[:, None], o_ref[:, None]) < TOL["bf16"]
    assert slice_rel_err(S[picks].cpu().numpy(), S_ref, head_axis=1) < 1e-5


def test_decode_without_rotation(rn):
    B, H, d = 2, 2, 64
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((B, H, d)).astype(np.float32) for _ in range(3))
    S = torch.zeros(B, H, d, d, device="cuda")
    o = rn.retnet_retention_step(dev(q, "f32"), dev(k, "f32"), dev(v, "f32"), [0.5, 1.0], S, 0,
                                 rotate=False)
    o_ref, S_ref = oracle.retention_step(q, k, v, [0.5, 1.0], np.zeros((B, H, d, d)))
    assert slice_rel_err(host(o)[:, None], o_ref[:, None]) < 1e-5
    assert slice_rel_err(S.cpu().numpy(), S_ref, head_axis=1) < 1e-6


# ----------------------------------------------------------------- prefill
def run_prefill(rn, q, k, v, dtype, gam, chunk, algo, pos0=0, rotate=True, state_in=None,
                gate=None, weight=None, bias=None, want_state=True):
    B, n, H, dk = q.shape
    dv = v.shape[-1]
    sin = None if state_in is None else torch.from_numpy(state_in.astype(np.float32)).cuda()
    sout = torch.empty(B, H, dk, dv, device="cuda") if want_state else None
    out = rn.retnet_retention_chunkwise(
        dev(q, dtype), dev(k, dtype), dev(v, dtype), gam, chunk, pos0=pos0, rotate=rotate,
        state_in=sin, state_out=sout, gate=None if gate is None else dev(gate, dtype),
        weight=weight, bias=bias, algo=algo)
    torch.cuda.synchronize()
    return host(out), (None if sout is None else sout.cpu().numpy().astype(np.float64))


def tiny_inputs():
    w = wl.WORKLOADS["tiny"]
    q, k, v, _ = wl.make_prefill_inputs(w.batch, w.heads, w.seqlen, w.d, w.dtype, w.scale, w.seed)
    return w, q, k, v


def test_tiny_f32_against_all_three_forms(rn):
    w, q, k, v = tiny_inputs()
    gam = rn.retnet_default_gammas(w.heads)
    g64 = np.float32(gam).astype(np.float64)
    qr, kr = oracle.xpos_rotate(q), oracle.xpos_rotate(k)
    o_par, s_par = oracle.retention_parallel(qr, kr, v, g64)
    o_rec, s_rec = oracle.retention_recurrent(qr, kr, v, g64)
    o_chk, s_chk = oracle.retention_chunkwise(qr, kr, v, g64, w.chunk)
    got, st = run_prefill(rn, q, k, v, "f32", gam, w.chunk, "simt")
    for ref, sref in ((o_par, s_par), (o_rec, s_rec), (o_chk, s_chk)):
        assert slice_rel_err(got, ref) < TOL["f32"]
        assert slice_rel_err(st, sref, head_axis=1) < TOL["f32"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n,chunk", [(1, 64), (63, 64), (200, 64), (300, 128), (129, 1),
                                     (100, 7), (130, 1024)])
def test_simt_ragged_and_chunk_sizes(rn, dtype, n, chunk):
    rng = np.random.default_rng(5)
    B, H, d = 2, 3, 64
    q, k, v = (wl.normal(rng, (B, n, H, d), 0.125, dtype) for _ in range(3))
    gam = [0.5, 0.96875, 1.0]
    want, wstate = oracle.retention_prefill(q, k, v, np.float32(gam), chunk, pos0=3)
    got, st = run_prefill(rn, q, k, v, dtype, gam, chunk, "simt", pos0=3)
    assert slice_rel_err(got, want) < TOL[dtype]
    assert slice_rel_err(st, wstate, head_axis=1) < TOL[dtype]


@pytest.mark.parametrize("dk,dv", [(128, 64), (64, 256), (256, 256)])
def test_simt_head_dims_with_state_and_gate(rn, dk, dv):
    rng = np.random.default_rng(6)
    B, n, H, chunk = 1, 150, 2, 64
    q = wl.normal(rng, (B, n, H, dk), dk ** -0.5, "f32")
    k = wl.normal(rng, (B, n, H, dk), dk ** -0.5, "f32")
    v = wl.normal(rng, (B, n, H, dv), 1.0, "f32")
    g = wl.normal(rng, (B, n, H, dv), 1.0, "f32")
    s0 = rng.standard_normal((B, H, dk, dv)) * 0.05
    gam = [0.9, 0.999]
    want, wst = oracle.retention_prefill(q, k, v, np.float32(gam), chunk, pos0=11,
                                         state_in=s0.astype(np.float32), gate=g)
    got, st = run_prefill(rn, q, k, v, "f32", gam, chunk, "simt", pos0=11, state_in=s0, gate=g)
    assert slice_rel_err(got, want) < TOL["f32"]
    assert slice_rel_err(st, wst, head_axis=1) < TOL["f32"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_simt_and_decode_at_the_maximum_head_count(rn, dtype):
    # 256 heads (the most the library accepts) on the SIMT prefill, then one
    # decode step continuing from its state
    rng = np.random.default_rng(8)
    B, n, H, d, chunk = 1, 70, 256, 64, 64
    q, k, v = (wl.normal(rng, (B, n + 1, H, d), 0.125, dtype) for _ in range(3))
    gam = rn.retnet_default_gammas(H)
    want, wstate = oracle.retention_prefill(q[:, :n], k[:, :n], v[:, :n], np.float32(gam),
                                            chunk, pos0=1)
    got, st = run_prefill(rn, q[:, :n], k[:, :n], v[:, :n], dtype, gam, chunk, "simt", pos0=1)
    assert slice_rel_err(got, want) < TOL[dtype]
    assert slice_rel_err(st, wstate, head_axis=1) < TOL[dtype]
    qr = oracle.xpos_rotate(q[:, n:], 1 + n)[:, 0]
    kr = oracle.xpos_rotate(k[:, n:], 1 + n)[:, 0]
    o_ref, _ = oracle.retention_step(qr, kr, v[:, n], np.float32(gam), wstate)
    s_dev = torch.from_numpy(np.float32(st)).cuda()
    o = rn.retnet_retention_step(dev(q[:, n], dtype), dev(k[:, n], dtype), dev(v[:, n], dtype),
                                 gam, s_dev, 1 + n)
    assert slice_rel_err(host(o)[:, None], o_ref[:, None]) < TOL[dtype]


def test_simt_split_prefill_and_decode_continue(rn):
    rng = np.random.default_rng(8)
    B, n, H, d, m = 2, 160, 2, 64, 96
    q, k, v = (wl.normal(rng, (B, n + 1, H, d), 0.125, "f32") for _ in range(3))
    gam = rn.retnet_default_gammas(H)
    full, sfull = run_prefill(rn, q[:, :n], k[:, :n], v[:, :n], "f32", gam, 64, "simt")
    a, sa = run_prefill(rn, q[:, :m], k[:, :m], v[:, :m], "f32", gam, 64, "simt")
    b, sb = run_prefill(rn, q[:, m:n], k[:, m:n], v[:, m:n], "f32", gam, 64, "simt", pos0=m,
                        state_in=sa)
    assert slice_rel_err(np.concatenate([a, b], axis=1), full) < 1e-5
    assert slice_rel_err(sb, sfull, head_axis=1) < 1e-5
    # one decode step continues the prefill exactly like the recurrence
    S = torch.from_numpy(sfull.astype(np.float32)).cuda()
    o = rn.retnet_retention_step(dev(q[:, n], "f32"), dev(k[:, n], "f32"), dev(v[:, n], "f32"),
                                 gam, S, n)
    want, _ = oracle.retention_recurrent(oracle.xpos_rotate(q), oracle.xpos_rotate(k), v,
                                         np.float32(gam))
    assert slice_rel_err(host(o)[:, None], want[:, n:n + 1]) < TOL["f32"]


def test_empty_sequence_copies_state(rn):
    B, H, d = 2, 2, 64
    s0 = np.random.default_rng(9).standard_normal((B, H, d, d)).astype(np.float32)
    q = np.zeros((B, 0, H, d), np.float32)
    got, st = run_prefill(rn, q, q, q, "f32", [0.9, 0.9], 64, "simt", state_in=s0)
    assert got.shape == (B, 0, H, d)
    assert np.array_equal(st, s0.astype(np.float64))


def test_special_decays_match_textbook(rn):
    rng = np.random.default_rng(10)
    B, n, H, d = 1, 70, 2, 64
    q, k, v = (wl.normal(rng, (B, n, H, d), 0.125, "f32") for _ in range(3))
    got, _ = run_prefill(rn, q, k, v, "f32", [0.0, 1.0], 32, "simt", rotate=False)
    # gamma = 0: o_t = (q_t . k_t) v_t ; gamma = 1: prefix-sum linear attention
    want0 = (q[:, :, 0] * k[:, :, 0]).sum(-1, keepdims=True).astype(np.float64) * v[:, :, 0]
    prefix = np.cumsum(k[:, :, 1, :, None].astype(np.float64) * v[:, :, 1, None, :], axis=1)
    want1 = np.einsum("bnk,bnkv->bnv", q[:, :, 1].astype(np.float64), prefix)
    assert slice_rel_err(got[:, :, 0:1], want0[:, :, None]) < 1e-5
    assert slice_rel_err(got[:, :, 1:2], want1[:, :, None]) < 1e-5
