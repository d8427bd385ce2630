"""GPU parity of the tensor-core (tcgen05) prefill against the CPU oracle.

bf16 inputs, f32 accumulation; error = worst (batch, head) slice of
max|gpu - oracle| / max|oracle|, bound 2e-2.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import slice_rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def rn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_sequence_02_b200 as lib
    from linear_recurrent_sequence_02_b200.build import build
    build()
    lib.load_library()
    return lib


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).cuda()


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def run(rn, q, k, v, gam, chunk, algo="tensor", pos0=0, rotate=True, state_in=None, gate=None,
        weight=None, bias=None, want_state=True):
    B, n, H, d = q.shape
    sin = None if state_in is None else torch.from_numpy(np.float32(state_in)).cuda()
    sout = torch.full((B, H, d, d), float("nan"), device="cuda") if want_state else None
    out = rn.retnet_retention_chunkwise(
        dev(q), dev(k), dev(v), gam, chunk, pos0=pos0, rotate=rotate, state_in=sin,
        state_out=sout, gate=None if gate is None else dev(gate), weight=weight, bias=bias,
        algo=algo)
    rn.retnet_check_device_errors()
    return host(out), (None if sout is None else sout.cpu().numpy().astype(np.float64))


def inputs(B, n, H, seed, gate_width=0, d=256):
    return wl.make_prefill_inputs(B, H, n, d, "bf16", 1.0 / 16.0, seed, hidden=gate_width)


def test_single_tile(rn):
    q, k, v, _ = inputs(1, 128, 1, 11)
    gam = rn.retnet_default_gammas(1)
    want, ws = oracle.retention_prefill(q, k, v, np.float32(gam), 128)
    got, st = run(rn, q, k, v, gam, 128)
    assert slice_rel_err(got, want) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


@pytest.mark.parametrize("n,chunk", [(256, 128), (512, 512), (300, 128), (1101, 256),
                                     (640, 512), (2048, 1024), (77, 512), (300, 64),
                                     (517, 16), (1000, 100)])
def test_chunks_and_ragged_lengths(rn, n, chunk):
    B, H = 2, 3
    q, k, v, _ = inputs(B, n, H, 12 + n)
    gam = rn.retnet_default_gammas(H)
    want, ws = oracle.retention_prefill(q, k, v, np.float32(gam), chunk, pos0=5)
    got, st = run(rn, q, k, v, gam, chunk, pos0=5)
    assert slice_rel_err(got, want) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_state_in_gate_affine_no_rotation(rn):
    B, n, H = 2, 700, 2
    q, k, v, g = inputs(B, n, H, 21, gate_width=128)
    rng = np.random.default_rng(22)
    s0 = rng.standard_normal((B, H, 256, 256)) * 0.05
    w = rng.standard_normal(H * 256).astype(np.float32)
    b = rng.standard_normal(H * 256).astype(np.float32)
    gam = [0.9, 0.999]
    want, ws = oracle.retention_prefill(q, k, v, np.float32(gam), 256, rotate=False,
                                        state_in=np.float32(s0), gate=g,
                                        weight=w.reshape(H, 256), bias=b.reshape(H, 256))
    got, st = run(rn, q, k, v, gam, 256, rotate=False, state_in=s0, gate=g,
                  weight=torch.from_numpy(w).cuda(), bias=torch.from_numpy(b).cuda())
    assert slice_rel_err(got, want) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_more_work_items_than_sms(rn):
    # 3 x 4 (sequence, head) x 8 chunks x 2 row blocks = 192 output work items:
    # more than one per SM, so each persistent CTA walks several items.
    B, n, H = 3, 2048, 4
    q, k, v, g = inputs(B, n, H, 61, gate_width=256)
    gam = rn.retnet_default_gammas(H)
    want, ws = oracle.retention_prefill(q, k, v, np.float32(gam), 256, pos0=3, gate=g)
    got, st = run(rn, q, k, v, gam, 256, pos0=3, gate=g)
    assert slice_rel_err(got, want) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


# The state pass splits S into 128 x DVC blocks, one CTA each, with DVC =
# 64, 128 or 256 chosen from the number of sequence-heads and the SM count
# (148 on B200): 2 x 3 sequence-heads take 64 columns, 4 x 5 take 128, 3 x 13
# take 256 (one wave of 78 CTAs), 5 x 16 take 256 over two waves.
@pytest.mark.parametrize("B,H", [(2, 3), (4, 5), (3, 13), (5, 16)])
@pytest.mark.parametrize("n,chunk", [(300, 128), (700, 256)])
def test_state_pass_widths(rn, B, H, n, chunk):
    q, k, v, _ = inputs(B, n, H, 71 + B * H + n)
    rng = np.random.default_rng(72 + n)
    s0 = rng.standard_normal((B, H, 256, 256)) * 0.05
    gam = rn.retnet_default_gammas(H)
    want, ws = oracle.retention_prefill(q, k, v, np.float32(gam), chunk, pos0=9,
                                        state_in=np.float32(s0))
    got, st = run(rn, q, k, v, gam, chunk, pos0=9, state_in=s0)
    assert slice_rel_err(got, want) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_tensor_matches_simt_path(rn):
    B, n, H = 1, 1024, 4
    q, k, v, g = inputs(B, n, H, 31, gate_width=256)
    gam = rn.retnet_default_gammas(H)
    a, sa = run(rn, q, k, v, gam, 512, algo="tensor", gate=g)
    b, sb = run(rn, q, k, v, gam, 512, algo="simt", gate=g)
    assert slice_rel_err(a, b) < TOL
    assert slice_rel_err(sa, sb, head_axis=1) < TOL


def test_auto_picks_simt_outside_fold_range(rn):
    # gamma = 0.5 with chunk 512 is outside the decay fold's range: AUTO falls
    # back to SIMT, an explicit tensor request is refused.
    q, k, v, _ = inputs(1, 256, 2, 41)
    gam = [0.5, 0.9]
    want, _ = oracle.retention_prefill(q, k, v, np.float32(gam), 512)
    got, _ = run(rn, q, k, v, gam, 512, algo="auto")
    assert slice_rel_err(got, want) < TOL
    with pytest.raises(rn.RetnetError):
        run(rn, q, k, v, gam, 512, algo="tensor")


def test_split_prefill_through_state(rn):
    B, n, H, m = 2, 1536, 2, 640
    q, k, v, _ = inputs(B, n, H, 51)
    gam = rn.retnet_default_gammas(H)
    full, sfull = run(rn, q, k, v, gam, 512)
    a, sa = run(rn, q[:, :m], k[:, :m], v[:, :m], gam, 512)
    b, sb = run(rn, q[:, m:], k[:, m:], v[:, m:], gam, 512, pos0=m, state_in=sa)
    assert slice_rel_err(np.concatenate([a, b], axis=1), full) < TOL
    assert slice_rel_err(sb, sfull, head_axis=1) < TOL


# ------------------------------------------------------- full-size workloads
@pytest.mark.parametrize("name", ["layer200m", "layer3b"])
def test_layer_workloads_full(rn, name):
    w = wl.WORKLOADS[name]
    q, k, v, g = wl.make_prefill_inputs(w.batch, w.heads, w.seqlen, w.d, w.dtype, w.scale,
                                        w.seed, hidden=w.hidden)
    gam = rn.retnet_default_gammas(w.heads)
    want, ws = oracle.retention_prefill(q, k, v, np.float32(gam), w.chunk, gate=g)
    got, st = run(rn, q, k, v, gam, w.chunk, algo="auto", gate=g)
    assert slice_rel_err(got, want) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


@pytest.mark.parametrize("algo", ["tensor", "simt"])
def test_layer200m_chunk64(rn, algo):
    # chunk 64: the tensor path computes it with 128-token chunks (the result
    # does not depend on the chunk length); the SIMT path uses 64 as given
    w = wl.WORKLOADS["layer200m"]
    q, k, v, g = wl.make_prefill_inputs(2, w.heads, w.seqlen, w.d, w.dtype, w.scale, w.seed,
                                        hidden=w.hidden)
    gam = rn.retnet_default_gammas(w.heads)
    want, ws = oracle.retention_prefill(q, k, v, np.float32(gam), 64, gate=g)
    got, st = run(rn, q, k, v, gam, 64, algo=algo, gate=g)
    assert slice_rel_err(got, want) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_long7b_full(rn):
    w = wl.WORKLOADS["long7b"]
    q, k, v, _ = wl.make_prefill_inputs(w.batch, w.heads, w.seqlen, w.d, w.dtype, w.scale, w.seed)
    gam = rn.retnet_default_gammas(w.heads)
    want, ws = oracle.retention_prefill(q, k, v, np.float32(gam), w.chunk)
    got, st = run(rn, q, k, v, gam, w.chunk, algo="auto")
    assert slice_rel_err(got, want) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_decode7b_after_long_prefill(rn):
    """State from an 8192-token prefill, then 256 decode steps.

    The post-prefill state is checked against the oracle at batch 1 and 8
    (sampled sequences); decode outputs and the final state are checked for
    sampled sequences at every batch, the oracle continuing from the GPU's
    post-prefill state.
    """
    w = wl.WORKLOADS["decode7b"]
    H, d, n = w.heads, w.d, w.seqlen
    gam = rn.retnet_default_gammas(H)
    g64 = np.float32(gam).astype(np.float64)
    for batch in w.decode_batches:
        q, k, v = wl.make_prefill_inputs_device(batch, H, n, d, w.scale, w.seed, "cuda")
        sample = [0] if batch == 1 else [0, batch // 3, batch - 1]
        state = torch.empty(batch, H, d, d, device="cuda")
        rn.retnet_retention_chunkwise(q, k, v, gam, w.chunk, state_out=state)
        torch.cuda.synchronize()
        if batch <= 8:
            hq, hk, hv = (host(x[sample]) for x in (q, k, v))
            _, s_ref = oracle.retention_prefill(hq, hk, hv, g64, w.chunk)
            assert slice_rel_err(state.cpu().numpy()[sample], s_ref, head_axis=1) < TOL
        del q, k, v
        S = state.cpu().numpy()[sample].astype(np.float64)
        qd, kd, vd = wl.make_decode_inputs(batch, H, w.decode_steps, d, "bf16", w.scale,
                                           w.seed + 7)
        worst = 0.0
        for s in range(w.decode_steps):
            o = rn.retnet_retention_step(dev(qd[s]), dev(kd[s]), dev(vd[s]), gam, state, n + s)
            qr = oracle.xpos_rotate(qd[s][sample][:, None], n + s)[:, 0]
            kr = oracle.xpos_rotate(kd[s][sample][:, None], n + s)[:, 0]
            o_ref, S = oracle.retention_step(qr, kr, vd[s][sample], g64, S)
            worst = max(worst, slice_rel_err(host(o)[sample][:, None], o_ref[:, None]))
        assert worst < TOL, (batch, worst)
        assert slice_rel_err(state.cpu().numpy()[sample], S, head_axis=1) < TOL
        del state
        torch.cuda.empty_cache()


@pytest.mark.parametrize("pairs", [1, 2, 0])
@pytest.mark.parametrize("B,n,H,chunk", [(2, 1101, 3, 256), (1, 2048, 2, 1024), (2, 640, 2, 512),
                                         (1, 77, 1, 512), (3, 1500, 2, 512)])
def test_output_pass_on_pairs_and_single(rn, pairs, B, n, H, chunk):
    # the same prefill through the paired and the single-CTA output pass:
    # state in, gate with affine, ragged last chunk
    q, k, v, g = inputs(B, n, H, 70 + n, gate_width=128)
    rng = np.random.default_rng(n)
    s0 = rng.standard_normal((B, H, 256, 256)) * 0.05
    w = rng.standard_normal(H * 256).astype(np.float32)
    b = rng.standard_normal(H * 256).astype(np.float32)
    gam = rn.retnet_default_gammas(H)
    want, ws = oracle.retention_prefill(q, k, v, np.float32(gam), chunk, pos0=7,
                                        state_in=np.float32(s0), gate=g,
                                        weight=w.reshape(H, 256), bias=b.reshape(H, 256))
    rn.retnet_set_output_pairing(pairs)
    try:
        got, st = run(rn, q, k, v, gam, chunk, pos0=7, state_in=s0, gate=g,
                      weight=torch.from_numpy(w).cuda(), bias=torch.from_numpy(b).cuda())
    finally:
        rn.retnet_set_output_pairing(0)
    assert slice_rel_err(got, want) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_maximum_head_count(rn):
    # 256 heads, the most the library accepts: the decay constants reach
    # gamma = 1 in float32, the state pass runs several waves of CTAs and the
    # output pass more items than it has CTAs; n = 300 leaves a ragged chunk.
    B, n, H = 1, 300, 256
    q, k, v, _ = inputs(B, n, H, 81)
    gam = rn.retnet_default_gammas(H)
    assert gam[-1] == 1.0
    want, ws = oracle.retention_prefill(q, k, v, np.float32(gam), 128, pos0=2)
    got, st = run(rn, q, k, v, gam, 128, pos0=2)
    assert slice_rel_err(got, want) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL
