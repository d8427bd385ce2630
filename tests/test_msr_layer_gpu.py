"""GPU parity of the projection GEMM (retnet_linear) and of the multi-scale
retention layer (retnet_msr_layer) against the CPU oracle.

bf16 operands, float32 accumulation; error = worst slice of
max|gpu - oracle| / max|oracle| (per sequence for the layer, per output for
the GEMM), bound 2e-2, as for the prefill.
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


@pytest.mark.parametrize("m,k,n", [(128, 64, 256), (1000, 1024, 512), (300, 2560, 2560),
                                   (4097, 1024, 4096), (1, 128, 256), (300, 192, 256),
                                   (513, 64, 512)])
def test_linear_against_oracle(rn, m, k, n):
    # up to 128 rows: single CTAs (128 x 256 tiles); above: CTA pairs (256 x 256),
    # whose stages hold two 64-wide K steps: K = 192 and 64 leave the last
    # stage's second step past the end of K (read as zeros)
    rng = np.random.default_rng(m + k + n)
    x = wl.normal(rng, (m, k), 1.0, "bf16")
    w = wl.normal(rng, (n, k), 1.0 / np.sqrt(k), "bf16")
    y = rn.retnet_linear(dev(x), dev(w))
    rn.retnet_check_device_errors()
    want = oracle.linear(x, w)
    # rows in groups of 64 as the slices
    pad = (-m) % 64
    got = np.concatenate([host(y), np.zeros((pad, n))]).reshape(-1, 64, 1, n)
    ref = np.concatenate([want, np.zeros((pad, n))]).reshape(-1, 64, 1, n)
    assert slice_rel_err(got, ref) < TOL
    # and elementwise against the float32 product of the same bf16 values
    ref32 = torch.from_numpy(x) @ torch.from_numpy(w).T
    assert torch.allclose(y.float().cpu(), ref32, rtol=1e-2, atol=1e-2 * float(ref32.abs().max()))


def test_linear_rows_beyond_the_last_tile_untouched(rn):
    # 200 rows: the second 128-row tile is ragged; rows past 200 of the
    # output buffer must stay as they were
    rng = np.random.default_rng(3)
    x = dev(wl.normal(rng, (200, 256), 1.0, "bf16"))
    w = dev(wl.normal(rng, (256, 256), 1.0 / 16, "bf16"))
    buf = torch.full((256, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    rn.retnet_linear(x, w, out=buf[:200])
    rn.retnet_check_device_errors()
    assert torch.all(buf[200:] == 7.0)


def _layer(rn, B, n, hidden, H, d, chunk, seed, pos0=0, affine=False, state=False):
    x, wqkvg, wo = wl.make_msr_inputs(B, n, hidden, H, d, seed)
    gam = rn.retnet_default_gammas(H)
    rng = np.random.default_rng(seed + 1)
    w = b = s0 = None
    if affine:
        w = rng.standard_normal(H * d).astype(np.float32)
        b = rng.standard_normal(H * d).astype(np.float32)
    if state:
        s0 = (rng.standard_normal((B, H, d, d)) * 0.05).astype(np.float32)
    st = torch.full((B, H, d, d), float("nan"), device="cuda")
    y = rn.retnet_msr_layer(dev(x), dev(wqkvg), dev(wo), gam, chunk, pos0=pos0,
                            weight=None if w is None else torch.from_numpy(w).cuda(),
                            bias=None if b is None else torch.from_numpy(b).cuda(),
                            state_in=None if s0 is None else torch.from_numpy(s0).cuda(),
                            state_out=st)
    rn.retnet_check_device_errors()
    hd = H * d
    want, wstate = oracle.msr_layer(x, wqkvg[:hd], wqkvg[hd:2 * hd], wqkvg[2 * hd:3 * hd],
                                    wqkvg[3 * hd:], wo, np.float32(gam), chunk, pos0=pos0,
                                    state_in=s0,
                                    weight=None if w is None else w.reshape(H, d),
                                    bias=None if b is None else b.reshape(H, d))
    return host(y), want, st.cpu().numpy(), wstate


def test_msr_layer_small_ragged(rn):
    got, want, st, ws = _layer(rn, 2, 700, 512, 2, 256, 256, 31, pos0=4, affine=True,
                               state=True)
    assert slice_rel_err(got[:, :, None], want[:, :, None]) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_msr_layer_head_dim_64_runs_the_simt_retention(rn):
    # d = 64 (H d = 256): the projections on the tensor cores, the retention on SIMT
    got, want, st, ws = _layer(rn, 1, 300, 256, 4, 64, 64, 32)
    assert slice_rel_err(got[:, :, None], want[:, :, None]) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_msr_layer_200m_shape(rn):
    # the 200M layer: B = 8, n = 2048, hidden 1024, H = 4, d = 256, chunk 512
    w = wl.WORKLOADS["layer200m"]
    got, want, st, ws = _layer(rn, w.batch, w.seqlen, w.hidden, w.heads, w.d, w.chunk, 33)
    assert slice_rel_err(got[:, :, None], want[:, :, None]) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_msr_layer_folded_by_the_single_cta_gemm_at_chunk_64(rn):
    # 100 rows: the projection runs on single CTAs, whose epilogue rotates and
    # decay-folds Q and K; chunk 64 is computed with the fold over 128 tokens;
    # a far position exercises the angle reduction
    got, want, st, ws = _layer(rn, 1, 100, 256, 1, 256, 64, 34, pos0=5000, state=True)
    assert slice_rel_err(got[:, :, None], want[:, :, None]) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


@pytest.mark.parametrize("pairs", [1, 2])
def test_msr_layer_folded_operands_on_cta_pairs(rn, pairs):
    # the output pass on CTA pairs; in mode 1 the pairs fold raw q themselves,
    # which the layer's already folded Qt must not go through again
    rn.retnet_set_output_pairing(pairs)
    try:
        got, want, st, ws = _layer(rn, 1, 1100, 256, 2, 256, 512, 35, pos0=17, state=True)
    finally:
        rn.retnet_set_output_pairing(0)
    assert slice_rel_err(got[:, :, None], want[:, :, None]) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_msr_layer_fold_angles_far_and_straddling(rn):
    # The fold forms each row's angle (pos0 + t) theta_j from a table row every
    # 32 positions plus the remainder; n = 1100 is no multiple of 32, so the
    # 32 rows of a warp straddle two table rows, and pos0 = 123457 puts the
    # table's angles far from zero.
    got, want, st, ws = _layer(rn, 2, 1100, 512, 2, 256, 512, 37, pos0=123457, state=True)
    assert slice_rel_err(got[:, :, None], want[:, :, None]) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL


def test_msr_layer_with_the_widest_state_pass(rn):
    # 3 x 13 = 39 sequence-heads (hidden 13 x 256): the prefill's state pass
    # takes 256 d_v columns per CTA, fed by the projection's folded operands
    got, want, st, ws = _layer(rn, 3, 300, 3328, 13, 256, 128, 38, pos0=3, state=True)
    assert slice_rel_err(got[:, :, None], want[:, :, None]) < TOL
    assert slice_rel_err(st, ws, head_axis=1) < TOL
