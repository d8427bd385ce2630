"""GPU parity of the parallel form (retnet_retention_parallel) against the
oracle's parallel form, and against the chunkwise GPU path at full size.

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


def want_parallel(q, k, v, gam, pos0=0, rotate=True, gate=None):
    if rotate:
        q, k = oracle.xpos_rotate(q, pos0), oracle.xpos_rotate(k, pos0)
    o, _ = oracle.retention_parallel(q, k, v, np.float32(gam))
    return o if gate is None else oracle.groupnorm_swish(o, gate)


@pytest.mark.parametrize("n,pos0,rotate", [(128, 0, True), (300, 5, True), (1000, 0, False)])
def test_parallel_form_small(rn, n, pos0, rotate):
    B, H = 2, 3
    q, k, v, _ = wl.make_prefill_inputs(B, H, n, 256, "bf16", 1.0 / 16.0, 80 + n)
    gam = rn.retnet_default_gammas(H)
    got = rn.retnet_retention_parallel(dev(q), dev(k), dev(v), gam, pos0=pos0, rotate=rotate)
    rn.retnet_check_device_errors()
    assert slice_rel_err(host(got), want_parallel(q, k, v, gam, pos0, rotate)) < TOL


def test_parallel_form_gate_many_items(rn):
    # 2 x 4 sequence-heads x 16 row blocks = 128 items with up to 16 key tiles
    B, n, H = 2, 2048, 4
    q, k, v, g = wl.make_prefill_inputs(B, H, n, 256, "bf16", 1.0 / 16.0, 91, hidden=256)
    gam = rn.retnet_default_gammas(H)
    got = rn.retnet_retention_parallel(dev(q), dev(k), dev(v), gam, gate=dev(g))
    rn.retnet_check_device_errors()
    assert slice_rel_err(host(got), want_parallel(q, k, v, gam, gate=g)) < TOL


def test_parallel_matches_chunkwise_long(rn):
    # 7B-like 8k prefill: the parallel form against the chunkwise path
    w = wl.WORKLOADS["long7b"]
    q, k, v = wl.make_prefill_inputs_device(w.batch, w.heads, w.seqlen, w.d, w.scale, w.seed,
                                            torch.device("cuda"))
    gam = rn.retnet_default_gammas(w.heads)
    par = rn.retnet_retention_parallel(q, k, v, gam)
    chk = rn.retnet_retention_chunkwise(q, k, v, gam, w.chunk)
    rn.retnet_check_device_errors()
    assert slice_rel_err(host(par), host(chk)) < TOL


def test_parallel_refuses_fast_decays(rn):
    q, k, v, _ = wl.make_prefill_inputs(1, 2, 128, 256, "bf16", 1.0 / 16.0, 92)
    with pytest.raises(rn.RetnetError):
        rn.retnet_retention_parallel(dev(q), dev(k), dev(v), [0.5, 0.9])


@pytest.mark.parametrize("pairs", [1, 2, 0])
@pytest.mark.parametrize("n", [300, 640, 129])
def test_parallel_form_pairs_and_single(rn, pairs, n):
    # an odd number of 128-row blocks leaves the last CTA pair half empty
    B, H = 1, 2
    q, k, v, g = wl.make_prefill_inputs(B, H, n, 256, "bf16", 1.0 / 16.0, 95 + n, hidden=256)
    gam = rn.retnet_default_gammas(H)
    rn.retnet_set_output_pairing(pairs)
    try:
        got = rn.retnet_retention_parallel(dev(q), dev(k), dev(v), gam, pos0=3, gate=dev(g))
        rn.retnet_check_device_errors()
    finally:
        rn.retnet_set_output_pairing(0)
    assert slice_rel_err(host(got), want_parallel(q, k, v, gam, 3, gate=g)) < TOL
