"""GPU parity of the backward pass (retnet_retention_backward) against the
oracle's gradients of the parallel form through the rotation.

Error measure: worst (batch, head) slice of max|gpu - oracle| / max|oracle|;
bounds 1e-4 for float32 inputs (SIMT path) and 2e-2 for bfloat16 inputs
(tensor-core path when d = 256).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import record, slice_rel_err

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


def check(rn, dtype, B, n, H, dk, dv, chunk, pos0=0, rotate=True, algo="auto", seed=0, gam=None,
          term_scale=False):
    rng = np.random.default_rng(seed)
    q = wl.normal(rng, (B, n, H, dk), 1.0 / np.sqrt(dk), dtype)
    k = wl.normal(rng, (B, n, H, dk), 1.0 / np.sqrt(dk), dtype)
    v = wl.normal(rng, (B, n, H, dv), 1.0 / np.sqrt(dk), dtype)
    do = wl.normal(rng, (B, n, H, dv), 1.0, dtype)
    gam = rn.retnet_default_gammas(H) if gam is None else gam
    dq, dk_, dv_ = rn.retnet_retention_backward(dev(q, dtype), dev(k, dtype), dev(v, dtype),
                                                dev(do, dtype), gam, chunk, pos0=pos0,
                                                rotate=rotate, algo=algo)
    torch.cuda.synchronize()
    rn.retnet_check_device_errors()
    wq, wk, wv = oracle.retention_prefill_backward(q, k, v, np.float32(gam), do, pos0=pos0,
                                                   rotate=rotate)
    scales = (None, None, None)
    if term_scale:
        # Normalise by the size of the terms rather than of the result: the
        # same gradients of |q|, |k|, |v|, |dO| without rotation, which bound
        # every sum of products the result is made of.
        scales = oracle.retention_prefill_backward(np.abs(q), np.abs(k), np.abs(v),
                                                   np.float32(gam), np.abs(do), rotate=False)
    for got, want, scale, name in ((dq, wq, scales[0], "dq"), (dk_, wk, scales[1], "dk"),
                                   (dv_, wv, scales[2], "dv")):
        plain = slice_rel_err(host(got), want)      # recorded for the report either way
        if scale is None:
            err = plain
        else:
            diff = np.abs(host(got) - want).max(axis=(1, 3))
            err = record(float((diff / np.abs(scale).max(axis=(1, 3))).max()), "term-scaled")
        assert err < TOL[dtype], (name, err, plain)


@pytest.mark.parametrize("n,chunk", [(128, 128), (700, 256), (1024, 512)])
def test_backward_tensor_path(rn, n, chunk):
    check(rn, "bf16", 2, n, 3, 256, 256, chunk, pos0=5, algo="tensor", seed=n)


def test_backward_with_the_widest_state_pass(rn):
    # 3 x 13 = 39 sequence-heads: the three retentions' state passes take 256
    # d_v columns per CTA (78 CTAs in one wave on 148 SMs)
    check(rn, "bf16", 3, 300, 13, 256, 256, 128, pos0=2, algo="tensor", seed=77)


def test_backward_tensor_path_no_rotation_ragged(rn):
    check(rn, "bf16", 1, 333, 2, 256, 256, 128, rotate=False, algo="tensor", seed=3)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 256)])
def test_backward_simt_f32(rn, dk, dv):
    check(rn, "f32", 2, 200, 2, dk, dv, 64, pos0=17, seed=dk + dv)


def test_backward_simt_bf16_fast_decay(rn):
    # gamma = 0.5 is outside the tensor path's fold range at chunk 256: AUTO runs SIMT
    check(rn, "bf16", 1, 300, 2, 256, 256, 256, gam=[0.5, 0.9], seed=9)


def test_backward_layer200m_shape(rn):
    # the 200M-layer prefill shape (B = 8, H = 4, n = 2048, d = 256, chunk 512)
    w = wl.WORKLOADS["layer200m"]
    check(rn, "bf16", w.batch, w.seqlen, w.heads, w.d, w.d, w.chunk, algo="auto", seed=11)


@pytest.mark.parametrize("n", [1, 2])
def test_backward_shortest_sequences(rn, n):
    # With one or two tokens each gradient slice is a multiple of one or two
    # dot products; where one nearly cancels, the slice is tiny while the
    # bf16 rounding of the folded operands is set by the size of its terms,
    # so the bf16 case is measured against that size.
    check(rn, "bf16", 3, n, 2, 256, 256, 128, pos0=40, algo="tensor", seed=50 + n,
          term_scale=True)
    check(rn, "f32", 3, n, 2, 64, 128, 64, pos0=40, seed=60 + n)
