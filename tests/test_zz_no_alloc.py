"""The allocation-free prefill entry point against the regular one.

retnet_retention_chunkwise_noalloc serves callers that may not allocate
device memory at run time (a plugin in a serving process whose memory is
reserved up front, a latency-critical path that cannot afford cudaMalloc's
device-wide synchronisation): it runs the regular prefill kernels on a
scratch array built into the library.  This file is named to be collected
last; it passes alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from helpers import slice_rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_sequence_02_b200 as rn
    from linear_recurrent_sequence_02_b200.build import build
    build()
    lib = rn.load_library()
    P = ctypes.c_void_p
    lib.retnet_retention_chunkwise_noalloc.restype = ctypes.c_int
    lib.retnet_retention_chunkwise_noalloc.argtypes = [
        P, P, P, P, ctypes.c_int, P, ctypes.POINTER(rn._Shape), ctypes.c_longlong, ctypes.c_int,
        P, P, ctypes.POINTER(rn._Gate), ctypes.c_int, P]
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, q, k, v, gam, chunk, out, state_out, gate, pos0=0):
    import linear_recurrent_sequence_02_b200 as rn
    B, n, H, d = q.shape
    shape = rn._Shape(B, H, n, d, d, rn.BF16 if q.dtype == torch.bfloat16 else rn.F32)
    g = None if gate is None else rn._Gate(gate.data_ptr(), None, None, 1e-5)
    gbuf = (ctypes.c_float * H)(*gam)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.retnet_retention_chunkwise_noalloc(
        _ptr(q), _ptr(k), _ptr(v), gbuf, chunk, _ptr(out), ctypes.byref(shape), pos0, 1, None,
        _ptr(state_out), None if g is None else ctypes.byref(g), 0, stream)


def _inputs(seed, B=1, n=1000, H=2, d=256):
    q, k, v, g = wl.make_prefill_inputs(B, H, n, d, "bf16", 1.0 / 16.0, seed, hidden=256)
    return [torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (q, k, v, g)]


def test_noalloc_matches_regular_entry_point_twice(lib):
    import linear_recurrent_sequence_02_b200 as rn
    chunk = 256
    for seed in (901, 902):                       # two calls in a row, different inputs
        q, k, v, g = _inputs(seed)
        B, n, H, d = q.shape
        gam = rn.retnet_default_gammas(H)
        want_state = torch.empty(B, H, d, d, device="cuda")
        want = rn.retnet_retention_chunkwise(q, k, v, gam, chunk, gate=g, state_out=want_state)
        out = torch.full_like(want, float("nan"))
        state = torch.full_like(want_state, float("nan"))
        assert _noalloc(lib, q, k, v, gam, chunk, out, state, g) == 0
        torch.cuda.synchronize()
        rn.retnet_check_device_errors()
        # the same kernels on the same inputs: the same bits
        assert torch.equal(out, want)
        assert torch.equal(state, want_state)


def test_noalloc_float32_short_chunks_match_regular_entry_point(lib):
    # the float32 CUDA-core path (chunk 64, the tiny configuration's shape)
    # also takes its scratch from the built-in array
    import linear_recurrent_sequence_02_b200 as rn
    q, k, v = wl.make_prefill_inputs(1, 4, 256, 64, "f32", 1.0 / 8.0, 903)[:3]
    q, k, v = (torch.from_numpy(x).cuda() for x in (q, k, v))
    gam = rn.retnet_default_gammas(4)
    want_state = torch.empty(1, 4, 64, 64, device="cuda")
    want = rn.retnet_retention_chunkwise(q, k, v, gam, 64, state_out=want_state)
    for _ in range(2):
        out = torch.full_like(want, float("nan"))
        state = torch.full_like(want_state, float("nan"))
        assert _noalloc(lib, q, k, v, gam, 64, out, state, None) == 0
        torch.cuda.synchronize()
        rn.retnet_check_device_errors()
        assert torch.equal(out, want)
        assert torch.equal(state, want_state)


def test_noalloc_near_its_scratch_limit(lib):
    # the longest two-head bf16 prefill whose tensor-path scratch still fits
    # the 32 MiB array, so the array's last bytes are in use
    import oracle
    import linear_recurrent_sequence_02_b200 as rn
    B, H, d, chunk = 1, 2, 256, 512
    limit = 32 * 1024 * 1024
    n = 128
    while rn.retnet_chunkwise_workspace_size(B, H, n + 128, d, d, torch.bfloat16, chunk,
                                             "tensor") <= limit:
        n += 128
    need = rn.retnet_chunkwise_workspace_size(B, H, n, d, d, torch.bfloat16, chunk, "tensor")
    assert limit - 2 * 1024 * 1024 < need <= limit
    qn, kn, vn, gn = wl.make_prefill_inputs(B, H, n, d, "bf16", 1.0 / 16.0, 904, hidden=256)
    q, k, v, g = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (qn, kn, vn, gn))
    gam = rn.retnet_default_gammas(H)
    want_state = torch.empty(B, H, d, d, device="cuda")
    want = rn.retnet_retention_chunkwise(q, k, v, gam, chunk, gate=g, state_out=want_state)
    out = torch.full_like(want, float("nan"))
    state = torch.full_like(want_state, float("nan"))
    assert _noalloc(lib, q, k, v, gam, chunk, out, state, g) == 0
    torch.cuda.synchronize()
    rn.retnet_check_device_errors()
    assert torch.equal(out, want)
    assert torch.equal(state, want_state)
    y_ref, s_ref = oracle.retention_prefill(qn, kn, vn, np.float32(gam), chunk, gate=gn)
    assert slice_rel_err(out.float().cpu().numpy(), y_ref) < TOL
    assert slice_rel_err(state.cpu().numpy(), s_ref, head_axis=1) < TOL


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    import linear_recurrent_sequence_02_b200 as rn
    # the 200M-layer shape needs ~82 MB of scratch on the tensor path
    B, n, H, d = 8, 2048, 4, 256
    need = rn.retnet_chunkwise_workspace_size(B, H, n, d, d, torch.bfloat16, 512, "tensor")
    assert need > 32 * 1024 * 1024
    shape = rn._Shape(B, H, n, d, d, rn.BF16)
    gbuf = (ctypes.c_float * H)(*rn.retnet_default_gammas(H))
    P = ctypes.c_void_p
    # fake aligned pointers: the call must refuse before touching them
    st = lib.retnet_retention_chunkwise_noalloc(P(256), P(256), P(256), gbuf, 512, P(256),
                                                ctypes.byref(shape), 0, 1, None, None, None, 0,
                                                None)
    assert st == 5                                # RETNET_ERR_WORKSPACE
