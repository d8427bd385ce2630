"""The debug build of the library (libretnet_debug.so: index checks that
report through the device error word, and test hooks) on the GPU.

- A pipeline wait that runs out ends the kernel with RETNET_ERR_TIMEOUT and
  leaves the context usable: the hook makes the state pass's first CTA skip
  its first TMA load, so its MMA warp's wait gives up after 1 ms; the CTA
  lets its other loads land, frees its tensor memory and returns.  The next
  call (hooks off) gives the bits of the default library.  Nothing faults,
  traps or waits without a limit.
- The index checks stay quiet on ragged and multi-launch shapes of every
  hot-path kernel, and the debug build computes the same bits as the default
  one.
"""
import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu

TIMEOUT, BOUNDS = 4, 6          # RETNET_ERR_TIMEOUT, RETNET_ERR_BOUNDS


@pytest.fixture(scope="module")
def rn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import linear_recurrent_sequence_02_b200 as lib
    from linear_recurrent_sequence_02_b200.build import build
    build()
    build(variant="debug")
    lib.load_library()
    lib.load_library(lib.DEBUG_LIB_PATH)
    return lib


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).cuda()


def _prefill(rn, q, k, v, gam, chunk, gate=None, state_in=None, pos0=0):
    B, n, H, d = q.shape
    st = torch.full((B, H, d, d), float("nan"), device="cuda")
    y = rn.retnet_retention_chunkwise(q, k, v, gam, chunk, pos0=pos0, gate=gate,
                                      state_in=state_in, state_out=st, algo="tensor")
    return y, st


# (B, H): the state pass at 64, 128 and 256 columns per CTA (6, 20 and 39
# sequence-heads on 148 SMs); the skipped load is in its first CTA
@pytest.mark.parametrize("B,H", [(1, 1), (4, 5), (3, 13)])
def test_timeout_path_reports_and_the_context_stays_usable(rn, B, H):
    q, k, v, _ = (None if x is None else _dev(x)
                  for x in wl.make_prefill_inputs(B, H, 256, 256, "bf16", 1 / 16, 801))
    gam = rn.retnet_default_gammas(H)
    ref_y, ref_s = _prefill(rn, q, k, v, gam, 128)          # default library
    rn.retnet_check_device_errors()
    with rn.using_library(rn.DEBUG_LIB_PATH):
        rn.retnet_check_device_errors()                      # start from a clear word
        rn.retnet_test_set_hooks(1_000_000, True)            # 1 ms limit, skip a load
        try:
            _prefill(rn, q, k, v, gam, 128)
            with pytest.raises(rn.RetnetError) as e:
                rn.retnet_check_device_errors()
            assert e.value.status == TIMEOUT
        finally:
            rn.retnet_test_set_hooks(2_000_000_000, False)
        # the same process and context, hooks off: a normal call, no error
        y, s = _prefill(rn, q, k, v, gam, 128)
        rn.retnet_check_device_errors()
    assert torch.equal(y, ref_y)
    assert torch.equal(s, ref_s)
    # and the default library still works alongside
    y2, s2 = _prefill(rn, q, k, v, gam, 128)
    rn.retnet_check_device_errors()
    assert torch.equal(y2, ref_y) and torch.equal(s2, ref_s)


@pytest.mark.parametrize("B,n,H,chunk", [(2, 1101, 3, 256), (1, 77, 2, 512), (3, 300, 2, 64),
                                         (1, 2048, 16, 512), (4, 700, 5, 256), (3, 300, 13, 128)])
def test_index_checks_quiet_and_bits_equal_prefill(rn, B, n, H, chunk):
    q, k, v, g = (_dev(x) for x in wl.make_prefill_inputs(B, H, n, 256, "bf16", 1 / 16,
                                                          810 + n, hidden=256))
    gam = rn.retnet_default_gammas(H)
    rng = np.random.default_rng(n)
    s0 = torch.from_numpy(rng.standard_normal((B, H, 256, 256)).astype(np.float32) * 0.05).cuda()
    want = _prefill(rn, q, k, v, gam, chunk, gate=g, state_in=s0, pos0=9)
    rn.retnet_check_device_errors()
    with rn.using_library(rn.DEBUG_LIB_PATH):
        got = _prefill(rn, q, k, v, gam, chunk, gate=g, state_in=s0, pos0=9)
        rn.retnet_check_device_errors()                      # raises on a failed check
    assert torch.equal(got[0], want[0])
    assert torch.equal(got[1], want[1])


@pytest.mark.parametrize("tokens", [1, 5, 30])
def test_index_checks_quiet_and_bits_equal_decode(rn, tokens):
    B, H, d = 3, 16, 256
    rng = np.random.default_rng(820 + tokens)
    q, k, v = (torch.from_numpy(rng.standard_normal((B, tokens, H, d)).astype(np.float32) / 16)
               .to(torch.bfloat16).cuda() for _ in range(3))
    s0 = torch.from_numpy(rng.standard_normal((B, H, d, d)).astype(np.float32) * 0.1).cuda()
    gam = rn.retnet_default_gammas(H)

    def run():
        st = s0.clone()
        if tokens == 1:
            o = rn.retnet_retention_step(q[:, 0], k[:, 0], v[:, 0], gam, st, 8192)
        else:
            o = rn.retnet_retention_recurrent(q, k, v, gam, st, 8192)
        return o, st

    want = run()
    rn.retnet_check_device_errors()
    with rn.using_library(rn.DEBUG_LIB_PATH):
        got = run()
        rn.retnet_check_device_errors()
    assert torch.equal(got[0], want[0])
    assert torch.equal(got[1], want[1])


@pytest.mark.parametrize("B,n,chunk", [(1, 100, 64), (2, 700, 256)])
def test_index_checks_quiet_and_bits_equal_msr_layer(rn, B, n, chunk):
    # the layer's projection GEMM (single CTAs at 100 rows, CTA pairs at 1400)
    # with its epilogue rotation and decay fold, and the prefolded prefill
    H, d, hidden = 2, 256, 512
    x, wqkvg, wo = (_dev(a) for a in wl.make_msr_inputs(B, n, hidden, H, d, 830 + n))
    gam = rn.retnet_default_gammas(H)
    rng = np.random.default_rng(n + 1)
    s0 = torch.from_numpy(rng.standard_normal((B, H, d, d)).astype(np.float32) * 0.05).cuda()

    def run():
        st = torch.full((B, H, d, d), float("nan"), device="cuda")
        y = rn.retnet_msr_layer(x, wqkvg, wo, gam, chunk, pos0=11, state_in=s0, state_out=st)
        return y, st

    want = run()
    rn.retnet_check_device_errors()
    with rn.using_library(rn.DEBUG_LIB_PATH):
        got = run()
        rn.retnet_check_device_errors()
    assert torch.equal(got[0], want[0])
    assert torch.equal(got[1], want[1])
