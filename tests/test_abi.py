"""CPU checks of the C ABI: the library loads, exports every declared symbol,
and host-side validation rejects bad calls before touching CUDA."""
import ctypes
import os
import re

import numpy as np
import pytest

import linear_recurrent_sequence_02_b200 as rn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "retnet.h")


_DECL = r"RETNET_API[^;(]*?\b(retnet_\w+)\s*\("
_HOOKS_BLOCK = r"#ifdef RETNET_TEST_HOOKS(.*?)#endif"


def declared_functions():
    """Entry points the default library exports (the header minus the
    debug-build-only block)."""
    text = re.sub(_HOOKS_BLOCK, "", open(HEADER).read(), flags=re.S)
    return sorted(set(re.findall(_DECL, text)))


def debug_only_functions():
    blocks = re.findall(_HOOKS_BLOCK, open(HEADER).read(), flags=re.S)
    return sorted(set(re.findall(_DECL, "".join(blocks))))


@pytest.fixture(scope="module")
def lib():
    from linear_recurrent_sequence_02_b200.build import build
    build()
    return rn.load_library()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("retnet_retention_chunkwise", "retnet_retention_step", "retnet_groupnorm_swish",
                 "retnet_xpos_rotate", "retnet_default_gammas", "retnet_chunkwise_workspace_size",
                 "retnet_check_device_errors", "retnet_status_string",
                 "retnet_kernel_launch_count"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    # nothing else leaks out of the shared object under a retnet_ prefix
    out = os.popen(f"nm -D --defined-only {rn.LIB_PATH}").read()
    exported = sorted(set(re.findall(r"\b(retnet_\w+)\b", out)))
    assert exported == declared_functions()


def test_debug_build_exports_the_test_hooks_and_nothing_else_differs(lib):
    from linear_recurrent_sequence_02_b200.build import build
    path = build(variant="debug")
    hooks = debug_only_functions()
    assert hooks == ["retnet_test_error_word", "retnet_test_set_hooks"]
    out = os.popen(f"nm -D --defined-only {path}").read()
    exported = sorted(set(re.findall(r"\b(retnet_\w+)\b", out)))
    assert exported == sorted(declared_functions() + hooks)
    # the default library has no hook
    assert not hasattr(lib, "retnet_test_set_hooks")


def test_status_strings(lib):
    assert rn.retnet_status_string(0) == "ok"
    assert "invalid" in rn.retnet_status_string(1)
    assert rn.retnet_status_string(99) == "unknown status"


def test_default_gammas_match_closed_form(lib):
    g = rn.retnet_default_gammas(16)
    assert g[0] == 0.96875 and g[3] == 0.99609375
    assert g[15] == np.float32(1 - 2.0 ** -20)
    buf = (ctypes.c_float * 1)()
    assert lib.retnet_default_gammas(0, buf) == 1
    assert lib.retnet_default_gammas(257, buf) == 1
    assert lib.retnet_default_gammas(4, None) == 1


def _shape(B=1, H=4, n=256, dk=64, dv=64, dt=0):
    return rn._Shape(B, H, n, dk, dv, dt)


def test_workspace_size_validation(lib):
    n = ctypes.c_size_t(0)
    s = _shape()
    assert lib.retnet_chunkwise_workspace_size(ctypes.byref(s), 64, 1, ctypes.byref(n)) == 0
    assert n.value > 0
    assert lib.retnet_chunkwise_workspace_size(ctypes.byref(s), 0, 1, ctypes.byref(n)) == 1
    assert lib.retnet_chunkwise_workspace_size(ctypes.byref(s), 2048, 1, ctypes.byref(n)) == 1
    bad = _shape(dk=96)
    assert lib.retnet_chunkwise_workspace_size(ctypes.byref(bad), 64, 1, ctypes.byref(n)) == 2
    neg = _shape(B=-1)
    assert lib.retnet_chunkwise_workspace_size(ctypes.byref(neg), 64, 1, ctypes.byref(n)) == 1
    assert lib.retnet_chunkwise_workspace_size(None, 64, 1, ctypes.byref(n)) == 1


def test_tensor_path_takes_short_chunks_as_128(lib):
    # chunks below 128 run on the tensor path with 128-token chunks: the same
    # workspace as chunk 128; 384 (not a tile multiple the path serves) does not
    s = _shape(B=2, H=4, n=1000, dk=256, dv=256, dt=1)
    sizes = {}
    for chunk in (16, 64, 100, 128):
        n = ctypes.c_size_t(0)
        assert lib.retnet_chunkwise_workspace_size(ctypes.byref(s), chunk, 2, ctypes.byref(n)) == 0
        sizes[chunk] = n.value
    assert len(set(sizes.values())) == 1
    n = ctypes.c_size_t(0)
    assert lib.retnet_chunkwise_workspace_size(ctypes.byref(s), 384, 2, ctypes.byref(n)) == 2


def _chunkwise(lib, q=16, k=16, v=16, out=16, gam=(0.9,) * 4, chunk=64, shape=None, pos0=0,
               rotate=1, sin=None, sout=None, algo=1, ws=256, wsb=1 << 30):
    s = shape or _shape()
    g = None if gam is None else (ctypes.c_float * len(gam))(*gam)
    P = ctypes.c_void_p
    return lib.retnet_retention_chunkwise(P(q), P(k), P(v), g, chunk, P(out), ctypes.byref(s),
                                          pos0, rotate, P(sin), P(sout), None, algo, P(ws), wsb,
                                          None)


def test_chunkwise_rejects_before_launch(lib):
    # Fake, aligned, never-dereferenced addresses: every case must fail validation
    assert _chunkwise(lib, q=None) == 1                    # null input
    assert _chunkwise(lib, q=18) == 1                      # misaligned input
    assert _chunkwise(lib, gam=None) == 1                  # no gammas
    assert _chunkwise(lib, gam=(0.9, 0.9, 0.9, 1.5)) == 1  # gamma outside [0, 1]
    assert _chunkwise(lib, gam=(0.9, 0.9, 0.9, float("nan"))) == 1
    assert _chunkwise(lib, chunk=0) == 1
    assert _chunkwise(lib, pos0=-1) == 1
    assert _chunkwise(lib, rotate=2) == 1
    assert _chunkwise(lib, sin=8) == 1                     # misaligned state
    assert _chunkwise(lib, algo=7) == 1
    assert _chunkwise(lib, shape=_shape(dk=80)) == 2       # unsupported head dim
    assert _chunkwise(lib, ws=None) == 5                   # missing workspace
    assert _chunkwise(lib, wsb=16) == 5                    # too small
    assert _chunkwise(lib, ws=272) == 5                    # not 256-byte aligned
    # an empty batch is a no-op that succeeds without touching memory
    assert _chunkwise(lib, q=None, k=None, v=None, out=None, shape=_shape(B=0)) == 0


def test_step_and_groupnorm_reject_before_launch(lib):
    P = ctypes.c_void_p
    g4 = (ctypes.c_float * 4)(0.9, 0.9, 0.9, 0.9)
    assert lib.retnet_retention_step(None, P(16), P(16), g4, P(16), P(16), 2, 4, 64, 64, 0, 0, 1,
                                     None) == 1
    assert lib.retnet_retention_step(P(16), P(16), P(16), g4, P(20), P(16), 2, 4, 64, 64, 0, 0,
                                     1, None) == 1
    assert lib.retnet_retention_step(P(16), P(16), P(16), g4, P(16), P(16), 2, 4, 96, 64, 0, 0,
                                     1, None) == 2
    assert lib.retnet_retention_step(P(16), P(16), P(16), g4, P(16), P(16), 2, 4, 64, 64, 5, 0,
                                     1, None) == 1
    assert lib.retnet_retention_step(P(16), P(16), P(16), None, P(16), P(16), 2, 4, 64, 64, 0, 0,
                                     1, None) == 1
    assert lib.retnet_retention_step(None, None, None, g4, None, None, 0, 4, 64, 64, 0, 0, 1,
                                     None) == 0
    assert lib.retnet_groupnorm_swish(P(16), P(16), None, None, 1e-5, 10, 4, 60, 1, P(16),
                                      None) == 1
    assert lib.retnet_groupnorm_swish(P(16), None, None, None, 1e-5, 10, 4, 64, 1, P(16),
                                      None) == 1
    assert lib.retnet_groupnorm_swish(P(16), P(16), None, None, -1.0, 10, 4, 64, 1, P(16),
                                      None) == 1
    assert lib.retnet_groupnorm_swish(None, None, None, None, 1e-5, 0, 4, 64, 1, None, None) == 0
    assert lib.retnet_xpos_rotate(P(16), P(16), 1, 4, 2, 6, 0, 0, None) == 1    # d % 8 != 0
    assert lib.retnet_xpos_rotate(P(16), P(16), 1, 4, 2, 8, 0, -3, None) == 1   # pos0 < 0


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 4, 2, 8)
    with pytest.raises(ValueError):
        rn.retnet_xpos_rotate(x)


def _parallel(lib, q=1024, k=1024, v=1024, out=1024, gam=(0.9,) * 4, shape=None, pos0=0,
              rotate=1, ws=1024, wsb=1 << 40):
    s = shape or _shape(dk=256, dv=256, dt=1)
    g = None if gam is None else (ctypes.c_float * len(gam))(*gam)
    P = ctypes.c_void_p
    return lib.retnet_retention_parallel(P(q), P(k), P(v), g, P(out), ctypes.byref(s), pos0,
                                         rotate, None, P(ws), wsb, None)


def test_parallel_form_rejects_before_launch(lib):
    n = ctypes.c_size_t(0)
    s = _shape(dk=256, dv=256, dt=1)
    assert lib.retnet_parallel_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
    assert n.value > 0
    f32 = _shape(dk=256, dv=256, dt=0)
    assert lib.retnet_parallel_workspace_size(ctypes.byref(f32), ctypes.byref(n)) == 2
    assert lib.retnet_parallel_workspace_size(None, ctypes.byref(n)) == 1
    # fake, aligned, never-dereferenced addresses: every case fails validation
    assert _parallel(lib, q=None) == 1
    assert _parallel(lib, gam=None) == 1
    assert _parallel(lib, gam=(0.9, 0.9, 0.9, 1.5)) == 1
    assert _parallel(lib, pos0=-1) == 1
    assert _parallel(lib, rotate=3) == 1
    assert _parallel(lib, shape=_shape(dk=64, dv=64, dt=1)) == 2   # tensor path only: d = 256
    assert _parallel(lib, gam=(0.5, 0.9, 0.9, 0.9)) == 2           # decay too fast to fold
    assert _parallel(lib, ws=None) == 5
    assert _parallel(lib, wsb=16) == 5
    assert _parallel(lib, ws=1024 + 256) == 5                      # not 1024-byte aligned
    assert _parallel(lib, q=None, k=None, v=None, out=None, shape=_shape(B=0, dk=256, dv=256,
                                                                         dt=1)) == 0


def test_recurrent_form_rejects_before_launch(lib):
    P = ctypes.c_void_p
    g4 = (ctypes.c_float * 4)(0.9, 0.9, 0.9, 0.9)

    def call(q=16, state=16, shape=None, pos0=0, rotate=1, gam=g4):
        s = shape or _shape(B=2, H=4, n=8, dk=64, dv=64, dt=1)
        return lib.retnet_retention_recurrent(P(q), P(16), P(16), gam, P(state), P(16),
                                              ctypes.byref(s), pos0, rotate, None)

    assert lib.retnet_retention_recurrent(P(16), P(16), P(16), g4, P(16), P(16), None, 0, 1,
                                          None) == 1                       # no shape
    assert call(q=None) == 1
    assert call(q=24) == 1                                                  # misaligned
    assert call(state=None) == 1
    assert call(pos0=-1) == 1
    assert call(rotate=2) == 1
    assert call(gam=None) == 1
    assert call(shape=_shape(B=2, H=4, n=8, dk=96, dv=64, dt=1)) == 2       # head dim
    assert call(shape=_shape(B=2, H=4, n=-1, dk=64, dv=64, dt=1)) == 1
    # an empty run succeeds without touching memory
    assert call(q=None, state=None, shape=_shape(B=2, H=4, n=0, dk=64, dv=64, dt=1)) == 0


def test_backward_rejects_before_launch(lib):
    P = ctypes.c_void_p
    g4 = (ctypes.c_float * 4)(0.9, 0.9, 0.9, 0.9)
    n = ctypes.c_size_t(0)
    s = _shape(B=2, H=4, n=300, dk=256, dv=256, dt=1)
    assert lib.retnet_backward_workspace_size(ctypes.byref(s), 512, 0, ctypes.byref(n)) == 0
    assert n.value > 0
    assert lib.retnet_backward_workspace_size(ctypes.byref(s), 0, 0, ctypes.byref(n)) == 1
    odd = _shape(B=2, H=4, n=300, dk=64, dv=128, dt=1)
    assert lib.retnet_backward_workspace_size(ctypes.byref(odd), 512, 2, ctypes.byref(n)) == 2

    def call(q=1024, dout=1024, dq=1024, shape=None, chunk=512, pos0=0, rotate=1, algo=0,
             gam=g4, ws=1024, wsb=1 << 40):
        sh = shape or s
        return lib.retnet_retention_backward(P(q), P(1024), P(1024), P(dout), gam, chunk, P(dq),
                                             P(1024), P(1024), ctypes.byref(sh), pos0, rotate,
                                             algo, P(ws), wsb, None)

    assert call(q=None) == 1
    assert call(dout=24) == 1                                   # misaligned
    assert call(dq=None) == 1
    assert call(pos0=-1) == 1
    assert call(rotate=2) == 1
    assert call(algo=9) == 1
    assert call(gam=None) == 1
    assert call(chunk=0) == 1
    assert call(shape=_shape(B=2, H=4, n=300, dk=96, dv=256, dt=1)) == 2
    assert call(algo=2, shape=_shape(B=2, H=4, n=300, dk=64, dv=64, dt=1)) == 2
    assert call(ws=None) == 5
    assert call(wsb=64) == 5
    assert call(ws=1024 + 512) == 5                             # not 1024-byte aligned
    assert call(q=None, dout=None, dq=None, shape=_shape(B=0, H=4, n=300, dk=256, dv=256,
                                                         dt=1)) == 0


def test_bindings_refuse_host_tensors(lib):
    """Every binding checks device, dtype and shape before calling the
    library, so no host pointer ever reaches a kernel."""
    import torch
    q = torch.zeros(1, 4, 2, 64)
    gam = [0.9, 0.9]
    state = torch.zeros(1, 2, 64, 64)
    with pytest.raises(ValueError):
        rn.retnet_retention_chunkwise(q, q, q, gam, 64)
    with pytest.raises(ValueError):
        rn.retnet_retention_parallel(q, q, q, gam)
    with pytest.raises(ValueError):
        rn.retnet_retention_recurrent(q, q, q, gam, state, 0)
    with pytest.raises(ValueError):
        rn.retnet_retention_backward(q, q, q, q, gam, 64)
    with pytest.raises(ValueError):
        rn.retnet_retention_step(q[:, 0], q[:, 0], q[:, 0], gam, state, 0)
    with pytest.raises(ValueError):
        rn.retnet_groupnorm_swish(q, q)


def test_bench_work_counts_match_the_formulas():
    """The per-unit figures bench.py divides by are the algorithmic counts
    written out for d = 256 and chunk 512."""
    import bench
    d, C = 256, 512
    assert bench.algorithmic_flops_per_token_head(d, C) == 524_800          # (dk+dv)(C+1) + 4 dk dv
    assert bench.output_kernel_flops_per_token_head(d, C) == 2 * d * (C + 1) + 2 * d * d
    assert bench.state_kernel_flops_per_token_head(d) == 2 * d * d
    assert bench.prep_kernel_bytes_per_token_head(d) == 2048                 # q, k in; Qt, Kt out
    assert bench.parallel_flops_per_token_head(d, 2047) == 2 * d * 2048


def test_bench_output_pass_bytes_at_the_long_prefill():
    """Algorithmic bytes of one output-pass launch at B=1, H=16, n=8192,
    chunk 512: Qt, Kt, V read and O written once (2 B each per element),
    plus S_prev (d x d bf16) for the 15 chunks after the first."""
    import bench
    th = 1 * 16 * 8192
    want = th * 256 * 2 * 4 + 16 * 15 * 256 * 256 * 2
    assert bench.output_kernel_bytes(1, 16, 8192, 256, 512, False) == want == 299_892_736
    # with a gate: G read once more
    assert bench.output_kernel_bytes(1, 16, 8192, 256, 512, True) == want + th * 256 * 2


def test_bench_kernel_hash_covers_its_section_only(tmp_path, monkeypatch):
    """The stored ncu traffic is keyed by a hash of one banner-delimited
    section of a .cu file and the headers: it changes with that section and
    the headers, not with another section."""
    import bench
    csrc = tmp_path / "linear_recurrent_sequence_02_b200" / "csrc"
    csrc.mkdir(parents=True)
    banner = bench.SECTION_BANNER
    (csrc / "k.cu").write_text(f"{banner}alpha\nint a;\n{banner}beta\nint b;\n")
    (csrc / "h.cuh").write_text("int h;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_source_sha("k.cu", "alpha", ["h.cuh"])
    assert base is not None
    (csrc / "k.cu").write_text(f"{banner}alpha\nint a;\n{banner}beta\nint b2;\n")
    assert bench.kernel_source_sha("k.cu", "alpha", ["h.cuh"]) == base
    (csrc / "k.cu").write_text(f"{banner}alpha\nint a2;\n{banner}beta\nint b2;\n")
    assert bench.kernel_source_sha("k.cu", "alpha", ["h.cuh"]) != base
    (csrc / "k.cu").write_text(f"{banner}alpha\nint a;\n{banner}beta\nint b;\n")
    (csrc / "h.cuh").write_text("int h2;\n")
    assert bench.kernel_source_sha("k.cu", "alpha", ["h.cuh"]) != base
    assert bench.kernel_source_sha("k.cu", "gamma", ["h.cuh"]) is None


def test_bench_stored_traffic_matches_the_current_output_pass():
    """The recorded ncu traffic is reported only while its source hash
    matches; it does match the output pass as committed."""
    import bench
    rec = bench.NCU_TRAFFIC[("tc_output", "long7b")]
    assert bench.kernel_source_sha(rec["source"], rec["section"], rec["headers"]) == rec["sha256"]
    assert bench.measured_traffic("tc_output", "long7b") == rec["bytes"]
    assert bench.measured_traffic("tc_output", "layer200m") is None


def test_linear_and_msr_layer_reject_before_launch(lib):
    P = ctypes.c_void_p
    # retnet_linear(x, w, y, rows, in, out, stream)
    assert lib.retnet_linear(None, P(1024), P(1024), 100, 1024, 512, None) == 1
    assert lib.retnet_linear(P(1024), P(1024), P(24), 100, 1024, 512, None) == 1   # misaligned
    assert lib.retnet_linear(P(1024), P(1024), P(1024), -1, 1024, 512, None) == 1
    assert lib.retnet_linear(P(1024), P(1024), P(1024), 100, 1000, 512, None) == 2  # K % 64
    assert lib.retnet_linear(P(1024), P(1024), P(1024), 100, 1024, 300, None) == 2  # N % 256
    assert lib.retnet_linear(None, None, None, 0, 1024, 512, None) == 0             # no rows
    n = ctypes.c_size_t(0)
    s = _shape(B=2, H=4, n=300, dk=256, dv=256, dt=1)
    assert lib.retnet_msr_workspace_size(ctypes.byref(s), 1024, 512, ctypes.byref(n)) == 0
    assert n.value >= 5 * 600 * 1024 * 2
    assert lib.retnet_msr_workspace_size(ctypes.byref(s), 1000, 512, ctypes.byref(n)) == 2
    f32 = _shape(B=2, H=4, n=300, dk=256, dv=256, dt=0)
    assert lib.retnet_msr_workspace_size(ctypes.byref(f32), 1024, 512, ctypes.byref(n)) == 2
    uneq = _shape(B=2, H=4, n=300, dk=256, dv=128, dt=1)
    assert lib.retnet_msr_workspace_size(ctypes.byref(uneq), 1024, 512, ctypes.byref(n)) == 2
    assert lib.retnet_msr_workspace_size(ctypes.byref(s), 1024, 512, None) == 1
    g4 = (ctypes.c_float * 4)(0.9, 0.9, 0.9, 0.9)
    bad = (ctypes.c_float * 4)(0.9, 1.5, 0.9, 0.9)

    def call(x=1024, y=1024, gam=g4, pos0=0, eps=1e-5, ws=1024, wsb=1 << 40, hidden=1024):
        return lib.retnet_msr_layer(P(x), P(1024), P(1024), gam, 512, P(y), ctypes.byref(s),
                                    hidden, pos0, None, None, eps, None, None, P(ws), wsb, None)

    assert call(x=None) == 1
    assert call(y=8) == 1
    assert call(gam=None) == 1
    assert call(gam=bad) == 1
    assert call(pos0=-1) == 1
    assert call(eps=-1.0) == 1
    assert call(hidden=100) == 2
    assert call(ws=None) == 5
    assert call(wsb=1024) == 5
    assert call(ws=1024 + 256) == 5


def test_bench_executed_flops_count_tiles_up_to_the_diagonal():
    # chunk 512 = 4 row blocks of 128: 1 + 2 + 3 + 4 = 10 key tiles per chunk,
    # each 4 * 128 * 256 flops per row (Q K^T and P V), 2.5 tiles per row on
    # average; plus Qt S_prev for 15 of 16 chunks and the state pass's Kt^T V
    import bench
    tiles = 4 * 128 * 256 * (1 + 2 + 3 + 4) / 4
    want = tiles + 2 * 256 * 256 * 15 / 16 + 2 * 256 * 256
    assert bench.executed_flops_per_token_head(256, 512, 8192) == want == 581_632
    # chunks below 128 are computed as 128: one tile per row block
    want64 = 4 * 128 * 256 * 1 + 2 * 256 * 256 * 15 / 16 + 2 * 256 * 256
    assert bench.executed_flops_per_token_head(256, 64, 2048) == want64
    # the parallel form: one chunk of n / 128 row blocks, no state terms
    assert bench.executed_flops_per_token_head(256, 0, 1024, parallel=True) == \
        4 * 128 * 256 * sum(range(1, 9)) / 8
