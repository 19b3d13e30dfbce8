"""Host-side checks of the C ABI (no GPU): the library loads, exports every
symbol include/hga.h declares, and rejects bad arguments before launching."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hga():
    from long_context_hga_b200 import build
    build.build()
    from long_context_hga_b200 import hga as mod
    return mod


def _declared():
    src = open(os.path.join(ROOT, "include", "hga.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hga_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(hga):
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(hga.LIB, n), n
    assert set(hga.EXPORTED) == set(names)


def test_status_strings(hga):
    for code, name in [(0, "HGA_OK"), (1, "HGA_ERR_INVALID_ARG"),
                       (2, "HGA_ERR_UNSUPPORTED"), (3, "HGA_ERR_CUDA"),
                       (4, "HGA_ERR_DEVICE_CHECK"), (5, "HGA_ERR_TIMEOUT"),
                       (6, "HGA_ERR_IO"), (7, "HGA_ERR_CAPACITY")]:
        assert hga.status_string(code) == name


def test_param_validation(hga):
    P = hga.Params
    ok = P(32, 4, 128, local=512, top_chunks=32, top_groups=64)
    assert hga.validate_params(ok) == 0
    assert hga.validate_params(P(32, 5, 128)) == hga.HGA_ERR_INVALID_ARG
    assert hga.validate_params(P(0, 1, 128)) == hga.HGA_ERR_INVALID_ARG
    assert hga.validate_params(P(8, 2, 96)) == hga.HGA_ERR_UNSUPPORTED
    assert hga.validate_params(P(8, 2, 128, sink=32)) == hga.HGA_ERR_INVALID_ARG
    assert hga.validate_params(P(8, 2, 128, local=100)) == hga.HGA_ERR_INVALID_ARG
    assert hga.validate_params(P(8, 2, 128, chunk=60)) == hga.HGA_ERR_INVALID_ARG
    assert hga.validate_params(P(8, 2, 128, chunk=128, sink=128)) == hga.HGA_ERR_UNSUPPORTED
    assert hga.LIB.hga_validate_params(None) == hga.HGA_ERR_INVALID_ARG
    bad = ok.c()
    bad.dtype = 7
    assert hga.LIB.hga_validate_params(ctypes.byref(bad)) == hga.HGA_ERR_INVALID_ARG
    # fp16 V storage: only with bf16 q/k, and the flag is 0 or 1
    assert hga.validate_params(P(32, 4, 128, v_f16=True)) == 0
    assert hga.validate_params(P(32, 4, 128, dtype="fp32", v_f16=True)) == hga.HGA_ERR_INVALID_ARG
    bad = ok.c()
    bad.v_f16 = 2
    assert hga.LIB.hga_validate_params(ctypes.byref(bad)) == hga.HGA_ERR_INVALID_ARG
    # q_ready is a promise about the stream (0 or 1)
    assert hga.validate_params(P(32, 4, 128, q_ready=True)) == 0
    bad = ok.c()
    bad.q_ready = -1
    assert hga.LIB.hga_validate_params(ctypes.byref(bad)) == hga.HGA_ERR_INVALID_ARG


def test_index_capacity(hga):
    P = hga.Params
    p = P(32, 4, 128, local=512, top_chunks=32, top_groups=64)
    assert hga.index_capacity(p, 65536, 0) == 32
    assert hga.index_capacity(p, 65536, 1) == 64
    pa = P(32, 8, 128, top_chunks=0, top_groups=0)
    assert hga.index_capacity(pa, 32768, 0) == 512
    assert hga.index_capacity(pa, 32768, 1) == 4096
    assert hga.index_capacity(P(2, 1, 64, top_chunks=40), 1024, 0) == 16
    assert hga.index_capacity(p, 65536, 2) == -1
    assert hga.index_capacity(P(3, 2, 128), 1024, 0) == -1


def test_bad_arguments_rejected_before_launch(hga):
    """Host-detected errors return before any CUDA call (so they work here,
    where there is no device) and launch nothing."""
    L, P = hga.LIB, hga.Params
    p = P(8, 2, 128).c()
    pp = ctypes.byref(p)
    n0 = hga.launch_count()
    fake = ctypes.c_void_p(0x1000)
    # segment start not on a block boundary
    assert L.hga_route_chunks(pp, fake, 32, 64, fake, 1024, fake, fake, None) == 1
    # segment beyond the capacity
    assert L.hga_attend(pp, fake, 0, 2000, fake, fake, 1024, fake, fake, fake,
                        None, None) == 1
    # null pointers
    assert L.hga_attend(pp, None, 0, 64, fake, fake, 1024, fake, fake, fake,
                        None, None) == 1
    assert L.hga_route_groups(pp, fake, 0, 64, fake, 1024, None, fake, fake,
                              fake, None) == 1
    # summaries: unaligned start, reversed range, beyond capacity
    assert L.hga_build_summaries(pp, fake, 1024, 8, 64, fake, fake, None) == 1
    assert L.hga_build_summaries(pp, fake, 1024, 128, 64, fake, fake, None) == 1
    assert L.hga_build_summaries(pp, fake, 1024, 0, 2048, fake, fake, None) == 1
    # fp16 V conversion: overlapping (not identical) buffers, unaligned,
    # reversed range, fp32 params
    assert L.hga_convert_v(pp, fake, 1024, 0, 64, ctypes.c_void_p(0x1000 + 256), None) == 1
    assert L.hga_convert_v(pp, ctypes.c_void_p(0x1008), 1024, 0, 64, ctypes.c_void_p(1 << 40),
                           None) == 1
    assert L.hga_convert_v(pp, fake, 1024, 64, 0, ctypes.c_void_p(1 << 40), None) == 1
    p32 = P(8, 2, 128, dtype="fp32").c()
    assert L.hga_convert_v(ctypes.byref(p32), fake, 1024, 0, 64, ctypes.c_void_p(1 << 40),
                           None) == 1
    assert L.hga_convert_v(pp, fake, 1024, 64, 64, ctypes.c_void_p(1 << 40), None) == 0
    # segment commit (summaries + fp16 V): overlapping buffers, unaligned V,
    # fp32 params with a V output, unaligned start, reversed range; without a
    # V output it is hga_build_summaries
    out16 = ctypes.c_void_p(1 << 40)
    assert L.hga_commit(pp, fake, fake, 1024, 0, 64, fake, fake, ctypes.c_void_p(0x1000 + 256),
                        None) == 1
    assert L.hga_commit(pp, fake, ctypes.c_void_p(0x1008), 1024, 0, 64, fake, fake, out16,
                        None) == 1
    assert L.hga_commit(ctypes.byref(p32), fake, fake, 1024, 0, 64, fake, fake, out16, None) == 1
    assert L.hga_commit(pp, fake, fake, 1024, 8, 64, fake, fake, out16, None) == 1
    assert L.hga_commit(pp, fake, fake, 1024, 128, 64, fake, fake, out16, None) == 1
    assert L.hga_commit(pp, fake, None, 1024, 8, 64, fake, fake, None, None) == 1
    assert L.hga_commit(pp, fake, fake, 1024, 64, 64, fake, fake, out16, None) == 0
    # backward: V stored as fp16 is not accepted, unaligned or missing outputs
    p16 = P(8, 2, 128, v_f16=True).c()
    f32 = ctypes.c_void_p(1 << 40)
    assert L.hga_attend_backward(ctypes.byref(p16), fake, 0, 64, fake, fake, 1024, fake, fake,
                                 fake, fake, fake, f32, f32, f32, None) == 1
    assert L.hga_attend_backward(pp, fake, 0, 64, fake, fake, 1024, fake, fake, fake, fake,
                                 fake, ctypes.c_void_p((1 << 40) + 4), f32, f32, None) == 1
    assert L.hga_attend_backward(pp, fake, 0, 64, fake, fake, 1024, fake, fake, fake, None,
                                 fake, f32, f32, f32, None) == 1
    assert L.hga_attend_backward(pp, fake, 32, 64, fake, fake, 1024, fake, fake, fake, fake,
                                 fake, f32, f32, f32, None) == 1
    assert L.hga_attend_backward(pp, None, 0, 0, None, None, 1024, None, None, None, None,
                                 None, None, None, None, None) == 0
    # decode step: position outside the cache, fp16 copy aliasing v, params
    # that already say fp16 V
    assert L.hga_decode_step(pp, fake, 1024, fake, fake, 1024, fake, fake, fake, fake, fake,
                             fake, None, fake, None, None) == 1
    assert L.hga_decode_step(pp, fake, 70, fake, fake, 1024, fake, fake, fake, fake, fake,
                             fake, fake, fake, None, None) == 1
    assert L.hga_decode_step(ctypes.byref(p16), fake, 70, fake, fake, 1024, fake, fake, fake,
                             fake, fake, fake, None, fake, None, None) == 1
    # causal-routing forward: no query buffer, a segment off the block grid
    assert L.hga_forward_causal(pp, None, 64, 64, fake, fake, 1024, fake, fake, fake, fake,
                                fake, fake, fake, None, None) == 1
    assert L.hga_forward_causal(pp, fake, 32, 64, fake, fake, 1024, fake, fake, fake, fake,
                                fake, fake, fake, None, None) == 1
    assert L.hga_forward_causal(pp, None, 64, 0, None, None, 1024, None, None, None, None,
                                None, None, None, None, None) == 0
    # empty work is a no-op, not an error
    assert L.hga_build_summaries(pp, None, 1024, 64, 64, None, None, None) == 0
    assert L.hga_route_chunks(pp, None, 0, 0, None, 1024, None, None, None) == 0
    assert L.hga_attend(pp, None, 0, 0, None, None, 1024, None, None, None,
                        None, None) == 0
    # unsupported head_dim
    p96 = P(8, 2, 96).c()
    assert L.hga_attend(ctypes.byref(p96), fake, 0, 64, fake, fake, 1024, fake,
                        fake, fake, None, None) == 2
    assert hga.launch_count() == n0


def test_product_path_has_no_oracle_import():
    """The package never imports the oracle (test infrastructure only)."""
    pkg = os.path.join(ROOT, "long_context_hga_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.replace("oracle)", ""), f


def test_wait_hooks_reject_bad_arguments(hga):
    """The bounded-wait controls refuse bad values before touching a device."""
    assert hga.LIB.hga_set_wait_limit_ns(999_999) == hga.HGA_ERR_INVALID_ARG
    assert hga.LIB.hga_set_wait_limit_ns(60_000_000_001) == hga.HGA_ERR_INVALID_ARG
    assert hga.LIB.hga_selftest_wait(None, None) == hga.HGA_ERR_INVALID_ARG
    assert hga.LIB.hga_selftest_wait(ctypes.c_void_p(12), None) == hga.HGA_ERR_INVALID_ARG
    assert hga.LIB.hga_debug_stall_next_attend(-2) == hga.HGA_ERR_INVALID_ARG
    assert hga.LIB.hga_debug_stall_next_attend(3) == hga.HGA_OK
    assert hga.LIB.hga_debug_stall_next_attend(-1) == hga.HGA_OK      # cleared again
