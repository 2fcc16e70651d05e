"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports every entry point the header declares, sizes workspaces as
documented and rejects invalid arguments before touching the device.

Invalid-argument calls here use placeholder pointers that must never be
dereferenced: every call is chosen so that host validation rejects it first.
They are skipped when a GPU is visible (the GPU suite covers validation with
real device buffers).
"""
import ctypes
import math
import os
import re

import pytest
import torch

from mixed_precision_int8_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "llmint8.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def _declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LLMINT8_API\s+[\w\s\*]*?\b(llmint8_\w+)\s*\(",
                                 text)))


def test_header_declares_the_entry_points_of_the_boundary():
    names = _declared_functions()
    for required in ("llmint8_prepare_weight", "llmint8_matmul",
                     "llmint8_quantize_rows", "llmint8_workspace_size",
                     "llmint8_status_string"):
        assert required in names
    assert set(names) == set(binding.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_library_has_no_torch_or_oracle_dependency():
    import subprocess
    out = subprocess.run(["ldd", binding.LIB_PATH], capture_output=True,
                         text=True).stdout
    assert "torch" not in out and "oracle" not in out


def test_status_strings(lib):
    for code in range(-8, 1):
        assert binding.status_string(code)
    assert binding.status_string(-3) == "pointer breaks the alignment rules"


def test_workspace_size_formula(lib):
    def a256(x):
        return (x + 255) // 256 * 256

    for s, h, o in [(16, 256, 256), (2048, 4096, 4096), (8, 12288, 49152),
                    (3, 272, 784)]:
        nw = (h + 31) // 32
        state = 256 + a256(4 * ((133144 + 31) // 32))  # status + accumulation bitmask
        kcap = max(h, (h + 63) // 64 * 64)  # outlier tiles: the wide layout's stride
        exp = (state + a256(4 * nw) + a256(4 * (nw + 1)) + a256(4 * h)
               + a256(4 * s) + a256(s * h) + a256(2 * s * kcap) + a256(2 * kcap * o)
               + a256(4 * ((o + 127) // 128)) + a256(4 * 16 * o))
        assert lib.llmint8_workspace_size(s, h, o) == exp
        assert (lib.llmint8_workspace_size_host(s, h, o)
                == exp + a256(2 * s * h) + a256(2 * s * o))
    assert lib.llmint8_workspace_size(-1, 16, 16) == 0
    assert lib.llmint8_decode_max_rows() == 16


needs_no_gpu = pytest.mark.skipif(torch.cuda.is_available(),
                                  reason="placeholder pointers: CPU box only")

FAKE = ctypes.c_void_p(1 << 20)  # 16/256-aligned, never dereferenced


def _weight(h, o, wq=FAKE, aw=FAKE):
    return binding.llmint8_weight(h, o, wq, aw)


def test_wait_selftest_validates_its_arguments_on_the_host(lib):
    state = 17152  # LLMINT8_WORKSPACE_STATE_BYTES
    assert lib.llmint8_wait_selftest(None, state, 10**6, None) == -1
    assert lib.llmint8_wait_selftest(ctypes.c_void_p((1 << 20) + 8), state, 10**6, None) == -3
    assert lib.llmint8_wait_selftest(FAKE, state - 1, 10**6, None) == -4
    assert lib.llmint8_wait_selftest(FAKE, state, 10, None) == -7
    assert lib.llmint8_wait_selftest(FAKE, state, 10**11, None) == -7


@needs_no_gpu
@pytest.mark.parametrize("h,o", [(8, 256), (100, 256), (133160, 256),
                                 (256, 8), (256, 100)])
def test_matmul_rejects_bad_shapes(lib, h, o):
    w = _weight(h, o)
    rc = lib.llmint8_matmul(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE,
                            1 << 40, None)
    assert rc == -2


@needs_no_gpu
def test_matmul_rejects_nulls_alignment_alpha_and_small_workspace(lib):
    w = _weight(256, 256)
    big = 1 << 40
    null_w = _weight(256, 256, wq=None)
    assert lib.llmint8_matmul(FAKE, 4, ctypes.byref(null_w), 6.0, FAKE, FAKE,
                              big, None) == -1
    assert lib.llmint8_matmul(None, 4, ctypes.byref(w), 6.0, FAKE, FAKE,
                              big, None) == -1
    assert lib.llmint8_matmul(ctypes.c_void_p((1 << 20) + 2), 4,
                              ctypes.byref(w), 6.0, FAKE, FAKE, big, None) == -3
    assert lib.llmint8_matmul(FAKE, 4, ctypes.byref(w), 6.0, FAKE,
                              ctypes.c_void_p((1 << 20) + 16), big, None) == -3
    for bad_alpha in (-1.0, math.nan):
        assert lib.llmint8_matmul(FAKE, 4, ctypes.byref(w), bad_alpha, FAKE,
                                  FAKE, big, None) == -7
    need = lib.llmint8_workspace_size(4, 256, 256)
    assert lib.llmint8_matmul(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE,
                              need - 1, None) == -4
    assert lib.llmint8_matmul(FAKE, -1, ctypes.byref(w), 6.0, FAKE, FAKE,
                              big, None) == -2
    # s == 0 is a validated no-op
    assert lib.llmint8_matmul(None, 0, ctypes.byref(w), 6.0, None, None, 0,
                              None) == 0
    # forcing the decode kernel beyond its row limit
    opts = binding.llmint8_matmul_opts()
    opts.path = 2
    assert lib.llmint8_matmul_ex(FAKE, 17, ctypes.byref(w), 6.0, FAKE, FAKE,
                                 big, ctypes.byref(opts), None) == -7
    for bad_path in (-1, binding.PATH_PREFILL_PAIR + 1):
        opts.path = bad_path
        assert lib.llmint8_matmul_ex(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE,
                                     big, ctypes.byref(opts), None) == -7


@needs_no_gpu
def test_prepare_and_quantize_rows_validation(lib):
    w = _weight(256, 256)
    assert lib.llmint8_prepare_weight(None, 256, 256, ctypes.byref(w),
                                      None) == -1
    assert lib.llmint8_prepare_weight(FAKE, 256, 512, ctypes.byref(w),
                                      None) == -2
    assert lib.llmint8_prepare_weight(FAKE, 24, 256, ctypes.byref(w),
                                      None) == -2
    nb = lib.llmint8_quantize_rows_scratch_size(256)
    assert nb > 0
    args = [FAKE, 4, 256, 6.0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, nb, None]
    bad = list(args)
    bad[2] = 250
    assert lib.llmint8_quantize_rows(*bad) == -2
    bad = list(args)
    bad[10] = nb - 1
    assert lib.llmint8_quantize_rows(*bad) == -4
    bad = list(args)
    bad[3] = -0.5
    assert lib.llmint8_quantize_rows(*bad) == -7
    bad = list(args)
    bad[6] = None
    assert lib.llmint8_quantize_rows(*bad) == -1


def test_scale_mode_constants_match_the_header():
    text = open(HEADER).read()
    got = dict(re.findall(r"#define\s+LLMINT8_SCALE_(\w+)\s+(\d+)", text))
    assert int(got["VECTORWISE"]) == binding.SCALE_VECTORWISE
    assert int(got["TENSORWISE"]) == binding.SCALE_TENSORWISE
    wo = dict(re.findall(r"#define\s+LLMINT8_WO_(\w+)\s+(\d+)", text))
    assert (int(wo["SHARED"]), int(wo["BEFORE_GEMM"]), int(wo["EACH_CTA"])) == (
        binding.WO_SHARED, binding.WO_BEFORE_GEMM, binding.WO_EACH_CTA)
    paths = dict(re.findall(r"#define\s+LLMINT8_PATH_(\w+)\s+(\d+)", text))
    assert {k: int(v) for k, v in paths.items()} == {
        "AUTO": binding.PATH_AUTO, "PREFILL": binding.PATH_PREFILL,
        "DECODE": binding.PATH_DECODE, "PREFILL_SINGLE": binding.PATH_PREFILL_SINGLE,
        "PREFILL_PAIR": binding.PATH_PREFILL_PAIR}
    bits = dict(re.findall(r"#define\s+LLMINT8_DEV_(\w+)\s+(0x[0-9a-fA-F]+)", text))
    assert int(bits["TIMEOUT_SELFTEST"], 16) == binding.DEV_TIMEOUT_SELFTEST
    assert int(bits["OUTLIER_CAP"], 16) == binding.DEV_OUTLIER_CAP


@needs_no_gpu
def test_scale_modes_are_validated_on_the_host(lib):
    w = _weight(256, 256)
    assert lib.llmint8_prepare_weight_ex(FAKE, 256, 256, 2, ctypes.byref(w), None) == -7
    nb = lib.llmint8_quantize_rows_scratch_size(256)
    assert lib.llmint8_quantize_rows_ex(FAKE, 4, 256, 6.0, -1, FAKE, FAKE, FAKE, FAKE,
                                        FAKE, FAKE, nb, None) == -7
    big = 1 << 40
    for bad in (2, -1):
        opts = binding.llmint8_matmul_opts()
        opts.x_scale = bad
        assert lib.llmint8_matmul_ex(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE, big,
                                     ctypes.byref(opts), None) == -7
        assert lib.llmint8_matmul_host_ex(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE, big,
                                          ctypes.byref(opts), None) == -7


@needs_no_gpu
def test_noalloc_size_limit_is_checked_on_the_host(lib):
    s, h, o = 16, 4096, 8192
    assert lib.llmint8_workspace_size(s, h, o) > binding.NOALLOC_MAX_SCRATCH_BYTES
    w = _weight(h, o)
    assert lib.llmint8_matmul_noalloc(FAKE, s, ctypes.byref(w), 6.0, FAKE,
                                      None) == -9
    assert lib.llmint8_matmul_noalloc(FAKE, s, ctypes.byref(_weight(h, 24)),
                                      6.0, FAKE, None) == -2


@needs_no_gpu
def test_valid_call_without_a_gpu_reports_cuda_error_not_a_fallback(lib):
    # Arguments pass validation; with no device the library must fail, never
    # compute on the host.
    w = _weight(256, 256)
    need = lib.llmint8_workspace_size(4, 256, 256)
    rc = lib.llmint8_matmul(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE, need,
                            None)
    assert rc in (-5, -8)


def test_workspace_with_an_outlier_cap_is_small_for_the_175b_shapes(lib):
    """max_outliers shrinks the outlier tiles (2*s*cap + 2*cap*o bytes): at
    cap 64 the OPT-175B FFN and decode workspaces are tens of MB, against
    the worst case's 1.2 GB of W^O capacity alone."""
    def a256(x):
        return (x + 255) // 256 * 256

    def kcap(cap):  # more than 16: the wide layout, stride rounded up to 64
        return cap if cap <= 16 else (cap + 63) // 64 * 64

    for s, h, o in [(2048, 12288, 49152), (8, 12288, 49152), (16, 256, 256), (40, 272, 784)]:
        full = lib.llmint8_workspace_size(s, h, o)
        assert lib.llmint8_workspace_size_ex(s, h, o, 0) == full
        assert lib.llmint8_workspace_size_ex(s, h, o, h) == full
        for cap in (1, 16, 17, 64, 100):
            if cap > h:
                continue
            got = lib.llmint8_workspace_size_ex(s, h, o, cap)
            assert got == full - a256(2 * s * kcap(h)) - a256(2 * kcap(h) * o) \
                + a256(2 * s * kcap(cap)) + a256(2 * kcap(cap) * o)
            assert (lib.llmint8_workspace_size_host_ex(s, h, o, cap)
                    == got + a256(2 * s * h) + a256(2 * s * o))
    assert lib.llmint8_workspace_size(2048, 12288, 49152) > 1.2e9
    assert lib.llmint8_workspace_size_ex(2048, 12288, 49152, 64) < 40e6
    assert lib.llmint8_workspace_size_ex(8, 12288, 49152, 64) < 10e6
    assert lib.llmint8_workspace_size_ex(16, 256, 256, -1) == 0
    assert lib.llmint8_workspace_size_ex(16, 256, 256, 257) == 0


@needs_no_gpu
def test_outlier_cap_and_status_word_are_validated_on_the_host(lib):
    w = _weight(256, 256)
    big = 1 << 40
    for bad in (-1, 257):
        opts = binding.llmint8_matmul_opts()
        opts.max_outliers = bad
        assert lib.llmint8_matmul_ex(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE, big,
                                     ctypes.byref(opts), None) == -7
        assert lib.llmint8_matmul_host_ex(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE, big,
                                          ctypes.byref(opts), None) == -7
    # a workspace sized for cap 16 is enough for a call with cap 16 only
    opts = binding.llmint8_matmul_opts()
    opts.max_outliers = 16
    need = lib.llmint8_workspace_size_ex(4, 256, 256, 16)
    opts.status_host = None
    assert lib.llmint8_matmul(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE, need, None) == -4
    # a status word the device cannot address is refused before any work
    word = ctypes.c_int32(0)
    opts.status_host = ctypes.cast(ctypes.pointer(word), ctypes.c_void_p)
    assert lib.llmint8_matmul_ex(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE, need,
                                 ctypes.byref(opts), None) == -7
    n = ctypes.c_int32(0)
    assert lib.llmint8_read_outlier_tiles_ex(FAKE, big, 4, 256, 256, 300, ctypes.byref(n),
                                             None, None, None) == -7
    for bad in (-1, 3):
        opts = binding.llmint8_matmul_opts()
        opts.wo_build = bad
        assert lib.llmint8_matmul_ex(FAKE, 4, ctypes.byref(w), 6.0, FAKE, FAKE, big,
                                     ctypes.byref(opts), None) == -7


def test_prefill_kernel_query_checks_shapes_before_the_device(lib):
    """Bad sizes are LLMINT8_ERR_SHAPE on any host; without a usable GPU a
    valid query is an error code (CUDA or unsupported), never a kernel."""
    assert lib.llmint8_prefill_kernel(-1, 256, 256) == -2
    assert lib.llmint8_prefill_kernel(16, 0, 256) == -2
    assert lib.llmint8_prefill_kernel(16, 256, 0) == -2
    rc = lib.llmint8_prefill_kernel(2048, 4096, 4096)
    if torch.cuda.is_available():
        assert rc in (binding.PATH_PREFILL_SINGLE, binding.PATH_PREFILL_PAIR)
    else:
        assert rc < 0
