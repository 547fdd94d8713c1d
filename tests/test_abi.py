"""The C ABI library loads, exports every symbol ``include/gg.h`` declares, and rejects bad
host-visible arguments before touching a GPU. Runs without a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gg.h")


@pytest.fixture(scope="module")
def lib():
    from moe_grouped_gemm_ragged_b200 import _build
    _build.build()
    import moe_grouped_gemm_ragged_b200 as gg
    return gg.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"GG_API\s+[\w\s\*]+?\b(gg_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"gg_forward", "gg_dgrad", "gg_wgrad", "gg_masked_forward",
            "gg_status_string"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_has_sm100a_code_only():
    from moe_grouped_gemm_ragged_b200 import _build
    assert "arch=compute_100a,code=sm_100a" in " ".join(_build.NVCC_FLAGS)


def test_status_strings(lib):
    import moe_grouped_gemm_ragged_b200 as gg
    assert gg.status_string(0) == "GG_OK"
    for c in (1, 2, 3):
        assert gg.status_string(c).startswith("GG_ERR_")
    assert gg.version() >= 100


def test_host_argument_checks_need_no_gpu(lib):
    f = lib.gg_forward
    # null offsets, bad E, bad sizes -> invalid argument
    assert f(None, None, None, None, 10, 8, 8, 1, None, None) == 1
    fake = ctypes.c_void_p(4096)
    assert f(fake, fake, fake, fake, 10, 8, 8, 0, None, None) == 1
    assert f(fake, fake, fake, fake, 10, 0, 8, 1, None, None) == 1
    assert f(fake, fake, fake, fake, -1, 8, 8, 1, None, None) == 1
    # K or N not a multiple of 8, too many experts, misaligned offsets -> unsupported
    assert f(fake, fake, fake, fake, 10, 12, 8, 1, None, None) == 2
    assert f(fake, fake, fake, fake, 10, 8, 20, 1, None, None) == 2
    assert f(fake, fake, fake, fake, 10, 8, 8, 1025, None, None) == 2
    assert f(fake, fake, ctypes.c_void_p(4098), fake, 10, 8, 8, 1, None, None) == 2
    assert lib.gg_masked_forward(fake, fake, fake, fake, -1, 8, 8, 1, None, None) == 1


def test_watchdog_and_test_hook_setters(lib):
    import moe_grouped_gemm_ragged_b200 as gg
    prev = gg.set_watchdog_ns(123456789)
    assert gg.set_watchdog_ns(0) == 123456789
    gg.set_watchdog_ns(prev)
    assert gg.testing_skip_first_load(True) is False
    assert gg.testing_skip_first_load(False) is True


def test_python_binding_has_no_fallback():
    src = open(os.path.join(ROOT, "moe_grouped_gemm_ragged_b200", "__init__.py")).read()
    assert "import oracle" not in src and "from oracle" not in src


def test_host_step_checks_its_arguments_on_the_host(lib):
    """gg_layer_step_host reads the offsets on the host (they are host data there) and rejects
    decreasing or out-of-range offsets, bad sizes and null pointers before any CUDA call."""
    f = lib.gg_layer_step_host
    fake = ctypes.c_void_p(4096)

    def args(offs, K=8, N=8, rows=16, first=fake):
        o = ctypes.cast(offs, ctypes.c_void_p)
        return [first, fake, fake, o, fake, fake, fake] + [fake] * 7 + [rows, K, N, 3, 0, None,
                                                                        None]

    assert f(*args((ctypes.c_int32 * 3)(8, 4, 12))) == 1    # decreasing
    assert f(*args((ctypes.c_int32 * 3)(8, 12, 17))) == 1   # past the last row
    assert f(*args((ctypes.c_int32 * 3)(-1, 4, 12))) == 1   # negative
    good = (ctypes.c_int32 * 3)(4, 8, 12)
    assert f(*args(good, K=12)) == 2                         # K not a multiple of 8
    assert f(*args(good, first=None)) == 1                   # null pointer
    assert f(*(args(good)[:14] + [16, 8, 8, 3, -1, None, None])) == 1  # negative chunk count
