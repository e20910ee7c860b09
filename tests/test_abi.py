"""The C-ABI library: it loads, exports every function include/q4.h declares,
and rejects bad arguments on the host before touching CUDA.

These run without a GPU: every call below returns from argument validation,
which happens before any CUDA runtime call (q4.h, "Errors")."""
import ctypes
import subprocess

import pytest

import weight_only_bit_gemv_b200 as q4

OK, NULL, SHAPE, ALIGN = 0, 1, 2, 3
A = 1 << 20          # a 16-byte-aligned fake address; never dereferenced
MIS = A + 8          # misaligned


@pytest.fixture(scope="module")
def lib():
    return q4.load()


def test_exports_every_declared_function(lib):
    names = q4.header_functions()
    assert {"q4_pack", "q4_dequant", "q4_gemv", "q4_gemm", "q4_status_string",
            "q4_last_cuda_error", "q4_abi_version", "q4_timeout_flags",
            "q4_gemm_noalloc"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", q4.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)


def test_abi_version_and_strings(lib):
    assert q4.abi_version() == 1
    for code in range(7):
        s = q4.status_string(code)
        assert s.startswith(q4.STATUS[code])
    assert "unknown" in q4.status_string(99)
    assert lib.q4_last_cuda_error() == 0


def test_gemv_rejects_shapes(lib):
    f = lib.q4_gemv
    assert f(A, A, A, A, A, 2, 64, 256, None) == SHAPE        # M != 1
    assert f(A, A, A, A, A, 1, 64, 100, None) == SHAPE        # K % 64
    assert f(A, A, A, A, A, 1, 64, 0, None) == SHAPE          # K == 0
    assert f(A, A, A, A, A, 1, -1, 64, None) == SHAPE         # N < 0
    assert f(A, A, A, A, A, 1, 64, (1 << 20) + 64, None) == SHAPE   # K > Q4_MAX_K
    assert f(A, A, A, A, A, 1, 0, 64, None) == OK             # empty: no launch
    assert f(None, None, None, None, None, 1, 0, 64, None) == OK


def test_gemm_rejects(lib):
    f = lib.q4_gemm
    assert f(A, A, A, A, A, -1, 64, 64, None) == SHAPE
    assert f(A, A, A, A, A, 0, 64, 64, None) == OK
    assert f(A, A, A, A, A, 5, 0, 64, None) == OK
    assert f(None, A, A, A, A, 5, 64, 64, None) == NULL
    assert f(A, A, A, A, None, 5, 64, 64, None) == NULL
    assert f(A, MIS, A, A, A, 5, 64, 64, None) == ALIGN
    assert f(A, A, A, MIS, A, 5, 64, 64, None) == ALIGN
    assert f(A, A, A, A, MIS, 5, 64, 64, None) == ALIGN
    assert f(A, A, MIS, A, A, 5, 64, 64, None) == ALIGN


def test_gemm_noalloc_rejects(lib):
    f = lib.q4_gemm_noalloc
    K = 4096
    too_many = (8 << 20) // (2 * K) + 1          # one token past the fixed scratch
    assert f(A, A, A, A, A, too_many, 64, K, None) == 6   # Q4_ERR_TOO_LARGE
    assert f(A, A, A, A, A, -1, 64, K, None) == SHAPE
    assert f(None, A, A, A, A, too_many, 64, K, None) == NULL
    assert f(A, A, A, MIS, A, too_many, 64, K, None) == ALIGN
    assert f(A, A, A, A, A, 0, 64, K, None) == OK


def test_timeout_flags_rejects_null(lib):
    assert lib.q4_timeout_flags(None) == NULL


def test_pack_dequant_reject(lib):
    assert lib.q4_pack(A, A, A, A, 4, 96, None) == SHAPE
    assert lib.q4_pack(A, A, A, A, -4, 64, None) == SHAPE
    assert lib.q4_pack(A, A, A, A, 0, 64, None) == OK
    assert lib.q4_pack(A, None, A, A, 4, 64, None) == NULL
    assert lib.q4_pack(A, A, MIS, A, 4, 64, None) == ALIGN
    assert lib.q4_dequant(A, A, A, A, 4, 32, None) == SHAPE
    assert lib.q4_dequant(A, A, A, None, 4, 64, None) == NULL
    assert lib.q4_dequant(MIS, A, A, A, 4, 64, None) == ALIGN
    assert lib.q4_dequant(A, A, A, A, 0, 64, None) == OK


def test_embed_rows_rejects(lib):
    f = lib.q4_embed_rows
    assert f(A, A, A, A, A, 4, 64, 100, None) == SHAPE        # K % 64
    assert f(A, A, A, A, A, -1, 64, 64, None) == SHAPE        # n_ids < 0
    assert f(A, A, A, A, A, 4, -1, 64, None) == SHAPE         # N < 0
    assert f(None, None, None, None, None, 0, 64, 64, None) == OK   # no ids: no launch
    assert f(A, A, A, None, A, 4, 64, 64, None) == NULL       # ids
    assert f(A, A, A, A, None, 4, 64, 64, None) == NULL       # out
    assert f(A, A, A, MIS, A, 4, 64, 64, None) == ALIGN
    assert f(A, A, A, A, MIS, 4, 64, 64, None) == ALIGN


def test_two_bit_rejects(lib):
    for f in (lib.q4_pack2, lib.q4_dequant2):
        assert f(A, A, A, A, 4, 100, None) == SHAPE            # K % 64
        assert f(A, A, A, A, -1, 64, None) == SHAPE            # N < 0
        assert f(None, None, None, None, 0, 64, None) == OK    # N == 0: no launch
        assert f(None, A, A, A, 4, 64, None) == NULL
        assert f(MIS, A, A, A, 4, 64, None) == ALIGN
    g = lib.q4_gemv2
    assert g(A, A, A, A, A, 4, 100, None) == SHAPE              # K % 64
    assert g(A, A, A, A, A, 4, 98304 + 64, None) == SHAPE       # above Q4_GEMV2_MAX_K
    assert g(A, A, A, A, A, -1, 64, None) == SHAPE
    assert g(None, None, None, None, None, 0, 64, None) == OK   # N == 0: no launch
    assert g(A, A, A, None, A, 4, 64, None) == NULL
    assert g(A, A, A, A, MIS, 4, 64, None) == ALIGN


def test_ring_rejects(lib):
    import ctypes
    h = ctypes.c_void_p()
    assert lib.q4_ring_create(1 << 20, None) == NULL
    assert lib.q4_ring_create(0, ctypes.byref(h)) == SHAPE
    assert lib.q4_ring_gemm(None, A, A, A, A, A, 1, 64, 64, None) == NULL
    assert lib.q4_ring_destroy(None) == NULL


def test_binding_marshalling_checks():
    import torch
    cpu = torch.zeros(4, 32, dtype=torch.uint8)
    with pytest.raises(ValueError):
        q4.q4_gemv(cpu, torch.zeros(4, 1, dtype=torch.float16), torch.zeros(16, dtype=torch.float16),
                   torch.zeros(1, 64, dtype=torch.bfloat16))
    with pytest.raises(TypeError):
        q4.q4_pack(torch.zeros(4, 64, dtype=torch.float64), torch.zeros(16, dtype=torch.float16))


def test_two_bit_binding_marshalling_checks():
    import torch
    codes = torch.zeros(4, 16, dtype=torch.uint8)              # N = 4, K = 64
    scales = torch.zeros(4, 1, dtype=torch.float16)
    cb4 = torch.zeros(4, dtype=torch.float16)
    with pytest.raises(ValueError):                            # x of the wrong K
        q4.q4_gemv2(codes, scales, cb4, torch.zeros(1, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError):                            # M != 1
        q4.q4_gemv2(codes, scales, cb4, torch.zeros(2, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):                            # host tensors
        q4.q4_gemv2(codes, scales, cb4, torch.zeros(1, 64, dtype=torch.bfloat16))
    with pytest.raises(TypeError):
        q4.q4_pack2(torch.zeros(4, 64, dtype=torch.float64), cb4)
    with pytest.raises(ValueError):                            # codes not 2-D
        q4.q4_dequant2(torch.zeros(64, dtype=torch.uint8), scales, cb4)


def test_binding_has_every_header_name():
    """The binding exposes each entry point of include/q4.h under its C name."""
    missing = [n for n in q4.header_functions() if not callable(getattr(q4, n, None))]
    assert not missing, missing
    assert q4.q4_abi_version() == q4.abi_version()
    assert q4.q4_status_string(0) == q4.status_string(0)
    assert isinstance(q4.q4_last_cuda_error(), int)


def test_step_rejects(lib):
    """q4_step_create validates its list (and every linear as q4_gemm does)
    before it records anything."""
    h = ctypes.c_void_p()
    L = q4.Q4Linear
    good = L(A, A, A, A, A, 1, 64, 256)
    assert lib.q4_step_create((L * 1)(good), 1, None) == NULL
    assert lib.q4_step_create(None, 1, ctypes.byref(h)) == NULL
    assert lib.q4_step_create((L * 1)(good), 0, ctypes.byref(h)) == SHAPE
    assert lib.q4_step_create((L * 2)(good, L(A, A, A, A, A, 1, 64, 100)), 2,
                              ctypes.byref(h)) == SHAPE             # second linear: K % 64
    assert lib.q4_step_create((L * 2)(good, L(A, A, None, A, A, 4, 64, 64)), 2,
                              ctypes.byref(h)) == NULL
    assert lib.q4_step_create((L * 1)(L(A, A, A, MIS, A, 2, 64, 64)), 1, ctypes.byref(h)) == ALIGN
    assert h.value is None
    assert lib.q4_step_launch(None, None) == NULL
    assert lib.q4_step_destroy(None) == NULL


def test_wait_selftest_rejects(lib):
    out = ctypes.c_uint32(7)
    assert lib.q4_wait_selftest(1000, 0, None) == NULL
    assert lib.q4_wait_selftest(0, 0, ctypes.byref(out)) == SHAPE
    assert lib.q4_wait_selftest(1000001, 1, ctypes.byref(out)) == SHAPE


def test_bounds_flags_rejects_null(lib):
    assert lib.q4_bounds_flags(None) == NULL


def test_release_build_is_not_bounds_checked(lib):
    if q4.debug_selected():
        pytest.skip("Q4_LIBRARY=debug selects the bounds-checked build")
    assert lib.q4_bounds_checked() == 0
    assert q4.library_path().endswith("libq4.so")


def test_library_selection_rejects_unknown_names(monkeypatch):
    monkeypatch.setenv("Q4_LIBRARY", "fast")
    with pytest.raises(RuntimeError):
        q4.library_path()
    monkeypatch.setenv("Q4_LIBRARY", "debug")
    assert q4.library_path().endswith("libq4_debug.so")


def test_debug_build_exports_the_same_and_says_so():
    """libq4_debug.so (the -DQ4_DEBUG build) exports every declared function
    and reports itself as bounds-checked; it is loaded in a child process,
    since one process loads one of the two libraries."""
    from weight_only_bit_gemv_b200 import build as b
    b.build(debug=True)          # no-op when up to date
    out = subprocess.run(["nm", "-D", "--defined-only", b.DEBUG_LIBRARY],
                         capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in q4.header_functions() if n not in exported]
    assert not missing, missing
    code = ("import ctypes, weight_only_bit_gemv_b200 as q4; l = q4.load(False); "
            "print(q4.library_path(), l.q4_bounds_checked(), l.q4_bounds_flags(None))")
    import os
    import sys
    env = dict(os.environ, Q4_LIBRARY="debug")
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                         cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))), check=True)
    path, checked, null_status = res.stdout.split()
    assert path.endswith("libq4_debug.so") and checked == "1" and int(null_status) == NULL
