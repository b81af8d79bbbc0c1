"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol the
header declares, and validates arguments before touching a device."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxfp4_moe.h")


@pytest.fixture(scope="module")
def L():
    from mxfp4_quantized_moe_b200 import build
    build.build()
    from mxfp4_quantized_moe_b200 import _lib
    return _lib


def declared_symbols():
    src = open(HEADER).read()
    return re.findall(r"MXFP4_MOE_API\s+[\w\s\*]+?\b(mxfp4_moe_\w+)\s*\(", src)


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for must in ("mxfp4_moe_forward", "mxfp4_moe_backward_input", "mxfp4_moe_workspace_size",
                 "mxfp4_moe_transpose_weights", "mxfp4_moe_dequantize", "mxfp4_moe_check",
                 "mxfp4_moe_strerror"):
        assert must in syms


def test_library_exports_every_declared_symbol(L):
    lib = ctypes.CDLL(L.LIB_PATH)
    syms = declared_symbols()
    assert syms
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(L.SIGNATURES)


def test_debug_build_exports_the_same_symbols_and_reports_itself(L):
    """The debug build (device-side index checks) is the same boundary: every declared symbol,
    and mxfp4_moe_build_flags tells the two builds apart (a host-only call)."""
    from mxfp4_quantized_moe_b200 import build
    dbg_path = build.build(debug=True)
    rel = ctypes.CDLL(build.LIB)
    dbg = ctypes.CDLL(dbg_path)
    for s in declared_symbols():
        assert hasattr(dbg, s), s
    assert rel.mxfp4_moe_build_flags() == 0
    assert dbg.mxfp4_moe_build_flags() == 1
    assert L.lib.mxfp4_moe_build_flags() in (0, 1)


def test_unknown_gate_up_format_is_rejected(L):
    n = ctypes.c_size_t()
    for fmt, want in ((0, L.OK), (1, L.OK), (2, L.ERR_INVALID_ARG), (-1, L.ERR_INVALID_ARG)):
        d = L.Dims(64, 256, 256, 8, 2, 1.702, 7.0, fmt)
        assert L.lib.mxfp4_moe_workspace_size(ctypes.byref(d), ctypes.byref(n)) == want, fmt


def test_dims_struct_matches_header():
    """The ctypes mirror lists the header struct's fields in order."""
    from mxfp4_quantized_moe_b200 import _lib
    src = open(HEADER).read()
    body = re.search(r"typedef struct \{([^}]*)\} mxfp4_moe_dims;", src).group(1)
    names = re.findall(r"(\w+)\s*[,;]", body)
    assert names == [f[0] for f in _lib.Dims._fields_]


def test_error_codes_match_header(L):
    src = open(HEADER).read()
    codes = dict(re.findall(r"#define (MXFP4_MOE_\w+) \(?(-?\d+)\)?", src))
    assert int(codes["MXFP4_MOE_OK"]) == L.OK
    assert int(codes["MXFP4_MOE_ERR_INVALID_ARG"]) == L.ERR_INVALID_ARG
    assert int(codes["MXFP4_MOE_ERR_WORKSPACE_TOO_SMALL"]) == L.ERR_WORKSPACE_TOO_SMALL
    assert int(codes["MXFP4_MOE_ERR_UNSUPPORTED_DEVICE"]) == L.ERR_UNSUPPORTED_DEVICE
    assert int(codes["MXFP4_MOE_ERR_CUDA"]) == L.ERR_CUDA
    assert int(codes["MXFP4_MOE_ERR_DEVICE_TIMEOUT"]) == L.ERR_DEVICE_TIMEOUT
    assert int(codes["MXFP4_MOE_ERR_DEVICE_BOUNDS"]) == L.ERR_DEVICE_BOUNDS
    for c in (0, -1, -2, -3, -4, -5, -6, -99):
        assert L.strerror(c)


def _ws(L, *dims):
    n = ctypes.c_size_t()
    rc = L.lib.mxfp4_moe_workspace_size(ctypes.byref(L.Dims(*dims)), ctypes.byref(n))
    return rc, n.value


def test_workspace_size_formula(L):
    T, H, I, E, k = 8192, 2880, 2880, 32, 4
    rc, n = _ws(L, T, H, I, E, k, 1.702, 7.0)
    assert rc == 0
    A = T * k
    # saved GLU factors (bf16x2) + saved act + dH + rows (Xp / y / dYp / dX)
    big = A * (4 * I + 2 * I + 4 * I + 2 * H)
    # plus routing: idx, w, perm, inv, w_row (4 B each per assignment), the activation scales
    # of the block-scaled gate_up (one byte per 32 of H, rows padded to 96 bytes) and small
    # tables
    small = 20 * A + 96 * A
    assert big + small <= n < big + small + 1024 * 1024


@pytest.mark.parametrize("dims", [
    (0, 256, 256, 8, 2), (64, 250, 256, 8, 2), (64, 256, 100, 8, 2), (64, 256, 256, 0, 1),
    (64, 256, 256, 8, 9), (64, 256, 256, 257, 2), (64, 256, 256, 8, 0),
    (64, 256, 65536, 8, 2),  # tile scales would not fit shared memory
])
def test_bad_shapes_rejected(L, dims):
    rc, _ = _ws(L, *dims, 1.702, 7.0)
    assert rc == L.ERR_INVALID_ARG


def test_null_pointers_rejected_before_device(L):
    d = L.Dims(64, 256, 256, 8, 2, 1.702, 7.0)
    w = L.Weights()
    rc = L.lib.mxfp4_moe_forward(ctypes.byref(d), ctypes.byref(w), None, None, None, None, None,
                                 None, 0, None)
    assert rc == L.ERR_INVALID_ARG
    rc = L.lib.mxfp4_moe_backward_input(ctypes.byref(d), ctypes.byref(w), None, 0, None, None, 0,
                                        None, None, None, None)
    assert rc == L.ERR_INVALID_ARG
    rc = L.lib.mxfp4_moe_dequantize(None, None, 4, 64, None, None)
    assert rc == L.ERR_INVALID_ARG
    rc = L.lib.mxfp4_moe_grouped_matmul(2, 64, 64, 8, None, None, None, None, 0, None, None, None)
    assert rc == L.ERR_INVALID_ARG
    rc = L.lib.mxfp4_moe_dequantize(ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 48,
                                    ctypes.c_void_p(16), None)
    assert rc == L.ERR_INVALID_ARG  # K not a multiple of 32


def test_small_workspace_rejected_before_device(L):
    d = L.Dims(64, 256, 256, 8, 2, 1.702, 7.0)
    p = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    w = L.Weights(p, p, p, p, p, p)
    rc, need = _ws(L, 64, 256, 256, 8, 2, 1.702, 7.0)
    rc = L.lib.mxfp4_moe_forward(ctypes.byref(d), ctypes.byref(w), p, p, p, None, None, p,
                                 need - 1, None)
    assert rc == L.ERR_WORKSPACE_TOO_SMALL


def test_python_wrappers_have_no_cpu_path():
    """The torch-facing wrappers must refuse CPU tensors rather than compute on the host."""
    import torch
    from mxfp4_quantized_moe_b200 import moe
    with pytest.raises(ValueError):
        moe.dequantize(torch.zeros(4, 16, dtype=torch.uint8), torch.zeros(4, 1, dtype=torch.uint8))


def test_zipf_workload_realises_the_skew():
    """The skewed-routing recipe gives what the workload promises: the hottest expert near 25%
    of assignments and several experts under 16 rows (top-k on the generated logits)."""
    import torch
    from mxfp4_quantized_moe_b200 import inputs
    wl = inputs.WORKLOADS["gpt-oss-20b-moe-zipf-T16384"]
    lg = inputs.make_workload(wl, 0, with_dy=False)["logits"]
    h = torch.bincount(torch.topk(lg, wl.k, dim=1).indices.flatten(), minlength=wl.E)
    assert 0.22 <= float(h.max()) / float(h.sum()) <= 0.28
    assert int((h < 16).sum()) >= 5 and int(h.min()) >= 1


def test_selftest_arguments_checked_before_device(L):
    assert L.lib.mxfp4_moe_selftest_wait_timeout(None, 64, None) == L.ERR_INVALID_ARG
    p = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    assert L.lib.mxfp4_moe_selftest_wait_timeout(p, 8, None) == L.ERR_INVALID_ARG


def test_interleave_helper_arguments_checked_before_device(L):
    d = L.Dims(16, 256, 256, 4, 2, 1.702, 7.0)
    p = ctypes.c_void_p(1 << 20)  # never dereferenced
    assert L.lib.mxfp4_moe_interleave_gate_up(ctypes.byref(d), None, p, p, p, p, p, None) == L.ERR_INVALID_ARG
    bad = L.Dims(16, 250, 256, 4, 2, 1.702, 7.0)
    assert L.lib.mxfp4_moe_interleave_gate_up(ctypes.byref(bad), p, p, p, p, p, p, None) == L.ERR_INVALID_ARG


def test_no_usable_device_is_an_error_not_a_crash(L):
    """Valid arguments on a host without a B200: the call reports an error before enqueuing."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible: the fake pointers below would reach a launch")
    d = L.Dims(64, 256, 256, 8, 2, 1.702, 7.0)
    p = ctypes.c_void_p(1 << 20)
    w = L.Weights(p, p, p, p, p, p)
    rc, need = _ws(L, 64, 256, 256, 8, 2, 1.702, 7.0)
    rc = L.lib.mxfp4_moe_forward(ctypes.byref(d), ctypes.byref(w), p, p, p, None, None, p, need,
                                 None)
    assert rc in (L.ERR_CUDA, L.ERR_UNSUPPORTED_DEVICE)


def test_binding_without_the_library_fails_loudly(tmp_path):
    """No silent fallback: importing the binding without the built library raises ImportError."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "mxfp4_quantized_moe_b200")
    dst = tmp_path / "mxfp4_quantized_moe_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "csrc", "__pycache__"))
    code = ("import sys; sys.path.insert(0, %r)\n"
            "try:\n    import mxfp4_quantized_moe_b200.moe\nexcept ImportError as e:\n"
            "    print('IMPORT_ERROR', e); sys.exit(3)\nprint('LOADED')") % str(tmp_path)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300,
                       cwd=str(tmp_path))
    assert r.returncode == 3 and "IMPORT_ERROR" in r.stdout, r.stdout + r.stderr


def test_residual_entry_points_validate_before_the_device(L):
    """Bad shapes, missing operands, misalignment and an output overlapping an input are
    INVALID_ARG without any device call; a valid call reaches the device check (no GPU here)."""
    a = ctypes.c_void_p(1 << 20)          # 16-byte aligned addresses, never dereferenced
    b = ctypes.c_void_p((1 << 20) + (1 << 16))
    c = ctypes.c_void_p((1 << 20) + (2 << 16))
    odd = ctypes.c_void_p((1 << 20) + 8)
    rr = L.lib.mxfp4_moe_residual_router
    bad = [
        (4, 48, 8, a, b, a, None, c, None),     # H not a multiple of 32
        (4, 64, 0, a, b, a, None, c, None),     # E = 0
        (4, 64, 300, a, b, a, None, c, None),   # E > 256
        (4, 64, 8, None, b, a, None, c, None),  # no x
        (4, 64, 8, a, None, None, None, None, None),  # neither a residual nor logits
        (4, 64, 8, a, b, a, None, None, None),  # y without x_out
        (4, 64, 8, a, None, a, None, c, a),     # x_out without y
        (4, 64, 8, a, b, None, None, c, a),     # logits without w_r
        (4, 64, 8, odd, b, a, None, c, None),   # misaligned x
        (4, 64, 8, a, b, a, None, a, None),     # x_out overlaps x
    ]
    for args in bad:
        assert rr(*args, None) == L.ERR_INVALID_ARG, args
    assert rr(4, 64, 8, a, b, a, None, c, a, None) in (L.ERR_UNSUPPORTED_DEVICE, L.ERR_CUDA)
    gc = L.lib.mxfp4_moe_grad_chain
    for args in [(4, 48, 8, a, b, c, a, a), (4, 64, 0, a, b, c, a, a), (4, 64, 8, None, b, c, a, a),
                 (4, 64, 8, a, b, None, a, a), (4, 64, 8, a, b, c, odd, a)]:
        assert gc(*args, None) == L.ERR_INVALID_ARG, args
    assert gc(4, 64, 8, a, b, c, a, a, None) in (L.ERR_UNSUPPORTED_DEVICE, L.ERR_CUDA)
