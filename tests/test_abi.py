"""The C-ABI library without a GPU: it builds, loads, exports every symbol the
header declares, and its host-side checks reject bad arguments before any CUDA
call is made (no compute runs here)."""
import ctypes
import os
import re
import subprocess

import pytest

import int8_row_absmax_b200 as pkg
from int8_row_absmax_b200 import build as blbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitlinear.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bl_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    blbuild.build()
    return pkg.load()


def test_header_matches_binding_table():
    assert header_functions() == sorted(pkg.SIGNATURES)


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", pkg.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (bl_\w+)$", out, flags=re.M))
    assert set(header_functions()) == exported
    for name in header_functions():
        assert getattr(lib, name) is not None


def test_pack5_ldp(lib):
    assert [lib.bl_pack5_ldp(k) for k in (1, 5, 80, 81, 128, 2560, 6912, 8192, 11008)] == \
        [16, 16, 16, 32, 32, 512, 1392, 1648, 2208]
    assert lib.bl_pack5_ldp(0) == 0


def test_status_strings(lib):
    for code, name in pkg.STATUS.items():
        assert lib.bl_status_string(code).decode() == name


def test_workspace_sizes(lib):
    assert lib.bl_quantize_weights_workspace_size(0, 5) == 0
    assert lib.bl_quantize_weights_workspace_size(4, 4) == 16384
    # below 2^20 weights, or rows that are not whole 16-byte units: the two-pass
    # kernels and their 16 KB accumulator block
    assert lib.bl_quantize_weights_workspace_size(1023, 1024) == 16384
    assert lib.bl_quantize_weights_workspace_size(8192, 8190) == 16384
    # the single-pass quantizer adds per-warp lists of 20-weight groups to
    # re-code (8 bytes each, room for 1/8 of the groups) after the block
    big = lib.bl_quantize_weights_workspace_size(8192, 8192)
    assert big % 256 == 0 and big >= 16384 + 8192 * (8192 // 20 + 1)
    assert big < 8192 * 8192                      # well under the 4 n bytes of W
    assert lib.bl_quantize_weights_workspace_size(1024, 1024) > 16384
    assert lib.bl_linear_workspace_size(16, 64, 100, 1) >= 16 * 112 + 16 * 4


NULL = None


@pytest.mark.parametrize("case,expect", [
    # null weights / bad sizes / eps
    (lambda L: L.bl_linear(1, 1, 8, NULL, 0, 4, 8, 1, NULL, 1e-5, 1, 1, 1 << 20, NULL), 1),
    (lambda L: L.bl_linear(1, 1, 0, 16, 0, 4, 8, 1, NULL, 1e-5, 1, 1, 1 << 20, NULL), 1),
    (lambda L: L.bl_linear(1, 1, 8, 16, 0, 4, 8, 1, NULL, 0.0, 1, 1, 1 << 20, NULL), 1),
    (lambda L: L.bl_linear(1, 1, 8, 16, 0, 4, 8, 1, NULL, float("nan"), 1, 1, 1 << 20, NULL), 1),
    (lambda L: L.bl_linear(1, 1, 200000, 16, 0, 4, 200000, 1, NULL, 1e-5, 1, 1, 1 << 20, NULL), 1),
    (lambda L: L.bl_linear(1, -1, 8, 16, 0, 4, 8, 1, NULL, 1e-5, 1, 1, 1 << 20, NULL), 1),
    # I8 weights with ldw < K
    (lambda L: L.bl_linear(1, 1, 8, 16, 0, 4, 7, 1, NULL, 1e-5, 1, 1, 1 << 20, NULL), 1),
    # packed weights: unaligned pointer, bad stride
    (lambda L: L.bl_linear(16, 1, 8, 17, 1, 4, 16, 16, NULL, 1e-5, 16, 256, 1 << 20, NULL), 2),
    (lambda L: L.bl_linear(16, 1, 8, 16, 1, 4, 8, 16, NULL, 1e-5, 16, 256, 1 << 20, NULL), 2),
    # unknown format / path
    (lambda L: L.bl_linear(16, 1, 8, 16, 7, 4, 16, 16, NULL, 1e-5, 16, 256, 1 << 20, NULL), 1),
    (lambda L: L.bl_linear_ex(16, 1, 8, 16, 1, 4, 16, 16, NULL, 1e-5, 16, 256, 1 << 20, 9, NULL), 1),
    # workspace missing / too small / unaligned (M = 5: not the decode GEMV, which needs none)
    (lambda L: L.bl_linear(16, 5, 8, 16, 1, 4, 16, 16, NULL, 1e-5, 16, NULL, 0, NULL), 4),
    (lambda L: L.bl_linear(16, 5, 8, 16, 1, 4, 16, 16, NULL, 1e-5, 16, 256, 8, NULL), 4),
    (lambda L: L.bl_linear(16, 5, 8, 16, 1, 4, 16, 16, NULL, 1e-5, 16, 257, 1 << 20, NULL), 4),
    # M == 0 is a no-op success, nothing launched
    (lambda L: L.bl_linear(NULL, 0, 8, 16, 1, 4, 16, 16, NULL, 1e-5, NULL, NULL, 0, NULL), 0),
    (lambda L: L.bl_quantize_act(NULL, 0, 8, 1e-5, NULL, NULL, NULL), 0),
    # weight quantization argument checks
    (lambda L: L.bl_quantize_weights(NULL, 4, 4, 1e-5, 16, 16, 256, 1 << 20, NULL), 1),
    (lambda L: L.bl_quantize_weights(16, 4, 4, -1.0, 16, 16, 256, 1 << 20, NULL), 1),
    (lambda L: L.bl_quantize_weights(16, 4, 4, 1e-5, 16, 16, 256, 4, NULL), 4),
    (lambda L: L.bl_quantize_weights(18, 4, 4, 1e-5, 16, 16, 256, 1 << 20, NULL), 2),
    (lambda L: L.bl_absmean(16, 4, 4, 1e-5, 16, 255, 16384, NULL), 4),
    (lambda L: L.bl_absmean(16, 4, 4, 1e-5, 18, 256, 16384, NULL), 2),
    (lambda L: L.bl_absmean(16, 0, 4, 1e-5, 16, 256, 16384, NULL), 1),
    (lambda L: L.bl_ternarize(16, 4, 4, NULL, 16, NULL), 1),
    (lambda L: L.bl_ternarize_pack5(16, 4, 4, 16, 16, 8, NULL), 2),
    (lambda L: L.bl_quantize_weights_pack5(16, 4, 40, 1e-5, 16, 4, 16, 256, 1 << 20, NULL), 1),
    (lambda L: L.bl_quantize_weights_pack5(16, 4, 40, 1e-5, 16, 24, 16, 256, 1 << 20, NULL), 2),
    (lambda L: L.bl_pack(16, 4, 40, 16, 4, NULL), 1),
    (lambda L: L.bl_pack(16, 4, 40, 17, 16, NULL), 2),
    (lambda L: L.bl_unpack(NULL, 4, 40, 16, 16, NULL), 1),
    (lambda L: L.bl_linear_acc(NULL, 2, 8, 16, 1, 4, 16, 16, NULL), 1),
])
def test_host_validation(lib, case, expect):
    assert case(lib) == expect


def _cdiv(a, b):
    return -(-a // b)


def _al(v):
    return _cdiv(v, 256) * 256


@pytest.mark.parametrize("M,K,N", [(5, 8192, 8192), (64, 2560, 6912), (129, 700, 19000), (512, 4096, 11008),
                                   (640, 1040, 300), (4096, 4096, 11008), (8, 128, 256), (300, 1000, 1000)])
def test_tensor_core_plan_and_workspace(lib, M, K, N):
    """The tensor-core plan, on the host: act_quant + GEMM, + the unpack of packed
    weights beyond 4 row tiles of 128, + the reduction of a K split, which is
    taken when the output tiles (128 x 256; for M <= 128 the swapped GEMM's 128
    W rows) are fewer than half of 148 SMs and K has at least two K ranges
    (640-wide chunks; 640-trit chunks of four blocks when swapped), at most 8 splits.  The workspace holds X_q [M,
    ldx] and s, then the int8 copy of W_q, then the split's int32 partials."""
    swapped = M <= 128
    if swapped:      # few rows, packed weights: the swapped GEMM (128 W rows per tile, K in chunks of 640 trits)
        tiles = _cdiv(N, 128)
        split = max(1, min(148 // tiles, _cdiv(K, 640), 8))
    else:
        tiles = _cdiv(M, 128) * _cdiv(N, 256)
        split = max(1, min(148 // tiles, _cdiv(_cdiv(K, 128), 5), 8))
    n = ctypes.c_int(0)
    assert lib.bl_linear_plan(M, N, K, pkg.PACK5, pkg.PATH_TC, ctypes.byref(n)) == pkg.PATH_TC
    assert n.value == 2 + (M > 512) + (split > 1)
    # the swapped GEMM reads X_q in decode order: rows of whole packed words (20
    # trits), padded to whole 128-byte swizzle atoms
    ldx = _cdiv(20 * _cdiv(K, 20), 128) * 128 if M <= 128 else _cdiv(K, 16) * 16
    extra = (_al(N * _cdiv(K, 16) * 16) if M > 512 else 0) + (_al(split * M * N * 4) if split > 1 else 0)
    assert lib.bl_linear_ex_workspace_size(M, N, K, pkg.PACK5, pkg.PATH_TC) == _al(M * ldx) + _al(M * 4 + 4) + extra
    # bl_linear_acc_ex: the split's partials, and for the swapped GEMM the decode-order copy of X_q
    acc_extra = extra + (_al(M * ldx) if M <= 128 else 0)
    assert lib.bl_linear_acc_workspace_size(M, N, K, pkg.PACK5, pkg.PATH_TC) == acc_extra


def test_decode_gemv_needs_no_workspace(lib):
    for M in (1, 2, 3, 4):
        assert lib.bl_linear_ex_workspace_size(M, 6912, 2560, pkg.PACK5, pkg.PATH_GEMV) == 0
    for M in (1, 2, 3):
        assert lib.bl_linear_workspace_size(M, 6912, 2560, pkg.PACK5) == 0
    assert lib.bl_linear_workspace_size(4, 6912, 2560, pkg.PACK5) > 0      # the swapped GEMM from M = 4
    assert lib.bl_linear_workspace_size(1, 6912, 2560, pkg.I8) > 0      # one trit per byte: not the GEMV


def test_auto_path_crossover(lib):
    """AUTO: the decode GEMV for M <= 3 with packed weights and the tensor cores
    (the swapped GEMM up to M = 128) from M = 4; one trit per byte: from M = 5."""
    n = ctypes.c_int(0)
    for M in (1, 2, 3):
        assert lib.bl_linear_plan(M, 4096, 4096, pkg.PACK5, pkg.PATH_AUTO, ctypes.byref(n)) == pkg.PATH_GEMV
    for M in (4, 5, 8, 100, 4096):
        assert lib.bl_linear_plan(M, 4096, 4096, pkg.PACK5, pkg.PATH_AUTO, ctypes.byref(n)) == pkg.PATH_TC
    assert lib.bl_linear_plan(4, 4096, 4096, pkg.I8, pkg.PATH_AUTO, ctypes.byref(n)) != pkg.PATH_TC
    assert lib.bl_linear_plan(5, 4096, 4096, pkg.I8, pkg.PATH_AUTO, ctypes.byref(n)) == pkg.PATH_TC


@pytest.mark.parametrize("struct,cls", [("bl_linear_call", pkg.LinearCall), ("bl_host_io", pkg.HostIO)])
def test_call_struct_layout_matches_the_header(tmp_path, struct, cls):
    """The binding's bl_linear_call and bl_host_io mirror the C structs: size and
    every field's offset, as a C compiler lays them out from the header."""
    fields = [f for f, _ in cls._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"bitlinear.h\"\nint main(void){\n"
                   f"printf(\"%zu\\n\", sizeof({struct}));\n" +
                   "".join(f"printf(\"%zu\\n\", offsetof({struct}, {f}));\n" for f in fields) +
                   "return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-I", "/usr/local/cuda/include",
                    str(src), "-o", str(exe)], check=True)
    out = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert out[0] == ctypes.sizeof(cls)
    assert out[1:] == [getattr(cls, f).offset for f in fields]


def test_linear_group_host_checks(lib):
    """Group calls are validated before any launch; decode-GEMV calls need no
    workspace, the others need bl_linear's; flags other than
    BL_FLAG_STATIC_WEIGHTS are rejected; an empty group is a no-op."""
    C = pkg.LinearCall
    gemv = C(16, 1, 2560, 16, 6912, 512, pkg.PACK5, 1e-5, 16, None, 16)
    tc = C(16, 64, 2560, 16, 6912, 512, pkg.PACK5, 1e-5, 16, None, 16)
    arr = (C * 2)(gemv, tc)
    assert lib.bl_linear_group_workspace_size(arr, 1) == 0
    assert lib.bl_linear_group_workspace_size(arr, 2) == _al(lib.bl_linear_workspace_size(64, 6912, 2560, pkg.PACK5))
    assert lib.bl_linear_group(arr, 0, 0, None, 0, None) == 0
    assert lib.bl_linear_group(arr, 1, 0x1, None, 0, None) == 1            # unknown flag
    assert lib.bl_linear_group(arr, 2, 0, None, 0, None) == 4              # workspace missing
    bad = (C * 2)(gemv, C(16, 1, 2560, 17, 6912, 512, pkg.PACK5, 1e-5, 16, None, 16))
    assert lib.bl_linear_group(bad, 2, 0, None, 0, None) == 2              # unaligned packed W
    neg = (C * 1)(C(16, 1, 2560, 16, 6912, 512, pkg.PACK5, 0.0, 16, None, 16))
    assert lib.bl_linear_group(neg, 1, 0, None, 0, None) == 1              # eps <= 0


def test_linear_group_host_buffers_checks(lib):
    """The host-buffer group validates every call and its host pointers before
    it enqueues anything: an empty group is a no-op, a NULL io array or host
    pointer and unknown flags are invalid arguments, a missing workspace and a
    misaligned weight pointer are reported as for bl_linear_group."""
    C, H = pkg.LinearCall, pkg.HostIO
    gemv = C(16, 1, 2560, 16, 6912, 512, pkg.PACK5, 1e-5, 16, None, 16)
    tc = C(16, 64, 2560, 16, 6912, 512, pkg.PACK5, 1e-5, 16, None, 16)
    empty = C(16, 0, 2560, 16, 6912, 512, pkg.PACK5, 1e-5, 16, None, 16)
    arr = (C * 2)(gemv, tc)
    io = (H * 2)(H(64, 64), H(64, 64))
    f = lib.bl_linear_group_host
    assert f(arr, io, 0, 0, None, 0, None) == 0
    assert f(arr, None, 0, 0, None, 0, None) == 0
    assert f(arr, None, 1, 0, None, 0, None) == 1                          # io missing
    assert f(arr, (H * 1)(H(None, 64)), 1, 0, None, 0, None) == 1          # X_host missing
    assert f(arr, (H * 1)(H(64, None)), 1, 0, None, 0, None) == 1          # Y_host missing
    assert f((C * 1)(empty), (H * 1)(H(None, None)), 1, 0, None, 0, None) == 0   # M = 0: nothing to copy
    assert f(arr, io, 1, 0x1, None, 0, None) == 1                          # unknown flag
    assert f(arr, io, 2, 0, None, 0, None) == 4                            # workspace missing
    bad = (C * 2)(gemv, C(16, 1, 2560, 17, 6912, 512, pkg.PACK5, 1e-5, 16, None, 16))
    assert f(bad, io, 2, 0, None, 0, None) == 2                            # unaligned packed W


def test_static_weights_flag_is_a_flag(lib):
    """BL_FLAG_STATIC_WEIGHTS rides on `path` without changing the plan or the
    workspace; other high bits are rejected."""
    n = ctypes.c_int(0)
    F = pkg.FLAG_STATIC_WEIGHTS
    for M in (1, 4, 64):
        for path in (pkg.PATH_AUTO, pkg.PATH_GEMV, pkg.PATH_TC):
            assert lib.bl_linear_plan(M, 6912, 2560, pkg.PACK5, path | F, ctypes.byref(n)) == \
                lib.bl_linear_plan(M, 6912, 2560, pkg.PACK5, path, ctypes.byref(n))
            assert lib.bl_linear_ex_workspace_size(M, 6912, 2560, pkg.PACK5, path | F) == \
                lib.bl_linear_ex_workspace_size(M, 6912, 2560, pkg.PACK5, path)
    assert lib.bl_linear_ex(16, 1, 8, 16, 1, 4, 16, 16, NULL, 1e-5, 16, 256, 1 << 20, 0x200, NULL) == 1


def test_deployed_checkpoint_host_side(lib, tmp_path):
    """The checkpoint reader's host side against files the oracle writes: layer
    count, shapes, names and bias flags; malformed files give BL_ERR_IO; a
    save of no layers writes the oracle's header bytes."""
    import numpy as np
    from oracle import checkpoint
    rng = np.random.default_rng(3)
    layers = [{"name": "attn.q", "Wq": rng.integers(-1, 2, (7, 33)).astype(np.int8), "beta": np.float32(0.02)},
              {"name": "", "Wq": rng.integers(-1, 2, (2, 5)).astype(np.int8), "beta": np.float32(1),
               "bias": np.ones(2, np.float32)}]
    data = checkpoint.write_deployed(layers)
    path = tmp_path / "m.blt"
    path.write_bytes(data)
    n = ctypes.c_int(-1)
    assert lib.bl_deployed_count(str(path).encode(), ctypes.byref(n)) == 0 and n.value == 2
    N, K, hb = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int()
    name = ctypes.create_string_buffer(256)
    for i, (eN, eK, eb, en) in enumerate(((7, 33, 0, b"attn.q"), (2, 5, 1, b""))):
        assert lib.bl_deployed_layer_info(str(path).encode(), i, ctypes.byref(N), ctypes.byref(K),
                                          ctypes.byref(hb), name, 256) == 0
        assert (N.value, K.value, hb.value, name.value) == (eN, eK, eb, en)
    short = ctypes.create_string_buffer(4)
    assert lib.bl_deployed_layer_info(str(path).encode(), 0, None, None, None, short, 4) == 0
    assert short.value == b"att"
    assert lib.bl_deployed_layer_info(str(path).encode(), 2, None, None, None, None, 0) == 1
    for bad in (data[:-1], data + b"\0", b"XLT5" + data[4:], data[:4] + b"\2\0\0\0" + data[8:], b""):
        path.write_bytes(bad)
        assert lib.bl_deployed_count(str(path).encode(), ctypes.byref(n)) == 8
    assert lib.bl_deployed_count(str(tmp_path / "missing.blt").encode(), ctypes.byref(n)) == 8
    empty = tmp_path / "empty.blt"
    assert lib.bl_save_deployed(str(empty).encode(), None, 0, None) == 0
    assert empty.read_bytes() == checkpoint.write_deployed([])
    assert lib.bl_save_deployed(str(tmp_path / "no_dir" / "x.blt").encode(), None, 0, None) == 8


def test_backward_host_checks(lib):
    assert lib.bl_linear_backward_workspace_size(0, 4, 4) == 0
    # dX [M,K] splits: dY [M, ldN] and W^T [K, ldN] (hi and lo); dW: dY^T [N, ldM] and X^T [K, ldM]
    M, N, K = 5, 6, 7
    ldN, ldM = 8, 8
    expect = max(2 * (_al(M * ldN * 4) + _al(K * ldN * 4)), 2 * (_al(N * ldM * 4) + _al(K * ldM * 4)))
    assert lib.bl_linear_backward_workspace_size(M, N, K) == expect
    assert lib.bl_linear_backward(NULL, 16, 16, 2, 3, 4, 16, 16, 16, 256, 1 << 20, NULL) == 1   # no dY
    assert lib.bl_linear_backward(16, NULL, 16, 2, 3, 4, 16, 16, 16, 256, 1 << 20, NULL) == 1   # dW without X
    assert lib.bl_linear_backward(16, 16, NULL, 2, 3, 4, 16, 16, 16, 256, 1 << 20, NULL) == 1   # dX without W
    assert lib.bl_linear_backward(18, 16, 16, 2, 3, 4, 16, 16, 16, 256, 1 << 20, NULL) == 2
    assert lib.bl_linear_backward(16, 16, 16, 2, 3, 4, 16, 16, 16, NULL, 0, NULL) == 4
    assert lib.bl_linear_backward(16, 16, 16, 2, 3, 4, 16, 16, 16, 256, 8, NULL) == 4
    assert lib.bl_linear_backward(NULL, NULL, NULL, 0, 3, 4, NULL, NULL, NULL, NULL, 0, NULL) == 0
    assert lib.bl_linear_backward(16, 16, 16, 2, 0, 4, 16, 16, 16, 256, 1 << 20, NULL) == 1


def test_rmsnorm_quant_host_checks(lib):
    assert lib.bl_rmsnorm_quantize_act(NULL, 0, 8, 16, 1e-5, 1e-5, NULL, NULL, NULL) == 0
    assert lib.bl_rmsnorm_quantize_act(16, 2, 8, NULL, 1e-5, 1e-5, 16, 16, NULL) == 1
    assert lib.bl_rmsnorm_quantize_act(16, 2, 8, 16, 0.0, 1e-5, 16, 16, NULL) == 1
    assert lib.bl_rmsnorm_quantize_act(16, 2, 8, 16, 1e-5, float("inf"), 16, 16, NULL) == 1
    assert lib.bl_rmsnorm_quantize_act(16, 2, 49153, 16, 1e-5, 1e-5, 16, 16, NULL) == 1
    assert lib.bl_rmsnorm_quantize_act(18, 2, 8, 16, 1e-5, 1e-5, 16, 16, NULL) == 2


def test_selftest_timeout_host_checks(lib):
    """The timeout self-test's limit is checked on the host before any launch."""
    for limit in (0, 999, 10 ** 9 + 1):
        assert lib.bl_selftest_wait_timeout(limit, None) == 1     # BL_ERR_INVALID_ARG
