"""Host-side checks of the C ABI: the library builds, loads and exports every
function the header declares, and argument validation rejects bad calls
before anything touches a GPU.  No test here needs a GPU."""
import ctypes

import pytest

from structured_sparse_fp8_b200 import _lib
from structured_sparse_fp8_b200 import build as B


@pytest.fixture(scope="module")
def lib():
    B.build()
    return _lib.load()


def test_every_declared_function_is_exported(lib):
    names = _lib.header_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks a signature for {name}"


def test_status_strings_and_version(lib):
    assert lib.sp24_status_str(0) == b"ok"
    for code in range(-7, 0):
        assert lib.sp24_status_str(code) not in (b"ok", b"unknown status")
    assert b"sm_100a" in lib.sp24_version()


def test_workspace_sizes(lib):
    for op in range(4):
        assert lib.sp24_workspace_size(op, 16, 256, 256, 0) == 256
    # Shapes whose tiles fill whole waves of the 148 SMs need no scratch:
    # M=256 -> 128-token tiles, 2 x (18944 / 128) = 296 tiles = 2 waves.
    assert lib.sp24_workspace_size(_lib.OP_GEMM, 256, 18944, 4096, 0) == 0
    assert lib.sp24_workspace_size(_lib.OP_GEMM_DENSE, 256, 18944, 4096, 0) == 0
    # Otherwise the leftover tiles are split by k-blocks over up to every CTA
    # (at most two ways for tiles wider than 64 tokens): a 16 KB counter
    # prefix + one fp32 (rows x BN) partial tile per splitting CTA.  Prefill
    # M=4096 uses 224-token tiles of 256 W rows (N % 256 == 0): 19 x 48 = 912
    # tiles = 6 waves + 24 leftover, split over 48 CTAs.
    assert lib.sp24_workspace_size(_lib.OP_GEMM, 4096, 12288, 4096, 0) == 16384 + 48 * 256 * 224 * 4
    # N not a multiple of 256: 128-row tiles, 19 x 75 = 1425 tiles = 9 waves +
    # 93 leftover over 148 CTAs
    assert lib.sp24_workspace_size(_lib.OP_GEMM, 4096, 9600, 4096, 0) == 16384 + 148 * 128 * 224 * 4
    # down-proj M=256: 64 tiles of 112 k-blocks, each split over 2 CTAs
    assert lib.sp24_workspace_size(_lib.OP_GEMM, 256, 4096, 14336, 0) == 16384 + 128 * 128 * 128 * 4
    # decode: 16-token tiles
    assert lib.sp24_workspace_size(_lib.OP_GEMM, 1, 11008, 4096, 0) == 16384 + 148 * 128 * 16 * 4
    for m in (1, 64):
        ws = lib.sp24_workspace_size(_lib.OP_GEMM, m, 11008, 4096, 0)
        assert ws > 16384 and ws % 16 == 0
    # tiny: 2 tiles x 2 k-blocks -> 2 CTAs with one whole tile each
    assert lib.sp24_workspace_size(_lib.OP_GEMM, 16, 256, 256, 0) == 0
    assert lib.sp24_workspace_size(_lib.OP_GEMM, 0, 11008, 4096, 0) == 0
    # fused quantise (or lift) + GEMM: 256 bytes of counters, then the GEMM's
    # workspace at K (or K' = 3K/2)
    for m in (1, 8, 32, 64, 256):
        assert (lib.sp24_workspace_size(_lib.OP_QUANTIZE_GEMM_PACKED, m, 11008, 4096, 0)
                == 256 + lib.sp24_workspace_size(_lib.OP_GEMM_PACKED, m, 11008, 4096, 0))
        assert (lib.sp24_workspace_size(_lib.OP_LIFT_GEMM_PACKED, m, 4096, 4096, 0)
                == 256 + lib.sp24_workspace_size(_lib.OP_GEMM_PACKED, m, 4096, 6144, 0))
    assert lib.sp24_workspace_size(_lib.OP_QUANTIZE_GEMM_PACKED, 16, 256, 256, 0) == 256


FAKE = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced: calls fail validation first


def test_validation_rejects_bad_arguments_without_a_gpu(lib):
    ws = 256
    # null pointers
    assert lib.sp24_prune_compress(None, 128, 128, 0, FAKE, FAKE, FAKE, None, FAKE, ws, None, None) == _lib.SP24_ERR_NULL
    assert lib.fp8_quantize_pertensor(FAKE, 4, 32, None, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_NULL
    assert lib.sp24_gemm(FAKE, None, FAKE, None, None, FAKE, 4, 128, 128, 0, FAKE, ws, None, None) == _lib.SP24_ERR_NULL
    # dtype
    assert lib.sp24_prune_compress(FAKE, 128, 128, 7, FAKE, FAKE, FAKE, None, FAKE, ws, None, None) == _lib.SP24_ERR_DTYPE
    assert lib.sp24_gemm(FAKE, None, FAKE, FAKE, None, FAKE, 4, 128, 128, 9, FAKE, ws, None, None) == _lib.SP24_ERR_DTYPE
    # shapes: K not a multiple of the group/tile sizes, N not a multiple of 128, empty M
    assert lib.sp24_prune_compress(FAKE, 128, 12, 0, FAKE, FAKE, FAKE, None, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.slide68_decompose(FAKE, 128, 24, 0, FAKE, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.slide68_lift(FAKE, 0, 64, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.fp8_quantize_pertensor(FAKE, 4, 24, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.sp24_gemm(FAKE, None, FAKE, FAKE, None, FAKE, 4, 128, 192, 0, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.sp24_gemm(FAKE, None, FAKE, FAKE, None, FAKE, 4, 200, 256, 0, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.sp24_gemm(FAKE, None, FAKE, FAKE, None, FAKE, 0, 128, 256, 0, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.fp8_gemm_dense(FAKE, None, FAKE, None, FAKE, 4, 128, 64, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.sp24_prune_compress_packed(FAKE, 128, 192, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.sp24_prune_compress_packed(FAKE, 64, 128, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.sp24_prune_compress_packed(FAKE, 128, 128, FAKE, None, FAKE, ws, None, None) == _lib.SP24_ERR_NULL
    assert lib.slide68_decompose_packed(FAKE, 128, 128, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.slide68_decompose_packed(FAKE, 96, 256, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    # fused quantise + GEMM: M in [1, 256], N % 128, K % 128 (K % 256 with the lift)
    big = 1 << 30
    qg = lib.sp24_quantize_gemm_packed
    lg = lib.slide68_lift_gemm_packed
    assert qg(FAKE, 0, 128, 128, FAKE, None, FAKE, FAKE, FAKE, FAKE, big, None, None) == _lib.SP24_ERR_SHAPE
    assert qg(FAKE, 257, 128, 128, FAKE, None, FAKE, FAKE, FAKE, FAKE, big, None, None) == _lib.SP24_ERR_SHAPE
    assert qg(FAKE, 4, 192, 128, FAKE, None, FAKE, FAKE, FAKE, FAKE, big, None, None) == _lib.SP24_ERR_SHAPE
    assert qg(FAKE, 4, 128, 192, FAKE, None, FAKE, FAKE, FAKE, FAKE, big, None, None) == _lib.SP24_ERR_SHAPE
    assert lg(FAKE, 4, 128, 128, FAKE, None, FAKE, FAKE, FAKE, FAKE, big, None, None) == _lib.SP24_ERR_SHAPE
    assert qg(FAKE, 4, 128, 128, FAKE, None, None, FAKE, FAKE, FAKE, big, None, None) == _lib.SP24_ERR_NULL
    assert qg(FAKE, 4, 128, 128, FAKE, None, FAKE, None, FAKE, FAKE, big, None, None) == _lib.SP24_ERR_NULL
    assert lg(None, 4, 128, 256, FAKE, None, FAKE, FAKE, FAKE, FAKE, big, None, None) == _lib.SP24_ERR_NULL
    # per-token / per-channel scales
    assert lib.fp8_quantize_pertoken(FAKE, 4, 12, FAKE, FAKE, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.fp8_quantize_pertoken(FAKE, 0, 16, FAKE, FAKE, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.fp8_quantize_pertoken(FAKE, 4, 16, FAKE, None, None, None) == _lib.SP24_ERR_NULL
    assert lib.sp24_prune_compress_perchannel(FAKE, 4, 12, FAKE, FAKE, FAKE, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.sp24_prune_compress_perchannel(FAKE, 4, 16, FAKE, None, FAKE, None, None) == _lib.SP24_ERR_NULL
    gs = lib.sp24_gemm_packed_scaled
    assert gs(FAKE, FAKE, 1, FAKE, FAKE, 1, FAKE, 4, 192, 128, FAKE, big, None, None) == _lib.SP24_ERR_SHAPE
    assert gs(FAKE, None, 1, FAKE, FAKE, 1, FAKE, 4, 128, 128, FAKE, big, None, None) == _lib.SP24_ERR_NULL
    # general (2n-2):2n: 3 <= n <= 5, K % 2n == 0, K' % 16 == 0
    sd, sl = lib.slide_decompose, lib.slide_lift
    assert sd(FAKE, 64, 120, 6, FAKE, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert sd(FAKE, 64, 120, 2, FAKE, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert sd(FAKE, 64, 100, 3, FAKE, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert sd(FAKE, 64, 66, 3, FAKE, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE  # K-prime 88
    assert sd(FAKE, 0, 120, 5, FAKE, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert sd(FAKE, 64, 120, 3, FAKE, None, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_NULL
    assert sl(FAKE, 0, 120, 3, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert sl(FAKE, 4, 125, 5, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert sl(FAKE, 4, 120, 5, None, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_NULL
    # INT8: cols % 16 (activations), K % 8 (weights)
    assert lib.int8_quantize_pertensor(FAKE, 4, 24, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.int8_quantize_pertensor(FAKE, 0, 32, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.int8_quantize_pertensor(FAKE, 4, 32, FAKE, None, FAKE, ws, None, None) == _lib.SP24_ERR_NULL
    assert lib.sp24_prune_compress_int8(FAKE, 4, 12, FAKE, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_SHAPE
    assert lib.sp24_prune_compress_int8(FAKE, 4, 16, FAKE, FAKE, None, FAKE, ws, None, None) == _lib.SP24_ERR_NULL
    gi = lib.sp24_gemm_int8_packed
    assert gi(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 192, 128, FAKE, big, None, None) == _lib.SP24_ERR_SHAPE
    assert gi(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 128, 192, FAKE, big, None, None) == _lib.SP24_ERR_SHAPE
    assert gi(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 128, 128, FAKE, big, None, None) == _lib.SP24_ERR_SHAPE
    assert gi(None, FAKE, FAKE, FAKE, FAKE, 4, 128, 128, FAKE, big, None, None) == _lib.SP24_ERR_NULL
    # alignment
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert qg(FAKE, 4, 128, 128, FAKE, None, odd, FAKE, FAKE, FAKE, big, None, None) == _lib.SP24_ERR_ALIGN
    assert lib.fp8_quantize_pertoken(FAKE, 4, 16, odd, FAKE, None, None) == _lib.SP24_ERR_ALIGN
    assert lib.sp24_prune_compress_packed(FAKE, 128, 128, odd, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_ALIGN
    assert lib.fp8_quantize_pertensor(odd, 4, 32, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_ALIGN
    assert lib.slide_decompose(FAKE, 64, 120, 3, odd, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_ALIGN
    assert lib.slide_lift(odd, 4, 120, 5, FAKE, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_ALIGN
    assert lib.int8_quantize_pertensor(FAKE, 4, 32, odd, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_ALIGN
    assert lib.sp24_prune_compress_int8(FAKE, 4, 16, FAKE, odd, FAKE, FAKE, ws, None, None) == _lib.SP24_ERR_ALIGN
    assert lib.sp24_gemm_int8_packed(odd, FAKE, FAKE, FAKE, FAKE, 4, 128, 128, FAKE, big, None, None) == _lib.SP24_ERR_ALIGN
    assert lib.sp24_gemm(FAKE, None, odd, FAKE, None, FAKE, 4, 128, 128, 0, FAKE, ws, None, None) == _lib.SP24_ERR_ALIGN


def test_no_silent_fallback_without_a_sm100_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; the GPU suite covers real calls")
    # valid arguments on a machine without an sm_100 device: the call must refuse
    rc = lib.fp8_quantize_pertensor(FAKE, 4, 32, FAKE, FAKE, FAKE, 256, None, None)
    assert rc == _lib.SP24_ERR_ARCH
