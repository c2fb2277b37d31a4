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
    # fused quantise (or lift) + GEMM: 8 KB of counters, published copies and
    # per-CTA slots, then the GEMM's workspace at K (or K' = 3K/2)
    for m in (1, 8, 32, 64, 256):
        assert (lib.sp24_workspace_size(_lib.OP_QUANTIZE_GEMM_PACKED, m, 11008, 4096, 0)
                == 8192 + lib.sp24_workspace_size(_lib.OP_GEMM_PACKED, m, 11008, 4096, 0))
        assert (lib.sp24_workspace_size(_lib.OP_LIFT_GEMM_PACKED, m, 4096, 4096, 0)
                == 8192 + lib.sp24_workspace_size(_lib.OP_GEMM_PACKED, m, 4096, 6144, 0))
    assert lib.sp24_workspace_size(_lib.OP_QUANTIZE_GEMM_PACKED, 16, 256, 256, 0) == 8192


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


def _header_declarations():
    import re
    text = re.sub(r"/\*.*?\*/", "", open(_lib.HEADER).read(), flags=re.S)
    decls = {}
    for ret, name, params in re.findall(r"^\s*((?:const\s+)?[a-z_0-9]+\s*\**)\s*([a-z_0-9]+)\s*\(([^)]*)\)\s*;",
                                        text, flags=re.M):
        plist = [p.strip() for p in params.split(",") if p.strip() and p.strip() != "void"]
        decls[name] = (ret.strip(), plist)
    return decls


def _ctype_of(param):
    if "*" in param or "sp24_stream_t" in param:
        return ctypes.c_void_p
    if "int64_t" in param:
        return ctypes.c_int64
    if "size_t" in param:
        return ctypes.c_size_t
    if param.startswith("int ") or param == "int":
        return ctypes.c_int
    raise AssertionError(f"unclassified parameter {param!r}")


def test_binding_signatures_match_the_header():
    """Every ctypes signature has the header's parameter count and kinds
    (pointer, int, int64_t, size_t) and return type: a binding that passed
    an argument in the wrong slot or width would fail here, not on a GPU."""
    decls = _header_declarations()
    assert set(decls) == set(_lib.header_functions())
    rets = {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "const char *": ctypes.c_char_p}
    for name, (ret, params) in decls.items():
        res, args = _lib.SIGNATURES[name]
        assert rets[" ".join(ret.replace("*", " *").split())] is res, name
        assert [_ctype_of(p) for p in params] == list(args), name


def test_bindings_marshal_arguments_in_header_order(monkeypatch):
    """The Python bindings of the sliding-window and INT8 entry points pass
    the right tensors, sizes and stream in the header's order, and size their
    outputs as the header states (a recording stand-in for the library, CPU
    tensors; nothing is computed)."""
    import torch

    import structured_sparse_fp8_b200 as sp

    calls = {}

    class Recorder:
        def __getattr__(self, name):
            def f(*args):
                calls[name] = args
                return 512 if name == "sp24_workspace_size" else 0
            return f

    monkeypatch.setattr(sp._lib, "load", lambda: Recorder())
    monkeypatch.setattr(sp, "_require_cuda", lambda *ts: None)
    monkeypatch.setattr(sp, "_stream", lambda device: 777)
    ws = sp.Workspace("cpu")
    wsp = ws.get(512).data_ptr()

    def check(name, expect):
        got = calls[name]
        assert len(got) == len(_lib.SIGNATURES[name][1]), name
        assert got[:-3] + got[-2:] == expect[:-3] + expect[-2:], name   # all but the workspace size
        assert got[-3] >= 512 or name.endswith("packed"), name

    W = torch.zeros((8, 120), dtype=torch.bfloat16)
    d = sp.slide_decompose(W, 3, workspace=ws)
    assert d["values"].shape == (8, 80) and d["meta"].shape == (8, 20)   # K' = 120 * 4 / 3 = 160
    check("slide_decompose", (W.data_ptr(), 8, 120, 3, d["values"].data_ptr(), d["meta"].data_ptr(),
                              d["scale"].data_ptr(), wsp, 512, None, 777))
    X = torch.zeros((4, 120), dtype=torch.bfloat16)
    q, s = sp.slide_lift(X, 5, workspace=ws)
    assert q.shape == (4, 192) and q.dtype == torch.uint8                  # K' = 120 * 8 / 5
    check("slide_lift", (X.data_ptr(), 4, 120, 5, q.data_ptr(), s.data_ptr(), wsp, 512, None, 777))
    X = torch.zeros((4, 32), dtype=torch.bfloat16)
    q, s = sp.int8_quantize_pertensor(X, workspace=ws)
    assert q.shape == (4, 32) and q.dtype == torch.int8
    check("int8_quantize_pertensor", (X.data_ptr(), 4, 32, q.data_ptr(), s.data_ptr(), wsp, 512, None, 777))
    W = torch.zeros((8, 64), dtype=torch.bfloat16)
    c = sp.sp24_prune_compress_int8(W, workspace=ws)
    assert c["values"].shape == (8, 32) and c["values"].dtype == torch.int8 and c["meta"].shape == (8, 8)
    check("sp24_prune_compress_int8", (W.data_ptr(), 8, 64, c["values"].data_ptr(), c["meta"].data_ptr(),
                                       c["scale"].data_ptr(), wsp, 512, None, 777))
    xq = torch.zeros((4, 128), dtype=torch.int8)
    packed = torch.zeros(128 * 128 // 2 + 128 * 128 // 8, dtype=torch.uint8)
    sx, sw = torch.ones(1), torch.ones(1)
    y = sp.sp24_gemm_int8_packed(xq, sx, packed, sw, 128, workspace=ws)
    assert y.shape == (4, 128) and y.dtype == torch.bfloat16
    check("sp24_gemm_int8_packed", (xq.data_ptr(), sx.data_ptr(), packed.data_ptr(), sw.data_ptr(), y.data_ptr(),
                                    4, 128, 128, wsp, 512, None, 777))
    with pytest.raises(sp.Sp24Error):
        sp.sp24_gemm_int8_packed(xq.view(torch.uint8), sx, packed, sw, 128, workspace=ws)
