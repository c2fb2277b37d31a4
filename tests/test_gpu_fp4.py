"""FP4 (E2M1) with 2:4 weights through the C ABI against the CPU oracle.

Codes (two per byte, element 2i in the low nibble of byte i), metadata and
scales must be bit-exact; the sparse GEMM (tcgen05.mma.sp kind::f8f6f4 with
E2M1 operands) must meet |y - y_ref| <= 1e-3 * B + 1e-2 * |y_ref| elementwise
against the oracle's float64 GEMM on the decoded E2M1 codes.
"""
import numpy as np
import pytest
import torch

from oracle import sp24_oracle as O
from structured_sparse_fp8_b200 import workloads as WL

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _built():
    import __graft_entry__
    __graft_entry__.build()
    torch.cuda.set_device(DEV)


def sp():
    import structured_sparse_fp8_b200 as m
    return m


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def pack(codes):
    """E2M1 codes (0..15, last axis even) -> bytes, element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack(b):
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


# small tensors take the direct (division) form, large ones the table form
@pytest.mark.parametrize("shape,seed,scale", [((1, 32), 1, 1.0), ((3, 64), 2, 2.0), ((37, 4096), 3, 1.0),
                                              ((64, 14336), 4, 0.5), ((512, 4096), 5, 1.0)])
def test_fp4_quantize_bit_exact(shape, seed, scale):
    x = WL.random_bits(shape, seed, scale=scale)
    st = status()
    q, s = sp().fp4_quantize_pertensor(dev_bf16(x), status=st)
    ref_q, ref_s = O.fp4_quantize_pertensor(x)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert s.item() == float(ref_s)
    assert np.array_equal(unpack(q.cpu().numpy()), ref_q)


@pytest.mark.parametrize("amax_bits", [0x40C0, 0x3F80, 0x3D18, 0x447A])
def test_fp4_quantize_every_bf16_value(amax_bits):
    """Every finite bf16 value of magnitude <= amax, in each kernel form:
    every rounding decision of the E2M1 encoder at the scale amax / 6."""
    v = O.bf16_to_f32(np.arange(65536, dtype=np.uint16))
    amax = O.bf16_to_f32(np.array([amax_bits], dtype=np.uint16))[0]
    bits = np.arange(65536, dtype=np.uint16)[np.isfinite(v) & (np.abs(v) <= amax)]
    bits = np.concatenate([np.array([amax_bits], dtype=np.uint16), bits])
    # one thread-block cluster (<= 131072 values), the two-launch direct form,
    # the table form
    for reps in (1, 5, 40):
        flat = np.tile(bits, reps)
        k = 4096
        x = np.zeros(-(-len(flat) // k) * k, dtype=np.uint16)
        x[:len(flat)] = flat
        x = x.reshape(-1, k)
        q, s = sp().fp4_quantize_pertensor(dev_bf16(x))
        ref_q, ref_s = O.fp4_quantize_pertensor(x)
        assert s.item() == float(ref_s)
        assert np.array_equal(unpack(q.cpu().numpy()), ref_q), reps


@pytest.mark.parametrize("dist", ["normal", "ties", "student_t3"])
@pytest.mark.parametrize("shape", [(96, 256), (1024, 2048)])
def test_fp4_prune_compress_bit_exact(dist, shape):
    w = WL.random_bits(shape, 2400, scale=0.02, dist=dist)
    st = status()
    c = sp().sp24_prune_compress_fp4(dev_bf16(w), status=st)
    ref = O.sp24_prune_compress_fp4(w)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert c["scale"].item() == float(ref["scale"])
    assert np.array_equal(c["meta"].cpu().numpy(), ref["meta"])
    assert np.array_equal(unpack(c["values"].cpu().numpy()), ref["values"])


def _gemm_case(m, n, k, seed, check_rows=None):
    x = WL.random_bits((m, k), seed)
    w = WL.random_bits((n, k), seed + 1, scale=0.02)
    ref_q, ref_sx = O.fp4_quantize_pertensor(x)
    ref_w = O.sp24_prune_compress_fp4(w)
    xq = torch.from_numpy(pack(ref_q)).to(DEV)
    vals = torch.from_numpy(pack(ref_w["values"])).to(DEV)
    meta = torch.from_numpy(ref_w["meta"]).to(DEV)
    sx = torch.tensor([ref_sx], dtype=torch.float32, device=DEV)
    sw = torch.tensor([ref_w["scale"]], dtype=torch.float32, device=DEV)
    st = status()
    y = sp().sp24_gemm_fp4(xq, sx, vals, meta, sw, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = np.arange(m) if check_rows is None else check_rows
    xv = O.e2m1_decode(ref_q[rows])
    wv = O.e2m1_decode(ref_w["pruned_dense"])
    y_ref, b = O.gemm_ref(xv, wv, ref_sx, ref_w["scale"])
    yv = O.bf16_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16)[rows]).astype(np.float64)
    ok = O.within_tolerance(yv, y_ref, b)
    assert ok.all(), f"{int((~ok).sum())} of {ok.size} outside tolerance; first {np.argwhere(~ok)[:4].tolist()}"
    return y


@pytest.mark.parametrize("m,n,k", [(1, 128, 256), (16, 256, 512), (33, 384, 1024), (64, 128, 768),
                                   (200, 256, 512), (300, 384, 1280)])
def test_fp4_gemm_within_tolerance(m, n, k):
    _gemm_case(m, n, k, 2500 + m)


def test_fp4_gemm_decode_workload_and_end_to_end():
    """The decode up-projection shape on oracle operands (every output), and the
    whole FP4 path on the device: quantise X, prune + compress W, GEMM."""
    _gemm_case(8, 11008, 4096, 2600)
    x = WL.activation_bits(2, 64)
    w = WL.weight_bits(2)
    st = status()
    xq, sx = sp().fp4_quantize_pertensor(dev_bf16(x), status=st)
    c = sp().sp24_prune_compress_fp4(dev_bf16(w), status=st)
    y = sp().sp24_gemm_fp4(xq, sx, c["values"], c["meta"], c["scale"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = np.arange(0, 11008, 43)          # a sample of W rows, under the whole tensor's scale
    ref_q, ref_sx = O.fp4_quantize_pertensor(x)
    sw = O.fp4_scale_from_amax(O.amax(w))
    assert c["scale"].item() == float(sw)
    dense = np.where(O.prune24_mask(w[rows]), O.fp4_quantize_with_scale(w[rows], sw), 0).astype(np.uint8)
    assert np.array_equal(unpack(xq.cpu().numpy()), ref_q)
    y_ref, b = O.gemm_ref(O.e2m1_decode(ref_q), O.e2m1_decode(dense), ref_sx, sw)
    yv = O.bf16_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16)[:, rows]).astype(np.float64)
    assert O.within_tolerance(yv, y_ref, b).all()
