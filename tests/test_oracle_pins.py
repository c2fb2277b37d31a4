"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to an independent source: a library
routine (ml_dtypes / torch FP8 casts), brute force over every small case,
closed forms, invariants the pages state, or the hand-worked fixtures under
``tests/golden/``.  No test here needs a GPU.
"""
import itertools
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import sp24_oracle as O
from structured_sparse_fp8_b200 import workloads as WL

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# E4M3 encode / decode
# --------------------------------------------------------------------------

def _lib_e4m3(v32):
    return np.asarray(v32, dtype=np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def test_e4m3_decode_all_codes_match_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(codes)
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    same = (ours == lib) | (np.isnan(ours) & np.isnan(lib))
    assert same.all()


def test_e4m3_encode_every_bf16_value_in_range():
    bits = np.arange(65536, dtype=np.uint16)
    v = O.bf16_to_f32(bits)
    ok = np.isfinite(v) & (np.abs(v) <= 448.0)
    v = v[ok]
    assert (O.e4m3_encode(v) == _lib_e4m3(v)).all()
    t = torch.from_numpy(v.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (O.e4m3_encode(v) == t).all()


def test_e4m3_encode_strided_fp32_sweep_and_ties():
    # every 97th fp32 bit pattern from +0 up to 464 (beyond the last tie), both signs
    top = np.float32(464.0).view(np.uint32)
    pos = np.arange(0, int(top) + 1, 97, dtype=np.uint32).view(np.float32)
    v = np.concatenate([pos, -pos])
    assert (O.e4m3_encode(v) == _lib_e4m3(v)).all()
    # every midpoint between neighbouring E4M3 values, and one fp32 ulp either side
    grid = np.unique(np.abs(O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))))
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    probe = np.concatenate([mids, np.nextafter(mids, np.float32(0)),
                            np.nextafter(mids, np.float32(1e9))])
    probe = np.concatenate([probe, -probe])
    assert (O.e4m3_encode(probe) == _lib_e4m3(probe)).all()


def test_e4m3_saturates_above_448_and_keeps_sign_of_zero():
    big = np.array([448.0, 460.0, 464.0, 465.0, 1000.0, 3.0e38], dtype=np.float32)
    assert (O.e4m3_encode(big) == 0x7E).all()
    assert (O.e4m3_encode(-big) == 0xFE).all()
    tiny = np.array([0.0, 1e-30, 2.0 ** -10], dtype=np.float32)
    assert (O.e4m3_encode(tiny) == 0x00).all()
    assert (O.e4m3_encode(-tiny) == 0x80).all()


def _lib_bf16(v32):
    return np.asarray(v32, dtype=np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


def test_f32_to_bf16_rne_matches_library_casts():
    # every 65537th finite fp32 bit pattern of both signs (a stride that walks
    # through every low-16-bit residue, so ties, near-ties and exact values)
    u = np.arange(0, 0x7F800000, 65537, dtype=np.uint64).astype(np.uint32)
    v = np.concatenate([u, u | np.uint32(0x80000000)]).view(np.float32)
    assert (O.f32_to_bf16_rne(v) == _lib_bf16(v)).all()
    t = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (O.f32_to_bf16_rne(v) == t).all()
    # every midpoint between neighbouring bf16 values whose exponent field is
    # below the top one, with one fp32 ulp either side: ties go to the even
    # neighbour, everything else to the nearer one
    hi = np.arange(0x0000, 0x7F7F, dtype=np.uint32)
    mid = ((hi << np.uint32(16)) | np.uint32(0x8000)).view(np.float32)
    probe = np.concatenate([mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(np.inf))])
    probe = np.concatenate([probe, -probe])
    assert (O.f32_to_bf16_rne(probe) == _lib_bf16(probe)).all()
    # bf16 values themselves are fixed points
    exact = O.bf16_to_f32(np.arange(0x7F80, dtype=np.uint16))
    assert (O.f32_to_bf16_rne(exact) == np.arange(0x7F80, dtype=np.uint16)).all()


def test_e4m3_golden_landmarks():
    path = os.path.join(GOLDEN, "e4m3_landmarks.txt")
    rows = [ln.split("#")[0].split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    vals = np.array([float.fromhex(r[0]) for r in rows], dtype=np.float32)
    codes = np.array([int(r[1], 16) for r in rows], dtype=np.uint8)
    assert (O.e4m3_encode(vals) == codes).all()


# --------------------------------------------------------------------------
# Scale and quantisation
# --------------------------------------------------------------------------

def test_scale_closed_form_and_zero_tensor():
    x = WL.random_bits((64, 256), 1, scale=3.0)
    a = O.amax(x)
    assert a == np.max(np.abs(x.view(ml_dtypes.bfloat16).astype(np.float64)))
    s = O.scale_from_amax(a)
    assert s == np.float32(np.float32(a) / np.float32(448.0))
    codes, s2 = O.quantize_pertensor(x)
    assert s2 == s
    # the largest magnitude maps onto the top code 0x7E (= 448) exactly
    assert (codes & 0x7F).max() == 0x7E
    z = np.zeros((4, 16), dtype=np.uint16)
    cz, sz = O.quantize_pertensor(z)
    assert sz == np.float32(1.0) and (cz == 0).all()


def test_quantised_dequantised_error_within_e4m3_half_ulp():
    x = WL.random_bits((32, 512), 2)
    codes, s = O.quantize_pertensor(x)
    xv = O.bf16_to_f32(x).astype(np.float64)
    back = O.e4m3_decode(codes) * float(s)
    # relative half-ulp of a 3-bit mantissa, plus the subnormal quantum
    err = np.abs(back - xv)
    assert (err <= np.abs(xv) * 2.0 ** -4 + float(s) * 2.0 ** -10 * 1.0001).all()


# --------------------------------------------------------------------------
# 2:4 and 6:8 pruning against brute force
# --------------------------------------------------------------------------

ALPHABET = [0.0, -0.0, 1.0, -1.0, 2.0]


def _brute_keep(group_vals, keep):
    a = np.abs(np.asarray(group_vals, dtype=np.float64))
    best = None
    for subset in itertools.combinations(range(len(a)), keep):
        key = (-a[list(subset)].sum(), subset)     # max sum, then lexicographically lowest
        if best is None or key < best:
            best = key
    return set(best[1])


def test_prune24_exhaustive_over_tie_alphabet():
    groups = np.array(list(itertools.product(ALPHABET, repeat=4)))
    bits = WL.to_bf16_bits(groups)
    mask = O.prune24_mask(bits)
    for g, m in zip(groups, mask):
        assert set(np.nonzero(m)[0]) == _brute_keep(g, 2), g


def test_prune68_against_brute_force():
    rng = np.random.default_rng(5)
    groups = np.array(list(itertools.product([0.0, 1.0, 2.0], repeat=8)))   # 6561 tie-heavy groups
    groups = np.concatenate([groups * rng.choice([-1, 1], size=groups.shape),
                             rng.normal(size=(2000, 8))])
    bits = WL.to_bf16_bits(groups)
    mask = O.prune68_mask(bits)
    for g, m in zip(bits, mask):
        assert set(np.nonzero(m)[0]) == _brute_keep(O.bf16_to_f32(g), 6)


def test_prune24_matches_the_cookbook_topk_mask_when_no_ties():
    # Practical Example 1 of the cookbook keeps topk(2) of |w| per group of 4 along K.
    w = WL.random_bits((64, 256), 3, scale=0.02)
    wt = torch.from_numpy(O.bf16_to_f32(w).copy())
    g = wt.reshape(64, 64, 4).abs()
    top2 = g.topk(2, dim=-1).indices
    ref = torch.zeros_like(g, dtype=torch.bool).scatter_(-1, top2, True).reshape(64, 64, 4)
    # topk leaves the order of equal magnitudes open: compare the tie-free groups only
    gs = np.sort(g.numpy(), axis=-1)
    tie_free = (np.diff(gs, axis=-1) != 0).all(-1)
    assert tie_free.mean() > 0.9
    ours = O.prune24_mask(w).reshape(64, 64, 4)
    assert (ours[tie_free] == ref.numpy()[tie_free]).all()


def test_prune24_golden_hand_example():
    path = os.path.join(GOLDEN, "prune24_hand_example.txt")
    lines = [ln for ln in open(path) if ln.strip() and not ln.startswith("#")]
    w = np.array([[float(t) for t in ln.split()] for ln in lines[:2]])
    want_mask = np.array([[int(t) for t in ln.split()] for ln in lines[2:4]], dtype=bool)
    want_meta = np.array([[int(t, 16) for t in ln.split()] for ln in lines[4:6]], dtype=np.uint8)
    bits = WL.to_bf16_bits(w)
    mask = O.prune24_mask(bits)
    assert (mask == want_mask).all()
    _, meta = O.compress24(mask, bits)
    assert (meta == want_meta).all()


def test_exactly_two_nonzeros_per_group_on_workload_weights():
    w = WL.weight_bits(1)                    # 256 x 256, N(0, 0.02)
    assert (O.bf16_to_f32(w) != 0).all()     # no exact zeros in practice
    out = O.sp24_prune_compress(w, "bf16")
    nz = (O.bf16_to_f32(out["pruned_dense"]) != 0).reshape(256, 64, 4).sum(-1)
    assert (nz == 2).all()


# --------------------------------------------------------------------------
# Compression round trip and metadata validity
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["e4m3", "bf16"])
def test_compress_roundtrip_bit_exact(dtype):
    w = WL.random_bits((48, 320), 4, scale=0.02, dist="ties" if dtype == "bf16" else "normal")
    out = O.sp24_prune_compress(w, dtype)
    back = O.decompress24(out["values"], out["meta"], 320)
    assert (back == out["pruned_dense"]).all()
    nib = np.stack([out["meta"] & 0xF, out["meta"] >> 4], -1).reshape(48, 80)
    i0, i1 = nib & 3, nib >> 2
    assert (i0 < i1).all() and (i1 <= 3).all()


def test_amax_of_pruned_equals_amax_of_original():
    for seed in range(4):
        w = WL.random_bits((32, 256), 10 + seed, dist="student_t3")
        out = O.sp24_prune_compress(w, "bf16")
        assert O.amax(out["pruned_dense"]) == O.amax(w)


# --------------------------------------------------------------------------
# GEMM: compressed walk vs dense reference, closed-form special cases
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dist", ["normal", "ties"])
def test_sparse_walk_equals_dense_reference(dist):
    x = WL.random_bits((5, 64), 20, dist=dist)
    w = WL.random_bits((7, 64), 21, scale=0.02, dist=dist)
    xq, sx = O.quantize_pertensor(x)
    out = O.sp24_prune_compress(w, "e4m3")
    walk = O.sparse_gemm_walk(O.e4m3_decode(xq), O.e4m3_decode(out["values"]), out["meta"], sx, out["scale"])
    dense, _ = O.gemm_ref(O.e4m3_decode(xq), O.e4m3_decode(out["pruned_dense"]), sx, out["scale"])
    assert np.array_equal(walk, dense)


def test_selection_pattern_reduces_gemm_to_column_picks():
    # Row n of W keeps column c_n with value 1 and a second column with value 0,
    # so Y[:, n] must be exactly X[:, c_n] (a closed form independent of the GEMM).
    k, n = 64, 16
    rng = np.random.default_rng(7)
    cols = rng.integers(0, k, size=n)
    w = np.zeros((n, k))
    w[np.arange(n), cols] = 1.0
    bits = WL.to_bf16_bits(w)
    mask = O.prune24_mask(bits)
    vals, meta = O.compress24(mask, bits)
    x = O.bf16_to_f32(WL.random_bits((3, k), 8)).astype(np.float64)
    y = O.sparse_gemm_walk(x, O.bf16_to_f32(vals), meta)
    assert np.array_equal(y, x[:, cols])


def test_tolerance_rule_is_tight_enough_to_catch_a_dropped_group():
    x = WL.random_bits((4, 256), 30)
    w = WL.random_bits((8, 256), 31, scale=0.02)
    xq, sx = O.quantize_pertensor(x)
    out = O.sp24_prune_compress(w, "e4m3")
    xv, wv = O.e4m3_decode(xq), O.e4m3_decode(out["pruned_dense"])
    y, b = O.gemm_ref(xv, wv, sx, out["scale"])
    wv_bad = wv.copy()
    wv_bad[:, 0:4] = 0.0                   # drop one group of K
    y_bad, _ = O.gemm_ref(xv, wv_bad, sx, out["scale"])
    assert O.within_tolerance(O.bf16_to_f32(O.f32_to_bf16_rne(y.astype(np.float32))), y, b).all()
    assert not O.within_tolerance(y_bad, y, b).all()


# --------------------------------------------------------------------------
# 6:8 sliding windows and lifting
# --------------------------------------------------------------------------

def test_every_68_mask_decomposes_into_three_24_windows():
    for kept in itertools.combinations(range(8), 6):
        m = np.zeros(8, dtype=bool)
        m[list(kept)] = True
        pairs = O.window_assignment(m)
        assert len(pairs) == 3
        used = []
        for j, (p0, p1) in enumerate(pairs):
            assert 2 * j <= p0 < p1 <= 2 * j + 3
            used += [p0, p1]
        assert sorted(used) == sorted(kept)


def test_slide68_reconstructs_pruned_groups_and_gemm_exactly():
    w = WL.random_bits((12, 64), 40, scale=0.02)
    d = O.slide68_decompose(w, "bf16")
    assert d["values"].shape == (12, 48) and d["meta"].shape == (12, 12)   # K' = 1.5 K
    # scatter the expanded operand back onto K: it must equal the 6:8-pruned W
    recon = np.zeros((12, 64), dtype=np.uint16)
    rows, cols = np.nonzero(d["emask"])
    recon[rows, d["src"][rows, cols]] = d["expanded"][rows, cols]
    assert (recon == np.where(d["mask68"], w, 0)).all()
    assert (O.decompress24(d["values"], d["meta"], 96) == d["expanded"]).all()
    x = WL.random_bits((5, 64), 41)
    xv = O.bf16_to_f32(x).astype(np.float64)
    xl = xv[:, O.lift_columns(64)]
    y_lift, _ = O.gemm_ref(xl, O.bf16_to_f32(d["expanded"]))
    y_68, _ = O.gemm_ref(xv, O.bf16_to_f32(np.where(d["mask68"], w, 0)))
    assert np.array_equal(y_lift, y_68)


def test_slide68_golden_hand_example():
    path = os.path.join(GOLDEN, "slide68_hand_example.txt")
    lines = [ln for ln in open(path) if ln.strip() and not ln.startswith("#")]
    kept = [int(t) for t in lines[0].split()]
    want = [tuple(int(t) for t in ln.split()) for ln in lines[1:4]]
    m = np.zeros(8, dtype=bool)
    m[kept] = True
    assert O.window_assignment(m) == want
    want_cols = [int(t) for t in lines[4].split()]
    assert O.lift_columns(8).tolist() == want_cols


def test_lift_codes_are_gathered_codes_and_ratios():
    x = WL.random_bits((6, 64), 50)
    lifted, s = O.slide68_lift(x)
    codes, s2 = O.quantize_pertensor(x)
    assert s == s2 and (lifted == codes[:, O.lift_columns(64)]).all()
    assert lifted.shape[1] / x.shape[1] == 1.5           # gamma = (2N-2)/N for N = 4
    # dense-equivalent work ratio of 6:8-through-2:4 vs dense: 1.5 / 2 = 0.75 -> S_max 4/3
    assert (1.5 * 0.5) == 0.75 and abs(1 / 0.75 - 4 / 3) < 1e-12


# --------------------------------------------------------------------------
# Per-token activation scales, per-channel weight scales
# --------------------------------------------------------------------------

def _powers_of_two_rows(base_bits, n_rows):
    """Rows base * 2^j (exact in bf16: the exponent field of every nonzero
    value moves up by j)."""
    base = np.asarray(base_bits, dtype=np.uint16)
    nz = (base & 0x7FFF) != 0
    rows = [np.where(nz, base + np.uint16(j << 7), base).astype(np.uint16) for j in range(n_rows)]
    return np.stack(rows)


def test_pertoken_scales_follow_row_magnitude_exactly():
    base = WL.random_bits((1, 256), 71)[0]
    x = _powers_of_two_rows(base, 6)
    codes, scales = O.quantize_pertoken(x)
    assert scales.dtype == np.float32 and codes.dtype == np.uint8
    for j in range(6):
        # scaling a row by 2^j scales its amax, hence its scale, by 2^j and
        # leaves every quotient x / s, hence every code, unchanged
        assert scales[j] == np.float32(scales[0] * 2.0 ** j)
        assert np.array_equal(codes[j], codes[0])
        # the row's largest magnitude maps exactly to 448 (code 0x7E)
        assert (codes[j] & 0x7F).max() == 0x7E
    # a single row is quantised exactly as the per-tensor path quantises it
    c1, s1 = O.quantize_pertensor(x[3])
    assert np.array_equal(codes[3], c1) and scales[3] == s1


def test_pertoken_zero_row_takes_scale_one():
    x = WL.random_bits((3, 64), 72)
    x[1] = 0
    codes, scales = O.quantize_pertoken(x)
    assert scales[1] == np.float32(1.0) and not codes[1].any()


def test_perchannel_prune_selects_like_per_tensor_and_scales_each_row():
    base = WL.random_bits((1, 512), 73, scale=0.02)[0]
    w = _powers_of_two_rows(base, 5)
    r = O.sp24_prune_compress_perchannel(w)
    assert np.array_equal(r["mask"], O.prune24_mask(w))
    for j in range(5):
        assert r["scales"][j] == np.float32(r["scales"][0] * 2.0 ** j)
        assert np.array_equal(r["values"][j], r["values"][0])
        assert np.array_equal(r["meta"][j], r["meta"][0])
        assert (r["values"][j] & 0x7F).max() == 0x7E
    # one row alone is the per-tensor weight path of that row
    one = O.sp24_prune_compress(w[2:3], "e4m3")
    assert np.array_equal(r["values"][2], one["values"][0]) and r["scales"][2] == one["scale"]


def test_scaled_gemm_reduces_to_the_pinned_reference():
    x = O.e4m3_decode(WL.random_bits((4, 64), 74).astype(np.uint8) & 0x7E)
    w = O.e4m3_decode(WL.random_bits((6, 64), 75).astype(np.uint8) & 0x7E)
    y0, b0 = O.gemm_ref(x, w)
    sx = np.array([2.0 ** m for m in range(4)], dtype=np.float32)
    sw = np.array([2.0 ** -n for n in range(6)], dtype=np.float32)
    y, b = O.gemm_ref_scaled(x, w, sx, sw)
    assert np.array_equal(y, y0 * np.outer(sx, sw)) and np.array_equal(b, b0 * np.outer(sx, sw))
    y1, b1 = O.gemm_ref_scaled(x, w, np.float32(0.5), np.float32(3.0))
    y2, b2 = O.gemm_ref(x, w, np.float32(0.5), np.float32(3.0))
    assert np.array_equal(y1, y2) and np.array_equal(b1, b2)


# --------------------------------------------------------------------------
# General (2N-2):2N windows
# --------------------------------------------------------------------------

def test_general_slide_reduces_to_the_pinned_68_functions():
    w = WL.random_bits((5, 64), 91, scale=0.02, dist="ties")
    g, r68 = O.slide_decompose(w, 4), O.slide68_decompose(w, "e4m3")
    for key in ("values", "meta", "emask", "expanded"):
        assert np.array_equal(g[key], r68[key]), key
    assert g["scale"] == r68["scale"]
    assert np.array_equal(O.slide_lift_columns(64, 4), O.lift_columns(64))


@pytest.mark.parametrize("n", [3, 4, 5])
def test_general_slide_every_mask_fills_its_windows(n):
    g2 = 2 * n
    for pruned in itertools.combinations(range(g2), 2):
        kept = np.ones(g2, dtype=bool)
        kept[list(pruned)] = False
        pairs = O.slide_windows(kept, n)
        assert len(pairs) == n - 1
        for j, (p0, p1) in enumerate(pairs):
            assert 2 * j <= p0 < p1 <= 2 * j + 3
        assert sorted(p for pr in pairs for p in pr) == list(np.nonzero(kept)[0])


@pytest.mark.parametrize("n", [3, 5])
def test_general_slide_reconstructs_and_gemm_is_exact(n):
    k = 4 * n * 2
    w = WL.random_bits((6, k), 92 + n, scale=0.02)
    x = WL.random_bits((3, k), 94 + n)
    d = O.slide_decompose(w, n)
    kp = k * (2 * n - 2) // n
    assert d["expanded"].shape == (6, kp) and kp / k == (2 * n - 2) / n
    # every window is 2:4 and scattering the expanded operand back gives the
    # pruned, quantised W exactly
    assert (d["emask"].reshape(6, -1, 4).sum(axis=2) == 2).all()
    codes = O.quantize_with_scale(w, d["scale"])
    back = np.zeros_like(codes)
    for row in range(6):
        for col in np.nonzero(d["emask"][row])[0]:
            back[row, d["src"][row, col]] = d["expanded"][row, col]
    assert np.array_equal(back, np.where(d["mask"], codes, np.uint8(0)))
    # X' W'^T = X W_pruned^T exactly in float64 (products of E4M3 values)
    xq, sx = O.quantize_pertensor(x)
    xl, sxl = O.slide_lift(x, n)
    assert sxl == sx
    y1, _ = O.gemm_ref(O.e4m3_decode(xl), O.e4m3_decode(d["expanded"]))
    y2, _ = O.gemm_ref(O.e4m3_decode(xq), O.e4m3_decode(back))
    assert np.array_equal(y1, y2)


# ------------------------------------------------------------ INT8 W8A8 with 2:4 weights

def test_int8_golden_hand_example():
    lines = [ln.split() for ln in open(os.path.join(GOLDEN, "int8_hand_example.txt"))
             if ln.strip() and not ln.startswith("#")]
    for vals, codes, scale in ((lines[0], lines[1], lines[2]), (lines[3], lines[4], lines[5])):
        bits = WL.to_bf16_bits(np.array([float(v) for v in vals]))[None, :]
        q, s = O.int8_quantize_pertensor(bits)
        assert float(s) == float(scale[0])
        assert q[0].tolist() == [int(c) for c in codes]


def test_int8_matches_torch_quantizer_away_from_rounding_ties():
    """torch's per-tensor qint8 quantiser (zero point 0) rounds x / s to the
    nearest integer on its own code path; it multiplies by the reciprocal of
    s, so the comparison leaves out quotients within 1e-5 of a half-integer."""
    x = WL.random_bits((64, 512), 4000, dist="student_t3")
    q, s = O.int8_quantize_pertensor(x)
    xf = O.bf16_to_f32(x)
    tq = torch.quantize_per_tensor(torch.from_numpy(xf), float(s), 0, torch.qint8).int_repr().numpy()
    r = xf.astype(np.float64) / float(s)
    far = np.abs(np.abs(r - np.floor(r)) - 0.5) > 1e-5
    assert far.mean() > 0.99
    assert np.array_equal(q[far], tq[far])


def test_int8_every_bf16_value_within_half_a_step():
    """Every finite bf16 value with |x| <= amax = 3: the code is within half a
    step of x / s (plus the fp32 quotient's rounding), exact half-way cases go
    to the even code, |q| <= 127 and +-amax code to +-127."""
    s = O.int8_scale_from_amax(np.float32(3.0))
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = O.bf16_to_f32(bits)
    sel = np.isfinite(x) & (np.abs(x) <= 3.0)
    q = O.int8_quantize_with_scale(bits[sel], s).astype(np.int64)
    r = x[sel].astype(np.float64) / np.float64(s)
    assert (np.abs(q - r) <= 0.5 + 2.0 ** -23 * np.abs(r) + 1e-12).all()
    half = (2 * r == np.round(2 * r)) & (r != np.round(r))
    assert (q[half] % 2 == 0).all()
    assert np.abs(q).max() == 127
    ends = O.int8_quantize_with_scale(WL.to_bf16_bits(np.array([[3.0, -3.0]])), s)
    assert ends.tolist() == [[127, -127]]


def test_int8_zero_tensor_and_dequantisation_error():
    q, s = O.int8_quantize_pertensor(np.zeros((4, 16), dtype=np.uint16))
    assert s == np.float32(1.0) and not q.any()
    x = WL.random_bits((32, 256), 4050)
    q, s = O.int8_quantize_pertensor(x)
    err = np.abs(q.astype(np.float64) * np.float64(s) - O.bf16_to_f32(x).astype(np.float64))
    assert (err <= 0.5 * np.float64(s) * (1 + 1e-6)).all()


def test_int8_prune_compress_selects_like_fp8():
    w = WL.random_bits((64, 256), 4100, scale=0.02, dist="ties")
    d = O.sp24_prune_compress_int8(w)
    ref = O.sp24_prune_compress(w, "e4m3")
    assert np.array_equal(d["mask"], ref["mask"]) and np.array_equal(d["meta"], ref["meta"])
    assert np.array_equal(O.decompress24(d["values"], d["meta"], 256), d["pruned_dense"])
    q, s = O.int8_quantize_pertensor(w)
    assert s == d["scale"]
    assert np.array_equal(np.where(d["mask"], q, 0), d["pruned_dense"])


def test_int8_gemm_is_the_exact_integer_product():
    """The integer sums equal a walk over the compressed operand in plain
    loops (the pinned format), Y and B equal the pinned float64 reference on
    the same integers, and the largest K used keeps every sum inside int32."""
    x = WL.random_bits((3, 64), 4200)
    w = WL.random_bits((5, 64), 4201, scale=0.02)
    xq, sx = O.int8_quantize_pertensor(x)
    d = O.sp24_prune_compress_int8(w)
    y, b, acc = O.gemm_ref_int8(xq, d["pruned_dense"], sx, d["scale"])
    assert np.array_equal(O.sparse_gemm_walk(xq, d["values"], d["meta"]), acc.astype(np.float64))
    y2, b2 = O.gemm_ref(xq, d["pruned_dense"], sx, d["scale"])
    assert np.array_equal(y, y2) and np.array_equal(b, b2)
    assert 14336 // 2 * 127 * 127 < 2 ** 31


def _golden_cases(name):
    cases, cur = [], None
    for ln in open(os.path.join(GOLDEN, name)):
        if not ln.strip() or ln.startswith("#"):
            continue
        key, *rest = ln.split()
        if key == "n":
            cur = {"n": int(rest[0])}
            cases.append(cur)
        else:
            cur[key] = rest
    return cases


def test_general_slide_golden_hand_examples():
    for c in _golden_cases("slide_general_hand_example.txt"):
        n = c["n"]
        w = WL.to_bf16_bits(np.array([[float(v) for v in c["w"]]]))
        assert np.nonzero(O.slide_mask(w, n)[0])[0].tolist() == [int(v) for v in c["kept"]]
        pairs = [tuple(int(p) for p in wp.split(",")) for wp in c["windows"]]
        assert O.slide_windows(O.slide_mask(w, n)[0], n) == pairs
        d = O.slide_decompose(w, n)
        assert d["meta"][0].tolist() == [int(b, 16) for b in c["meta"]]
        assert d["src"][0][d["emask"][0]].tolist() == [int(v) for v in c["src"]]
        assert O.slide_lift_columns(2 * n, n).tolist() == [int(v) for v in c["lift"]]


# ------------------------------------------------------------ FP4 (E2M1) with 2:4 weights

def test_e2m1_decode_all_codes_match_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    want = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(O.e2m1_decode(codes), want)
    assert np.array_equal(np.signbit(O.e2m1_decode(codes)), codes >= 8)


def test_e2m1_encode_every_bf16_value_matches_ml_dtypes():
    """ml_dtypes' float4_e2m1fn cast (round to nearest even, saturating, sign
    kept on zero) over every finite bf16 value up to |x| = 16, and a strided
    fp32 sweep through every tie."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = O.bf16_to_f32(bits)
    x = x[np.isfinite(x) & (np.abs(x) <= 16)]
    assert np.array_equal(O.e2m1_encode(x), x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8))
    sweep = np.linspace(-7, 7, 56001, dtype=np.float32)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    sweep = np.concatenate([sweep, ties, -ties, np.nextafter(ties, 0), np.nextafter(ties, 9)])
    assert np.array_equal(O.e2m1_encode(sweep), sweep.astype(ml_dtypes.float4_e2m1fn).view(np.uint8))


def test_fp4_golden_hand_example():
    lines = [ln.split() for ln in open(os.path.join(GOLDEN, "fp4_hand_example.txt"))
             if ln.strip() and not ln.startswith("#")]
    for vals, codes, scale in ((lines[0], lines[1], lines[2]), (lines[3], lines[4], lines[5])):
        bits = WL.to_bf16_bits(np.array([float(v) for v in vals]))[None, :]
        q, s = O.fp4_quantize_pertensor(bits)
        assert float(s) == float(scale[0])
        assert q[0].tolist() == [int(c) for c in codes]


def test_fp4_scale_maps_amax_to_six_and_zero_tensor():
    x = WL.random_bits((16, 128), 4500, dist="student_t3")
    q, s = O.fp4_quantize_pertensor(x)
    xf = O.bf16_to_f32(x)
    top = np.abs(xf) == np.abs(xf).max()
    assert (q[top] & 7 == 7).all()
    dq = O.e2m1_decode(q) * np.float64(s)
    # relative error of a normal E2M1 value is at most a quarter (half of 2^-1)
    big = np.abs(xf) >= np.float64(s)
    assert (np.abs(dq[big] - xf[big]) <= 0.25 * np.abs(xf[big]) + 1e-12).all()
    q0, s0 = O.fp4_quantize_pertensor(np.zeros((2, 8), dtype=np.uint16))
    assert s0 == np.float32(1.0) and not q0.any()


def test_fp4_prune_compress_and_gemm_reduce_to_pinned_functions():
    w = WL.random_bits((32, 128), 4600, scale=0.02, dist="ties")
    d = O.sp24_prune_compress_fp4(w)
    ref = O.sp24_prune_compress(w, "e4m3")
    assert np.array_equal(d["mask"], ref["mask"]) and np.array_equal(d["meta"], ref["meta"])
    assert np.array_equal(O.decompress24(d["values"], d["meta"], 128), d["pruned_dense"])
    q, s = O.fp4_quantize_pertensor(w)
    assert s == d["scale"] and np.array_equal(np.where(d["mask"], q, 0), d["pruned_dense"])
    x = WL.random_bits((3, 128), 4601)
    xq, sx = O.fp4_quantize_pertensor(x)
    xv, wv = O.e2m1_decode(xq), O.e2m1_decode(d["pruned_dense"])
    y, _ = O.gemm_ref(xv, wv, sx, d["scale"])
    walk = O.sparse_gemm_walk(xv, O.e2m1_decode(d["values"]), d["meta"], sx, d["scale"])
    assert np.allclose(walk, y, rtol=0, atol=1e-12 * np.abs(y).max())
