"""CPU oracle for the 2:4 structured-sparse FP8 GEMM path (test infrastructure).

THIS MODULE IS TEST INFRASTRUCTURE.  Only the tests, the package's ``smoke()``
check and the benchmark's CPU-baseline leg may import it.  The product path
(the CUDA library behind ``include/sp24.h``) never calls it, shares no code,
table or constant generator with it, and must fail loudly when its extension
is missing instead of falling back to anything here.

Every function below is the plain definition of one step of the method,
written with numpy in float64 (FP8 codes, bf16 bit patterns and metadata are
integers).  Where the pages leave a step open the reading taken is stated in
the function's docstring.  Pages cited:

* "Deploying 2:4 Sparsity with FP8 on Hopper: A Production Cookbook"
  (the cookbook) -- pipeline steps 2-4 and 6, Practical Example 1
  ("2:4 mask application").
* "SlideSparse: Fast and Flexible (2N-2):2N Structured Sparsity" (the
  SlideSparse summary) -- Resumen tecnico §2 Metodologia: "Descomposicion de
  Ventana Deslizante", "Levantamiento de Activacion", "Pipeline de
  Implementacion"; the lay "Analogia de la Ventana Deslizante".
* the cookbook's Comparison Tables ("INT8 W8A8" recipe) and the SlideSparse
  summary's §3-§4 (INT8 and FP4 among its precisions) for the INT8 and FP4
  functions.
* "La Densite Dynamique et les Noyaux Non Structures ..." (the roadmap) --
  §Lacunes des noyaux (compressed metadata), §Interaction avec la
  quantification (per-tensor FP8 scaling).

Conventions shared with the CUDA path (fixed here, from the readings):

* bf16 tensors are passed around as ``uint16`` bit patterns.
* E4M3 means the OCP FP8 "E4M3FN" format: bias 7, 3 mantissa bits, no
  infinities, NaN = S.1111.111, largest finite 448.
* 2:4 groups are 4 contiguous values along K (the last axis).
* Compressed layout: ``values[n, 2g + t]`` is the t-th kept element of group
  g in ascending index order; ``meta[n, b]`` holds group 2b in bits 0-3 and
  group 2b+1 in bits 4-7, each nibble ``i0 | i1 << 2`` with ``i0 < i1``.

All functions are parity-pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0

# ---------------------------------------------------------------------------
# bf16 helpers (definition of the bf16 format: the top 16 bits of a float32)
# ---------------------------------------------------------------------------


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 bit patterns, round-to-nearest-even.

    Used only to express the bf16 rounding of an output; NaN is not expected.
    """
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = u + np.uint64(0x7FFF) + lsb
    return (u >> np.uint64(16)).astype(np.uint16)


def _require_finite(x: np.ndarray, what: str) -> None:
    if not np.all(np.isfinite(x)):
        raise ValueError(f"{what}: the method is defined for finite inputs only")


# ---------------------------------------------------------------------------
# FP8 E4M3 (per-tensor dynamic scaling: the cookbook, pipeline steps 3 and 6;
# the roadmap, §Interaction avec la quantification)
# ---------------------------------------------------------------------------


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Encode float32 values as E4M3 codes: round to nearest even, saturating.

    Written from the format's definition: a value with |v| >= 2**-6 has
    quantum 2**(e-3) where e = floor(log2 |v|); below that the grid is the
    subnormal one with quantum 2**-9.  Rounding is to nearest, ties to even
    (numpy's ``rint``), done in float64 where dividing by a power of two is
    exact.  Magnitudes that round above 448 saturate to 448 (the
    "satfinite" reading).  The sign of v is kept, so a negative value that
    rounds to zero gives the code 0x80.  NaN gives 0x7F.
    """
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v.astype(np.float64))
    neg = np.signbit(v)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    _require_finite(a, "e4m3_encode")
    _, ex = np.frexp(a)                      # a = m * 2**ex, m in [0.5, 1)
    e = np.maximum(ex.astype(np.int64) - 1, -6)
    quantum = np.ldexp(1.0, (e - 3).astype(np.int32))
    q = np.rint(a / quantum) * quantum       # nearest grid point, ties to even
    q = np.minimum(q, E4M3_MAX)              # saturate
    # q is now exactly representable; split it into exponent and mantissa.
    code = np.zeros(a.shape, dtype=np.int64)
    sub = q < 2.0 ** -6
    code = np.where(sub, np.rint(q / 2.0 ** -9).astype(np.int64), code)
    _, qex = np.frexp(np.where(sub, 1.0, q))
    qe = qex.astype(np.int64) - 1            # floor(log2 q) for normal q
    mant = np.rint(np.ldexp(np.where(sub, 1.0, q), (3 - qe).astype(np.int32))).astype(np.int64) - 8
    normal_code = ((qe + 7) << 3) | mant
    code = np.where(sub, code, normal_code)
    code = code | np.where(neg, 0x80, 0)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each E4M3 code as float64 (NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(ef == 0, m * 2.0 ** -9,
                   (1.0 + m / 8.0) * np.ldexp(1.0, (ef - 7).astype(np.int32)))
    val = np.where((ef == 15) & (m == 7), np.nan, val)
    return s * val


def amax(bits: np.ndarray) -> np.float32:
    """Largest |x| of a bf16 tensor, as float32 (exact: a max of bf16 values)."""
    x = bf16_to_f32(bits)
    _require_finite(x, "amax")
    if x.size == 0:
        return np.float32(0.0)
    return np.float32(np.max(np.abs(x)))


def scale_from_amax(a: np.float32) -> np.float32:
    """Per-tensor dequantisation scale s = amax / 448, one fp32 division.

    Reading: when amax is 0 the scale is taken as 1.0 (every code is then 0).
    """
    a = np.float32(a)
    if a == 0:
        return np.float32(1.0)
    return np.float32(a / np.float32(E4M3_MAX))


def quantize_with_scale(bits: np.ndarray, s: np.float32) -> np.ndarray:
    """E4M3 codes of x / s, the quotient taken as one correctly rounded fp32
    division (reading: divide by the dequantisation scale, not multiply by
    its reciprocal)."""
    x = bf16_to_f32(bits)
    v = (x / np.float32(s)).astype(np.float32)
    return e4m3_encode(v)


def quantize_pertensor(bits: np.ndarray):
    """Per-tensor dynamic E4M3 quantisation: returns (codes, scale)."""
    s = scale_from_amax(amax(bits))
    return quantize_with_scale(bits, s), s


# ---------------------------------------------------------------------------
# N:M magnitude pruning along K (the cookbook, pipeline step 4 and Practical
# Example 1; the SlideSparse summary, §1 for 6:8)
# ---------------------------------------------------------------------------


def keep_mask(bits: np.ndarray, group: int, keep: int) -> np.ndarray:
    """Magnitude N:M mask along the last axis.

    In every group of ``group`` contiguous values, element i beats element j
    when |w_i| > |w_j|, or |w_i| == |w_j| and i < j (ties go to the lower
    index; -0 and +0 are equal).  An element is kept when fewer than ``keep``
    elements of its group beat it, which keeps exactly ``keep`` per group.
    """
    w = bf16_to_f32(bits)
    _require_finite(w, "keep_mask")
    if w.shape[-1] % group:
        raise ValueError(f"K={w.shape[-1]} is not a multiple of {group}")
    a = np.abs(w).reshape(*w.shape[:-1], w.shape[-1] // group, group).astype(np.float64)
    idx = np.arange(group)
    ai = a[..., :, None]
    aj = a[..., None, :]
    beats = (aj > ai) | ((aj == ai) & (idx[None, :] < idx[:, None]))
    rank = beats.sum(axis=-1)
    return (rank < keep).reshape(w.shape)


def prune24_mask(bits: np.ndarray) -> np.ndarray:
    """2:4 magnitude mask: the two largest |w| of each 4 along K survive."""
    return keep_mask(bits, 4, 2)


def compress24(mask: np.ndarray, payload: np.ndarray):
    """Compress a 2:4-masked [N, K] array into (values [N, K/2], meta [N, K/8]).

    ``payload`` is whatever is stored per kept element (E4M3 codes or bf16
    bit patterns).  Requires exactly two kept elements per group of 4.
    """
    mask = np.asarray(mask, dtype=bool)
    n, k = mask.shape
    if k % 8:
        raise ValueError("compressed metadata needs K to be a multiple of 8")
    g = mask.reshape(n, k // 4, 4)
    if not np.all(g.sum(axis=-1) == 2):
        raise ValueError("every group of 4 must keep exactly 2 elements")
    pos = np.nonzero(g)[-1].reshape(n, k // 4, 2)          # ascending per group
    i0, i1 = pos[..., 0], pos[..., 1]
    p = np.asarray(payload).reshape(n, k // 4, 4)
    vals = np.take_along_axis(p, pos, axis=-1).reshape(n, k // 2)
    nib = (i0 | (i1 << 2)).astype(np.uint8)                # [n, k/4]
    meta = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return vals, meta


def decompress24(values: np.ndarray, meta: np.ndarray, k: int, fill=0):
    """Scatter compressed values back to a dense [N, K] array (``fill`` elsewhere)."""
    values = np.asarray(values)
    meta = np.asarray(meta, dtype=np.uint8)
    n = values.shape[0]
    nib = np.empty((n, k // 4), dtype=np.int64)
    nib[:, 0::2] = meta & 0xF
    nib[:, 1::2] = meta >> 4
    i0 = nib & 3
    i1 = nib >> 2
    out = np.full((n, k // 4, 4), fill, dtype=values.dtype)
    v = values.reshape(n, k // 4, 2)
    np.put_along_axis(out, i0[..., None], v[..., 0:1], axis=-1)
    np.put_along_axis(out, i1[..., None], v[..., 1:2], axis=-1)
    return out.reshape(n, k)


def sp24_prune_compress(w_bits: np.ndarray, out_dtype: str = "e4m3"):
    """The weight path for 2:4: prune, then quantise (E4M3) or keep (bf16), then compress.

    Returns a dict with ``values``, ``meta``, ``mask``, ``scale`` (None for
    bf16) and ``pruned_dense`` (E4M3 codes with 0x00 at pruned positions, or
    the pruned bf16 bit patterns with 0x0000 there).

    Reading: pruning ranks the original bf16 magnitudes, before quantisation
    (pruning is the first step of the pipeline, quantisation the third).  The
    weight scale is taken from the whole tensor's amax, which equals the
    pruned tensor's amax because each group's largest element is kept.
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    mask = prune24_mask(w_bits)
    if out_dtype == "e4m3":
        s = scale_from_amax(amax(w_bits))
        codes = quantize_with_scale(w_bits, s)
        dense = np.where(mask, codes, np.uint8(0)).astype(np.uint8)
        vals, meta = compress24(mask, codes)
        return dict(values=vals.astype(np.uint8), meta=meta, mask=mask, scale=s,
                    pruned_dense=dense)
    if out_dtype == "bf16":
        dense = np.where(mask, w_bits, np.uint16(0)).astype(np.uint16)
        vals, meta = compress24(mask, w_bits)
        return dict(values=vals.astype(np.uint16), meta=meta, mask=mask, scale=None,
                    pruned_dense=dense)
    raise ValueError(out_dtype)


# ---------------------------------------------------------------------------
# The GEMM Y = X W^T (reference) and its error bound
# ---------------------------------------------------------------------------


def gemm_ref(x_vals: np.ndarray, w_vals: np.ndarray, sx=1.0, sw=1.0):
    """Y[m, n] = sx * sw * sum_k x[m, k] * w[n, k] in float64, and the bound
    B[m, n] = |sx * sw| * sum_k |x[m, k] * w[n, k]|.

    ``x_vals``/``w_vals`` are the decoded operand values (float64).  Every
    product of two E4M3 (or bf16) values is exact in float64 and the float64
    sums carry far less error than any tolerance used against it.
    """
    x = np.asarray(x_vals, dtype=np.float64)
    w = np.asarray(w_vals, dtype=np.float64)
    s = float(np.float64(sx) * np.float64(sw))
    y = s * (x @ w.T)
    b = abs(s) * (np.abs(x) @ np.abs(w).T)
    return y, b


def sparse_gemm_walk(x_vals: np.ndarray, values: np.ndarray, meta: np.ndarray,
                     sx=1.0, sw=1.0) -> np.ndarray:
    """Y from the compressed operand directly, in plain loops (tiny shapes only).

    For each output (m, n) and each group g, the two stored values multiply
    x[m, 4g + i0] and x[m, 4g + i1].  Used to pin the compressed format
    against the dense reference.
    """
    x = np.asarray(x_vals, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    m_, k = x.shape
    n_ = v.shape[0]
    y = np.zeros((m_, n_))
    for m in range(m_):
        for n in range(n_):
            acc = 0.0
            for g in range(k // 4):
                byte = int(meta[n, g // 2])
                nib = (byte >> (4 * (g % 2))) & 0xF
                i0, i1 = nib & 3, nib >> 2
                acc += v[n, 2 * g] * x[m, 4 * g + i0]
                acc += v[n, 2 * g + 1] * x[m, 4 * g + i1]
            y[m, n] = acc
    return float(np.float64(sx) * np.float64(sw)) * y


def within_tolerance(y_gpu: np.ndarray, y_ref: np.ndarray, bound: np.ndarray,
                     rel_bound: float = 1e-3, rel_val: float = 1e-2) -> np.ndarray:
    """Elementwise pass mask of |y - y_ref| <= 1e-3 * B + 1e-2 * |y_ref|."""
    y = np.asarray(y_gpu, dtype=np.float64)
    return np.abs(y - y_ref) <= rel_bound * bound + rel_val * np.abs(y_ref)


# ---------------------------------------------------------------------------
# General (2N-2):2N through 2:4 windows (the SlideSparse summary, §2
# Metodologia: N-1 overlapping windows of 4 with stride 2 per 2N-group,
# expansion (2N-2)/N; 6:8 is N = 4)
# ---------------------------------------------------------------------------


def slide_mask(bits: np.ndarray, n: int) -> np.ndarray:
    """(2n-2):2n magnitude mask: the 2n-2 largest |w| of each 2n along K survive
    (ties to the lower index)."""
    return keep_mask(bits, 2 * n, 2 * n - 2)


def slide_windows(kept: np.ndarray, n: int):
    """Assign the 2n-2 kept positions of one 2n-group to its n-1 windows (window
    j covers positions 2j .. 2j+3): for j = 0 .. n-2 in turn, window j takes the
    two lowest-index kept positions in its range that no earlier window took
    (the reading of the 6:8 case, for any n).  Returns n-1 pairs (p0, p1)."""
    kept = [int(p) for p in np.nonzero(np.asarray(kept, dtype=bool))[0]]
    if len(kept) != 2 * n - 2:
        raise ValueError("a (2n-2):2n group must keep exactly 2n-2 positions")
    taken, out = set(), []
    for j in range(n - 1):
        cand = [p for p in kept if 2 * j <= p <= 2 * j + 3 and p not in taken]
        if len(cand) < 2:
            raise AssertionError("window assignment failed")
        taken.update(cand[:2])
        out.append((cand[0], cand[1]))
    if taken != set(kept):
        raise AssertionError("window assignment lost a kept position")
    return out


def slide_decompose(w_bits: np.ndarray, n: int):
    """(2n-2):2n prune, window decomposition and 2:4 compression over
    K' = K (2n-2)/n, E4M3 with the per-tensor weight scale.  Window j of group
    g owns expanded columns 4((n-1)g + j) .. +3; the element at position p of
    the group sits at slot p - 2j.  Returns values [N, K'/2], meta [N, K'/8],
    the mask, the expanded mask and codes [N, K'], the scale and ``src``."""
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    rows_, k = w_bits.shape
    g2 = 2 * n
    if k % g2:
        raise ValueError("K must be a multiple of 2n")
    kp = k // g2 * 4 * (n - 1)
    mask = slide_mask(w_bits, n)
    emask = np.zeros((rows_, kp), dtype=bool)
    src = np.full((rows_, kp), -1, dtype=np.int64)
    for row in range(rows_):
        for g in range(k // g2):
            for j, (p0, p1) in enumerate(slide_windows(mask[row, g2 * g:g2 * g + g2], n)):
                for p in (p0, p1):
                    col = 4 * ((n - 1) * g + j) + (p - 2 * j)
                    emask[row, col] = True
                    src[row, col] = g2 * g + p
    s = scale_from_amax(amax(w_bits))
    codes = quantize_with_scale(w_bits, s)
    r = np.arange(rows_)[:, None]
    wexp = np.where(emask, codes[r, np.maximum(src, 0)], np.uint8(0)).astype(np.uint8)
    vals, meta = compress24(emask, wexp)
    return dict(values=vals, meta=meta, mask=mask, emask=emask, scale=s, expanded=wexp, src=src)


def slide_lift_columns(k: int, n: int) -> np.ndarray:
    """Source column of X for every lifted column:
    X'[:, 4((n-1)g + j) + r] = X[:, 2n g + 2j + r]."""
    g2 = 2 * n
    cols = np.empty(k // g2 * 4 * (n - 1), dtype=np.int64)
    for g in range(k // g2):
        for j in range(n - 1):
            for r in range(4):
                cols[4 * ((n - 1) * g + j) + r] = g2 * g + 2 * j + r
    return cols


def slide_lift(x_bits: np.ndarray, n: int):
    """Per-tensor E4M3 quantisation of X fused with the lift to K' = K (2n-2)/n:
    returns (lifted codes [M, K'], scale)."""
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    if x_bits.shape[1] % (2 * n):
        raise ValueError("K must be a multiple of 2n")
    codes, s = quantize_pertensor(x_bits)
    return codes[:, slide_lift_columns(x_bits.shape[1], n)], s


# ---------------------------------------------------------------------------
# Per-token activation scales and per-channel weight scales (the SlideSparse
# summary, §2 "Pipeline de Implementacion": its fused quantisation kernel
# scales each token; the roadmap, §Interaction avec la quantification:
# finer-grained scales for layers with outliers)
# ---------------------------------------------------------------------------


def quantize_pertoken(bits: np.ndarray):
    """Per-token dynamic E4M3 quantisation of X [M, K]: row m gets its own
    scale s_m = amax|X[m, :]| / 448 (1.0 for an all-zero row) and the codes
    E4M3(x / s_m).  Returns (codes uint8 [M, K], scales float32 [M]).

    Reading: the per-tensor rule (scale_from_amax, quantize_with_scale)
    applied to each row on its own.
    """
    bits = np.asarray(bits, dtype=np.uint16)
    codes = np.empty(bits.shape, dtype=np.uint8)
    scales = np.empty(bits.shape[0], dtype=np.float32)
    for m in range(bits.shape[0]):
        codes[m], scales[m] = quantize_pertensor(bits[m])
    return codes, scales


def sp24_prune_compress_perchannel(w_bits: np.ndarray):
    """2:4 prune + per-output-channel E4M3 quantisation + compress: the same
    selection and layout as sp24_prune_compress, with row n of W quantised by
    its own scale s_n = amax|W[n, :]| / 448 (the amax of the pruned row too:
    each group's largest element is kept).  Returns a dict with ``values``,
    ``meta``, ``mask``, ``scales`` (float32 [N]) and ``pruned_dense``.
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    mask = prune24_mask(w_bits)
    codes = np.empty(w_bits.shape, dtype=np.uint8)
    scales = np.empty(w_bits.shape[0], dtype=np.float32)
    for n in range(w_bits.shape[0]):
        scales[n] = scale_from_amax(amax(w_bits[n]))
        codes[n] = quantize_with_scale(w_bits[n], scales[n])
    dense = np.where(mask, codes, np.uint8(0)).astype(np.uint8)
    vals, meta = compress24(mask, codes)
    return dict(values=vals.astype(np.uint8), meta=meta, mask=mask, scales=scales,
                pruned_dense=dense)


def gemm_ref_scaled(x_vals: np.ndarray, w_vals: np.ndarray, sx: np.ndarray, sw: np.ndarray):
    """Y[m, n] = sx[m] * sw[n] * sum_k x[m, k] * w[n, k] in float64 and the
    bound B[m, n] = |sx[m] * sw[n]| * sum_k |x[m, k] * w[n, k]|; a scalar
    sx or sw is the same scale for every row or column."""
    x = np.asarray(x_vals, dtype=np.float64)
    w = np.asarray(w_vals, dtype=np.float64)
    a = np.broadcast_to(np.asarray(sx, dtype=np.float64).reshape(-1), (x.shape[0],))
    b = np.broadcast_to(np.asarray(sw, dtype=np.float64).reshape(-1), (w.shape[0],))
    s = a[:, None] * b[None, :]
    return s * (x @ w.T), np.abs(s) * (np.abs(x) @ np.abs(w).T)


# ---------------------------------------------------------------------------
# INT8 W8A8 with 2:4 weights (the cookbook, Comparison Tables: the "INT8 W8A8"
# recipe; the SlideSparse summary, §3 Contribuciones Clave: INT8 among the
# supported precisions, and §4: its end-to-end result measured in INT8)
# ---------------------------------------------------------------------------

INT8_MAX = 127


def int8_scale_from_amax(a: np.float32) -> np.float32:
    """Symmetric per-tensor INT8 scale s = amax / 127, one fp32 division; 1.0
    when amax is 0.

    Reading: the pages name the recipe but give no formula; the plainest one
    is the E4M3 rule with the INT8 grid: a symmetric range [-127, 127] (no
    zero point, -128 unused) and the largest magnitude mapped to 127.
    """
    a = np.float32(a)
    if a == 0:
        return np.float32(1.0)
    return np.float32(a / np.float32(INT8_MAX))


def int8_quantize_with_scale(bits: np.ndarray, s: np.float32) -> np.ndarray:
    """INT8 codes q = clamp(round_half_even(RN_fp32(x / s)), -127, 127).

    The quotient is one correctly rounded fp32 division, as for E4M3; it is
    then rounded to the nearest integer, ties to even.  The clamp only
    matters where the fp32 quotient of the largest element lands a rounding
    error above 127.
    """
    x = bf16_to_f32(bits)
    _require_finite(x, "int8 quantisation")
    v = (x / np.float32(s)).astype(np.float32)
    return np.clip(np.rint(v), -INT8_MAX, INT8_MAX).astype(np.int8)


def int8_quantize_pertensor(bits: np.ndarray):
    """Per-tensor dynamic INT8 quantisation: returns (codes int8, scale)."""
    s = int8_scale_from_amax(amax(bits))
    return int8_quantize_with_scale(bits, s), s


def sp24_prune_compress_int8(w_bits: np.ndarray):
    """The 2:4 weight path with INT8 codes: the same selection (ranking the
    bf16 magnitudes, ties to the lower index) and layout as
    sp24_prune_compress, each kept value stored as its INT8 code under the
    per-tensor scale.  Returns a dict with ``values`` (int8 [N, K/2]),
    ``meta``, ``mask``, ``scale`` and ``pruned_dense`` (int8, 0 where pruned).
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    mask = prune24_mask(w_bits)
    s = int8_scale_from_amax(amax(w_bits))
    codes = int8_quantize_with_scale(w_bits, s)
    dense = np.where(mask, codes, np.int8(0)).astype(np.int8)
    vals, meta = compress24(mask, codes)
    return dict(values=vals.astype(np.int8), meta=meta, mask=mask, scale=s, pruned_dense=dense)


def gemm_ref_int8(xq: np.ndarray, wq: np.ndarray, sx=1.0, sw=1.0):
    """INT8 GEMM: the exact integer sums acc[m, n] = sum_k xq[m, k] wq[n, k]
    (int64; every partial sum of the shapes used fits int32), then
    Y = sx * sw * acc in float64 and the bound B = |sx * sw| * sum_k
    |xq wq|.  ``wq`` is the dense [N, K] code array (0 at pruned positions).
    Returns (Y, B, acc).
    """
    x = np.asarray(xq, dtype=np.int64)
    w = np.asarray(wq, dtype=np.int64)
    acc = x @ w.T
    s = float(np.float64(sx) * np.float64(sw))
    return s * acc.astype(np.float64), abs(s) * (np.abs(x) @ np.abs(w).T).astype(np.float64), acc


# ---------------------------------------------------------------------------
# FP4 (E2M1) with 2:4 weights (the SlideSparse summary, §3 Contribuciones
# Clave: FP4 among the supported precisions)
# ---------------------------------------------------------------------------

E2M1_MAX = 6.0
# magnitude of code c (bits: sign 3, exponent 2-1, mantissa 0; bias 1;
# exponent 0 is subnormal: 0 and 0.5)
_E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """Values (float64) of FP4 E2M1 codes 0..15 (bit 3 is the sign)."""
    c = np.asarray(codes, dtype=np.uint8)
    mag = _E2M1_GRID[c & 7]
    return np.where(c & 8, -mag, mag)


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """FP4 E2M1 code of each fp32 value: round to the nearest grid value,
    ties to the even code (mantissa bit 0), saturate at +-6, and keep the sign
    of a value that rounds to zero (code 8 for negatives), as E4M3 does."""
    v = np.asarray(v, dtype=np.float32)
    _require_finite(v, "e2m1_encode")
    a = np.abs(v).astype(np.float64)
    d = np.abs(a[..., None] - _E2M1_GRID)           # distance to each magnitude
    best = d.min(axis=-1, keepdims=True)
    # candidates at the minimal distance: one, or two at a tie; take the even index
    cand = d == best
    idx = np.where(cand[..., ::2].any(axis=-1),
                   np.argmax(cand & (np.arange(8) % 2 == 0), axis=-1),
                   np.argmax(cand, axis=-1))
    idx = np.where(a > E2M1_MAX, 7, idx)
    sign = np.signbit(v)
    return (idx + np.where(sign, 8, 0)).astype(np.uint8)


def fp4_scale_from_amax(a: np.float32) -> np.float32:
    """Per-tensor FP4 scale s = amax / 6 (one fp32 division); 1.0 when amax is 0.

    Reading: the pages list FP4 without a format; the plainest one in keeping
    with the per-tensor E4M3 and INT8 rules is the same rule on the E2M1 grid
    (largest magnitude 6), with no block scales.
    """
    a = np.float32(a)
    if a == 0:
        return np.float32(1.0)
    return np.float32(a / np.float32(E2M1_MAX))


def fp4_quantize_with_scale(bits: np.ndarray, s: np.float32) -> np.ndarray:
    """E2M1 codes of x / s, the quotient one correctly rounded fp32 division."""
    x = bf16_to_f32(bits)
    return e2m1_encode((x / np.float32(s)).astype(np.float32))


def fp4_quantize_pertensor(bits: np.ndarray):
    """Per-tensor dynamic FP4 quantisation: returns (codes uint8 0..15, scale)."""
    s = fp4_scale_from_amax(amax(bits))
    return fp4_quantize_with_scale(bits, s), s


def sp24_prune_compress_fp4(w_bits: np.ndarray):
    """The 2:4 weight path with FP4 codes: the selection and layout of
    sp24_prune_compress, each kept value stored as its E2M1 code (one code per
    entry of values [N, K/2]; how codes are packed into bytes is a storage
    matter for the kernels) under the per-tensor FP4 scale.  Returns a dict
    with ``values``, ``meta``, ``mask``, ``scale`` and ``pruned_dense`` (codes,
    0 where pruned)."""
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    mask = prune24_mask(w_bits)
    s = fp4_scale_from_amax(amax(w_bits))
    codes = fp4_quantize_with_scale(w_bits, s)
    dense = np.where(mask, codes, np.uint8(0)).astype(np.uint8)
    vals, meta = compress24(mask, codes)
    return dict(values=vals.astype(np.uint8), meta=meta, mask=mask, scale=s, pruned_dense=dense)


# ---------------------------------------------------------------------------
# 6:8 sliding-window decomposition and activation lifting (the SlideSparse
# summary, §2 Metodologia)
# ---------------------------------------------------------------------------


def prune68_mask(bits: np.ndarray) -> np.ndarray:
    """6:8 magnitude mask: the six largest |w| of each 8 along K survive
    (ties to the lower index, as for 2:4)."""
    return keep_mask(bits, 8, 6)


def window_assignment(kept: np.ndarray):
    """Assign the 6 kept positions of one 8-group to the 3 stride-2 windows.

    Window j covers positions 2j .. 2j+3.  Reading of "the extras spill into
    the next overlapping window": for j = 0, 1, 2 in turn, window j takes the
    two lowest-index kept positions in its range that no earlier window took.
    Returns a list of three (p0, p1) pairs, p0 < p1.
    """
    kept = [int(p) for p in np.nonzero(np.asarray(kept, dtype=bool))[0]]
    if len(kept) != 6:
        raise ValueError("a 6:8 group must keep exactly 6 positions")
    taken = set()
    out = []
    for j in range(3):
        cand = [p for p in kept if 2 * j <= p <= 2 * j + 3 and p not in taken]
        if len(cand) < 2:
            raise AssertionError("window assignment failed")  # impossible, see tests
        pick = cand[:2]
        taken.update(pick)
        out.append((pick[0], pick[1]))
    if taken != set(kept):
        raise AssertionError("window assignment lost a kept position")
    return out


def slide68_expand_mask_and_map(mask68: np.ndarray):
    """For a 6:8 mask [N, K], build the expanded 2:4 mask [N, 1.5K] and the
    source column of every kept expanded slot (-1 where the slot is empty).

    Expanded column of window j, slot r of group g is 12g + 4j + r; the
    element placed there is W[n, 8g + 2j + r].
    """
    n, k = mask68.shape
    kp = k * 3 // 2
    emask = np.zeros((n, kp), dtype=bool)
    src = np.full((n, kp), -1, dtype=np.int64)
    for row in range(n):
        for g in range(k // 8):
            pairs = window_assignment(mask68[row, 8 * g:8 * g + 8])
            for j, (p0, p1) in enumerate(pairs):
                for p in (p0, p1):
                    col = 12 * g + 4 * j + (p - 2 * j)
                    emask[row, col] = True
                    src[row, col] = 8 * g + p
    return emask, src


def slide68_decompose(w_bits: np.ndarray, out_dtype: str = "e4m3"):
    """6:8 prune, window decomposition and 2:4 compression over K' = 1.5K.

    Returns values [N, 3K/4], meta [N, 3K/16], the 6:8 mask, the expanded
    mask [N, 1.5K], the scale (E4M3; None for bf16) and the expanded dense
    operand W' [N, 1.5K] (codes or bf16 bits, zero in empty slots).
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    n, k = w_bits.shape
    if k % 8:
        raise ValueError("6:8 needs K to be a multiple of 8")
    m68 = prune68_mask(w_bits)
    emask, src = slide68_expand_mask_and_map(m68)
    if out_dtype == "e4m3":
        s = scale_from_amax(amax(w_bits))
        payload = quantize_with_scale(w_bits, s)
        zero = np.uint8(0)
    elif out_dtype == "bf16":
        s = None
        payload = w_bits
        zero = np.uint16(0)
    else:
        raise ValueError(out_dtype)
    rows = np.arange(n)[:, None]
    wexp = np.where(emask, payload[rows, np.maximum(src, 0)], zero).astype(payload.dtype)
    vals, meta = compress24(emask, wexp)
    return dict(values=vals, meta=meta, mask68=m68, emask=emask, scale=s,
                expanded=wexp, src=src)


def lift_columns(k: int) -> np.ndarray:
    """Source column of X for every lifted column: X'[:, 12g+4j+r] = X[:, 8g+2j+r]."""
    cols = np.empty(k * 3 // 2, dtype=np.int64)
    for g in range(k // 8):
        for j in range(3):
            for r in range(4):
                cols[12 * g + 4 * j + r] = 8 * g + 2 * j + r
    return cols


def slide68_lift(x_bits: np.ndarray):
    """Per-tensor E4M3 quantisation of X fused with the lift to K' = 1.5K.

    The scale is that of X itself (X' holds the same values, so the same
    amax).  Returns (lifted codes [M, 1.5K], scale).
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    k = x_bits.shape[1]
    if k % 8:
        raise ValueError("6:8 lifting needs K to be a multiple of 8")
    codes, s = quantize_pertensor(x_bits)
    return codes[:, lift_columns(k)], s
