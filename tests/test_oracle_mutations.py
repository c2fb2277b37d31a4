"""Planted mistakes in the oracle (CPU only) must fail its pins: evidence
that the pins of the INT8, FP4 and general sliding-window functions pin them.
Each case replaces one oracle function by a plausibly wrong version for the
duration of the test and runs the pin that should catch it."""
import numpy as np
import pytest

import test_oracle_pins as P
from oracle import sp24_oracle as O


def _fails(pin):
    with pytest.raises(AssertionError):
        pin()


def test_int8_ties_away_from_zero_is_caught(monkeypatch):
    def wrong(bits, s):
        v = (O.bf16_to_f32(bits) / np.float32(s)).astype(np.float32)
        q = np.sign(v) * np.floor(np.abs(v) + np.float32(0.5))
        return np.clip(q, -127, 127).astype(np.int8)
    monkeypatch.setattr(O, "int8_quantize_with_scale", wrong)
    _fails(P.test_int8_golden_hand_example)   # the half-step bound alone cannot see a tie's direction


def test_int8_scale_of_128_is_caught(monkeypatch):
    monkeypatch.setattr(O, "int8_scale_from_amax", lambda a: np.float32(np.float32(a) / np.float32(128)) if a else np.float32(1))
    _fails(P.test_int8_golden_hand_example)


def test_fp4_ties_away_from_zero_is_caught(monkeypatch):
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])

    def wrong(v):
        v = np.asarray(v, dtype=np.float32)
        a = np.abs(v).astype(np.float64)
        d = np.abs(a[..., None] - grid)
        idx = 7 - np.argmin(d[..., ::-1], axis=-1)     # ties to the larger magnitude
        idx = np.where(a > 6, 7, idx)
        return (idx + np.where(np.signbit(v), 8, 0)).astype(np.uint8)
    monkeypatch.setattr(O, "e2m1_encode", wrong)
    _fails(P.test_e2m1_encode_every_bf16_value_matches_ml_dtypes)
    _fails(P.test_fp4_golden_hand_example)


def test_slide_windows_from_the_right_are_caught(monkeypatch):
    def wrong(kept, n):
        kept = [int(p) for p in np.nonzero(np.asarray(kept, dtype=bool))[0]]
        taken, out = set(), []
        for j in range(n - 1):
            cand = [p for p in kept if 2 * j <= p <= 2 * j + 3 and p not in taken]
            pick = cand[-2:] if len(cand) >= 2 else cand
            taken.update(pick)
            out.append(tuple(pick))
        return out
    monkeypatch.setattr(O, "slide_windows", wrong)
    _fails(P.test_general_slide_golden_hand_examples)


def test_gemm_ref_int8_dropping_a_scale_is_caught(monkeypatch):
    real = O.gemm_ref_int8
    monkeypatch.setattr(O, "gemm_ref_int8", lambda xq, wq, sx=1.0, sw=1.0: real(xq, wq, sx, 1.0))
    _fails(P.test_int8_gemm_is_the_exact_integer_product)


# ------------------------------------------------------------ the core path's functions

def test_e4m3_decode_with_bias_8_is_caught(monkeypatch):
    real = O.e4m3_decode
    monkeypatch.setattr(O, "e4m3_decode", lambda codes: real(codes) / 2.0)
    _fails(P.test_e4m3_decode_all_codes_match_ml_dtypes)


def test_e4m3_truncation_instead_of_rounding_is_caught(monkeypatch):
    real_enc, real_dec = O.e4m3_encode, O.e4m3_decode

    def wrong(v):
        c = real_enc(v)
        up = np.abs(real_dec(c)) > np.abs(np.asarray(v, dtype=np.float64))
        return np.where(up & ((c & 0x7F) > 0), c - 1, c).astype(np.uint8)
    monkeypatch.setattr(O, "e4m3_encode", wrong)
    _fails(P.test_e4m3_encode_every_bf16_value_in_range)


def test_prune_ties_to_the_higher_index_are_caught(monkeypatch):
    def wrong(bits, group, keep):
        w = O.bf16_to_f32(bits)
        a = np.abs(w).reshape(*w.shape[:-1], w.shape[-1] // group, group).astype(np.float64)
        idx = np.arange(group)
        ai, aj = a[..., :, None], a[..., None, :]
        beats = (aj > ai) | ((aj == ai) & (idx[None, :] > idx[:, None]))
        return (beats.sum(axis=-1) < keep).reshape(w.shape)
    monkeypatch.setattr(O, "keep_mask", wrong)
    _fails(P.test_prune24_exhaustive_over_tie_alphabet)
    _fails(P.test_prune24_golden_hand_example)


def test_swapped_metadata_nibble_order_is_caught(monkeypatch):
    real = O.compress24

    def wrong(mask, payload):
        vals, meta = real(mask, payload)
        return vals, ((meta & 0x0F) << 4 | (meta >> 4)).astype(np.uint8)
    monkeypatch.setattr(O, "compress24", wrong)
    _fails(P.test_prune24_golden_hand_example)


def test_68_windows_from_the_right_are_caught(monkeypatch):
    def wrong(kept):
        kept = [int(p) for p in np.nonzero(np.asarray(kept, dtype=bool))[0]]
        taken, out = set(), []
        for j in range(3):
            cand = [p for p in kept if 2 * j <= p <= 2 * j + 3 and p not in taken][-2:]
            taken.update(cand)
            out.append(tuple(cand))
        return out
    monkeypatch.setattr(O, "window_assignment", wrong)
    _fails(P.test_slide68_golden_hand_example)


def test_e4m3_scale_with_the_wrong_maximum_is_caught(monkeypatch):
    monkeypatch.setattr(O, "scale_from_amax",
                        lambda a: np.float32(np.float32(a) / np.float32(240.0)) if a else np.float32(1.0))
    _fails(P.test_scale_closed_form_and_zero_tensor)


def test_pertoken_with_the_tensor_scale_is_caught(monkeypatch):
    def wrong(bits):
        codes, s = O.quantize_pertensor(bits)
        return codes, np.full(bits.shape[0], s, dtype=np.float32)
    monkeypatch.setattr(O, "quantize_pertoken", wrong)
    _fails(P.test_pertoken_scales_follow_row_magnitude_exactly)


def test_gemm_dropping_the_last_k_column_is_caught(monkeypatch):
    real = O.gemm_ref

    def wrong(x_vals, w_vals, sx=1.0, sw=1.0):
        x = np.array(x_vals, dtype=np.float64)
        x[:, -1] = 0.0
        return real(x, w_vals, sx, sw)
    monkeypatch.setattr(O, "gemm_ref", wrong)
    _fails(lambda: P.test_sparse_walk_equals_dense_reference("normal"))


def test_perchannel_with_the_tensor_scale_is_caught(monkeypatch):
    def wrong(w_bits):
        r = O.sp24_prune_compress(w_bits, "e4m3")
        return dict(values=r["values"], meta=r["meta"], mask=r["mask"],
                    scales=np.full(w_bits.shape[0], r["scale"], dtype=np.float32), pruned_dense=r["pruned_dense"])
    monkeypatch.setattr(O, "sp24_prune_compress_perchannel", wrong)
    _fails(P.test_perchannel_prune_selects_like_per_tensor_and_scales_each_row)


def test_general_lift_off_by_one_window_is_caught(monkeypatch):
    def wrong(k, n):   # windows at stride 1 instead of 2
        g2 = 2 * n
        cols = np.empty(k // g2 * 4 * (n - 1), dtype=np.int64)
        for g in range(k // g2):
            for j in range(n - 1):
                for r in range(4):
                    cols[4 * ((n - 1) * g + j) + r] = g2 * g + j + r
        return cols
    monkeypatch.setattr(O, "slide_lift_columns", wrong)
    _fails(P.test_general_slide_golden_hand_examples)


def test_bf16_truncation_is_caught(monkeypatch):
    def wrong(x):
        u = np.asarray(x, dtype=np.float32).view(np.uint32)
        return (u >> np.uint32(16)).astype(np.uint16)      # chops instead of rounding
    monkeypatch.setattr(O, "f32_to_bf16_rne", wrong)
    _fails(P.test_f32_to_bf16_rne_matches_library_casts)


def test_bf16_ties_away_from_zero_is_caught(monkeypatch):
    def wrong(x):
        u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
        return ((u + np.uint64(0x8000)) >> np.uint64(16)).astype(np.uint16)
    monkeypatch.setattr(O, "f32_to_bf16_rne", wrong)
    _fails(P.test_f32_to_bf16_rne_matches_library_casts)
