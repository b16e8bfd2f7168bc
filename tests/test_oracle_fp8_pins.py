"""Pins of the oracle's FP8 (E4M3) expert-weight path against things other than itself.

The reading pinned here: E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
infinities, largest finite 448), round to nearest even, saturating to +-448; one FP32 scale per
row, s = fl32(amax / 448) and q = e4m3(fl32(x / s)); an FP8 linear layer sums exact products
of decoded codes and applies the two row scales before one rounding to FP32.  The pages name
FP8 and NVFP4 checkpoints (news article "Reflection lança o Beam", section "Onde o Beam
economiza ..."; review page "обзор модели «Бим»") but no scale format.

Independent references: torch's float8_e4m3fn conversions (a library routine), the oracle's
own BF16 router-logit and expert functions (pinned in test_oracle_pins) on inputs that the
quantisation represents exactly, and invariants of the scales.
"""
import numpy as np
import pytest
import torch

import oracle


def _torch_codes(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def _positive_values() -> np.ndarray:
    """Decoded values of the finite non-negative codes 0x00 .. 0x7e, ascending."""
    return oracle.e4m3_to_f32(np.arange(0x7f, dtype=np.uint8)).astype(np.float64)


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f32(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert ours[0x7e] == 448.0 and ours[0x08] == 2.0 ** -6 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_matches_torch_in_range_and_on_ties():
    rng = np.random.default_rng(11)
    vals = [rng.normal(0, sc, 20000) for sc in (1e-3, 3e-2, 0.5, 4.0, 60.0, 300.0)]
    x = np.clip(np.concatenate(vals), -448, 448).astype(np.float32)
    v = _positive_values()
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)  # exact in FP32: ties between codes
    x = np.concatenate([x, v.astype(np.float32), mids, -mids, np.float32([0.0, -0.0])])
    ours = oracle.f32_to_e4m3(x)
    ref = _torch_codes(x)
    bad = np.flatnonzero(ours != ref)
    assert bad.size == 0, (x[bad[:5]], ours[bad[:5]], ref[bad[:5]])
    # ties go to the even code
    mid_codes = oracle.f32_to_e4m3(mids)
    assert np.all(mid_codes % 2 == 0)


def test_e4m3_saturates_and_keeps_nan():
    x = np.float32([448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3e38, -500.0, np.inf, -np.inf, np.nan])
    c = oracle.f32_to_e4m3(x)
    assert list(c[:7]) == [0x7e] * 7
    assert c[7] == 0xfe and c[8] == 0x7e and c[9] == 0xfe and c[10] == 0x7f


def test_quantize_rows_matches_torch_conversion_and_error_bounds():
    rng = np.random.default_rng(5)
    x = torch.from_numpy(rng.normal(0, 1, (64, 320)).astype(np.float32))
    x[3] *= 1e-4          # small magnitudes
    x[4, :] = 0.0         # an all-zero row
    x[5, 17] = 50.0       # one outlier
    xb = x.to(torch.bfloat16)
    q, s = oracle.quantize_rows_e4m3(xb)
    xf = xb.float()
    amax = xf.abs().amax(dim=1)
    s_ref = (amax / 448.0).numpy()
    assert np.array_equal(s, s_ref)
    nz = s_ref > 0
    q_ref = _torch_codes((xf[nz] / torch.from_numpy(s_ref[nz])[:, None]).numpy())
    assert np.array_equal(q[nz], q_ref)
    assert np.all(q[4] == 0) and s[4] == 0.0
    # the largest magnitude of every non-zero row becomes +-448
    big = xf.abs().argmax(dim=1).numpy()
    assert np.all(np.isin(q[np.arange(64)[nz], big[nz]], [0x7e, 0xfe]))
    # dequantisation error: at most half the code spacing, 2^-4 |x| in the normal range and
    # 2^-10 s among the subnormals
    xv = xf.numpy().astype(np.float64)
    dq = oracle.e4m3_to_f32(q).astype(np.float64) * s[:, None]
    bound = np.maximum(np.abs(xv) * 2.0 ** -4, s[:, None].astype(np.float64) * 2.0 ** -10)
    assert np.all(np.abs(dq - xv) <= bound)


def _exact_rows(rng, rows, cols, spread, center=0):
    """BF16 rows that E4M3 row quantisation represents exactly: random codes times 2^k
    (|k - center| <= spread), each row holding one +-448 * 2^k so that its scale is 2^k."""
    codes = rng.integers(0, 0x7f, (rows, cols)).astype(np.uint8)
    codes |= (rng.integers(0, 2, (rows, cols)) << 7).astype(np.uint8)
    codes[:, 0] = 0x7e
    k = rng.integers(center - spread, center + spread + 1, rows)
    vals = oracle.e4m3_to_f32(codes).astype(np.float64) * (2.0 ** k)[:, None]
    xb = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(xb.float().numpy().astype(np.float64), vals)  # exact in BF16
    return xb, codes, (2.0 ** k).astype(np.float32)


def test_quantize_rows_is_exact_on_representable_rows():
    rng = np.random.default_rng(2)
    xb, codes, scale = _exact_rows(rng, 40, 96, 6)
    q, s = oracle.quantize_rows_e4m3(xb)
    assert np.array_equal(s, scale)
    # -0.0 and +0.0 both decode to zero; compare the decoded values
    assert np.array_equal(oracle.e4m3_to_f32(q), oracle.e4m3_to_f32(codes))


def test_linear_fp8_equals_router_logits_on_exact_operands():
    """With power-of-two scales every operand is exact in BF16 / FP32, so the FP8 linear layer
    must equal the FP32-weight dot product of the router-logit function, bit for bit."""
    rng = np.random.default_rng(3)
    xb, xq, sx = _exact_rows(rng, 24, 128, 4)
    wb, wq, sw = _exact_rows(rng, 40, 128, 8)
    y = oracle.linear_fp8(xq, sx, wq, sw)
    ref = oracle.router_logits(xb, wb.float())
    assert np.array_equal(y, ref)


def test_linear_fp8_general_scales_match_float64():
    rng = np.random.default_rng(4)
    xq = rng.integers(0, 0xff, (16, 256)).astype(np.uint8)
    xq[(xq & 0x7f) == 0x7f] = 0x00  # no NaN codes
    wq = rng.integers(0, 0xff, (48, 256)).astype(np.uint8)
    wq[(wq & 0x7f) == 0x7f] = 0x01
    sx = rng.uniform(0.01, 2.0, 16).astype(np.float32)
    sw = rng.uniform(0.001, 0.1, 48).astype(np.float32)
    y = oracle.linear_fp8(xq, sx, wq, sw)
    X = oracle.e4m3_to_f32(xq).astype(np.float64)
    Wv = oracle.e4m3_to_f32(wq).astype(np.float64)
    ref = (X @ Wv.T) * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    np.testing.assert_allclose(y, ref.astype(np.float32), rtol=2 ** -23, atol=0)


def _fp8_expert(rng, d, I, spread, center=-10):
    """An expert whose weights E4M3 represents exactly (scales near 2^-10, so weights of the
    size the Beam shapes use)."""
    gb, gq, sg = _exact_rows(rng, I, d, spread, center)
    ub, uq, su = _exact_rows(rng, I, d, spread, center)
    db, dq, sd = _exact_rows(rng, d, I, spread, center)
    return (gb, ub, db), (gq, sg, uq, su, dq, sd)


def test_expert_mlp_fp8_gate_up_equal_bf16_expert_on_exact_operands():
    """Exactly representable input row and weights: the FP8 expert's SwiGLU activation must be
    the BF16 expert's, bit for bit (both are exact dot products rounded once)."""
    rng = np.random.default_rng(6)
    d, I = 128, 64
    bf, fp8 = _fp8_expert(rng, d, I, 3)
    x, _, _ = _exact_rows(rng, 1, d, 2, -8)
    _, a_bf16 = oracle.expert_mlp(x[0], *bf, return_act=True)
    _, a_fp8 = oracle.expert_mlp_fp8(x[0], *fp8, return_act=True)
    assert np.array_equal(a_fp8, a_bf16)


def test_expert_mlp_fp8_down_scales_are_per_output_row():
    rng = np.random.default_rng(7)
    d, I = 128, 64
    _, (gq, sg, uq, su, dq, sd) = _fp8_expert(rng, d, I, 3)
    x, _, _ = _exact_rows(rng, 1, d, 2, -8)
    y = oracle.expert_mlp_fp8(x[0], gq, sg, uq, su, dq, sd)
    # doubling the scale of output row c doubles y_c exactly and leaves the rest
    sd2 = sd.copy()
    sd2[5] *= 2
    y2 = oracle.expert_mlp_fp8(x[0], gq, sg, uq, su, dq, sd2)
    assert y2[5] == 2 * y[5] and np.array_equal(np.delete(y2, 5), np.delete(y, 5))
    # permuting the down projection's output rows permutes y
    perm = rng.permutation(d)
    y3 = oracle.expert_mlp_fp8(x[0], gq, sg, uq, su, dq[perm], sd[perm])
    assert np.array_equal(y3, y[perm])
    # the activation feeding the down projection is quantised: y differs from the
    # unquantised down projection by at most the E4M3 step of the activation (|rel| <= 2^-4)
    _, a = oracle.expert_mlp_fp8(x[0], gq, sg, uq, su, dq, sd, return_act=True)
    av = oracle.bf16_to_f32(a).astype(np.float64)
    full = (oracle.e4m3_to_f32(dq).astype(np.float64) * sd[:, None]) @ av
    scale = (np.abs(oracle.e4m3_to_f32(dq).astype(np.float64) * sd[:, None]) @ np.abs(av))
    assert np.all(np.abs(y - full) <= 2.0 ** -4 * scale + 1e-30)
    assert not np.array_equal(y.astype(np.float64), full.astype(np.float32).astype(np.float64))


def test_moe_tokens_fp8_is_weighted_sum_of_fp8_experts():
    rng = np.random.default_rng(8)
    d, I, E, k, T = 128, 64, 4, 2, 5
    experts = {e: _fp8_expert(rng, d, I, 3)[1] for e in range(E)}
    h = torch.from_numpy(rng.normal(0, 1, (T, d)).astype(np.float32)).to(torch.bfloat16)
    idx = np.array([[0, 1], [1, 3], [0, 2], [2, 3], [1, 2]], np.int32)
    w = rng.uniform(0.5, 2.0, (T, k)).astype(np.float32)
    out = oracle.moe_tokens_fp8(np.arange(T), h, idx, w, experts)
    for t in range(T):
        ys = [oracle.expert_mlp_fp8(h[t], *experts[e]).astype(np.float64) for e in idx[t]]
        ref = sum(float(w[t, j]) * ys[j] for j in range(k))
        assert np.array_equal(out[t], ref.astype(np.float32))
