"""Pins of the oracle's NVFP4 expert-weight path against things other than itself.

The reading pinned here:
- Codes are E2M1: 1 sign bit, 2 exponent bits with bias 1 and 1 mantissa bit, giving the
  magnitudes 0, 0.5, 1, 1.5, 2, 3, 4 and 6, with no infinities and no NaN.
- Rounding is to the nearest value, ties to the even code, saturating to +-6.
- Each block of 16 consecutive elements of a row has an E4M3 scale, and each row an FP32
  scale:
    s = fl32(amax / 2688)
    bs = e4m3(fl32(fl32(m_b / s) / 6))
    q = e2m1(fl32(x / fl32(s * bs)))
- A linear layer sums the exact products of codes and block scales, then applies the two row
  scales before one rounding to FP32.

The pages name NVFP4 checkpoints but give no scale format (news article "Reflection lança o
Beam", section "Onde o Beam economiza ..."; review page "обзор модели «Бим»").

Independent references:
- the E2M1 value table of the OCP microscaling formats, written out;
- nearest-value search by brute force;
- rows that the format represents exactly, built from chosen codes and scales;
- a float64 matmul of decoded operands;
- the oracle's BF16 router-logit and expert functions (pinned in test_oracle_pins), on
  operands that NVFP4 represents exactly.
"""
import numpy as np
import torch

import oracle

# E2M1 magnitudes of codes 0..7 (OCP Microscaling Formats v1.0, FP4 E2M1 table)
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _brute_force_code(v: float) -> int:
    a = abs(v)
    if a >= 6.0:  # saturation (far above 6 every distance rounds to the same double)
        return 7 | (8 if np.signbit(v) else 0)
    dist = [abs(a - m) for m in E2M1_TABLE]
    best = min(dist)
    ties = [c for c in range(8) if dist[c] == best]
    code = ties[0] if len(ties) == 1 else next(c for c in ties if c % 2 == 0)
    return code | (8 if np.signbit(v) else 0)


def test_e2m1_decode_matches_the_format_table():
    vals = oracle.e2m1_to_f32(np.arange(16, dtype=np.uint8))
    assert list(vals[:8]) == E2M1_TABLE
    assert list(vals[8:]) == [-m for m in E2M1_TABLE]
    assert np.signbit(vals[8])  # code 8 is -0


def test_e2m1_encode_is_nearest_with_ties_to_even_and_saturates():
    rng = np.random.default_rng(21)
    mids = [(a + b) / 2 for a, b in zip(E2M1_TABLE[:-1], E2M1_TABLE[1:])]
    x = np.concatenate([rng.uniform(-7.5, 7.5, 20000), np.array(E2M1_TABLE), np.array(mids),
                        -np.array(mids), [6.5, 7.0, 100.0, -1e30, 1e-30, 0.0, -0.0]])
    x = x.astype(np.float32)
    ours = oracle.f32_to_e2m1(x)
    ref = np.array([_brute_force_code(float(v)) for v in x], np.uint8)
    bad = np.flatnonzero(ours != ref)
    assert bad.size == 0, (x[bad[:5]], ours[bad[:5]], ref[bad[:5]])
    # the hand cases: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    hand = oracle.e2m1_to_f32(oracle.f32_to_e2m1(np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])))
    assert list(hand) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]


def _exact_rows(rng, rows, cols, spread, center=0):
    """BF16 rows that NVFP4 represents exactly, with their codes, block scales and row scales.

    The row scale is 2^k (|k - center| <= spread): one block holds a +-6 with block scale 448,
    so amax = 2688 * 2^k.  Every block holds one +-6 and a normal E4M3 block scale, so its
    scale comes back exactly, and every element is a code value times that scale times 2^k."""
    assert cols % 16 == 0
    nb = cols // 16
    codes = rng.integers(0, 16, (rows, cols)).astype(np.uint8)
    first = np.arange(nb) * 16
    codes[:, first] = np.where(rng.integers(0, 2, (rows, nb)) == 1, 0x7, 0xF)
    # normal E4M3 codes 0x20..0x5f (2^-3 .. 2^4 range): exact products with the codes
    bs = rng.integers(0x20, 0x60, (rows, nb)).astype(np.uint8)
    bs[:, 0] = 0x7E  # 448: this block carries the row maximum
    k = rng.integers(center - spread, center + spread + 1, rows)
    vals = (oracle.e2m1_to_f32(codes).astype(np.float64)
            * np.repeat(oracle.e4m3_to_f32(bs).astype(np.float64), 16, axis=1)
            * (2.0 ** k)[:, None])
    xb = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(xb.float().numpy().astype(np.float64), vals)  # exact in BF16
    return xb, codes, bs, (2.0 ** k).astype(np.float32)


def test_quantize_rows_nvfp4_is_exact_on_representable_rows():
    rng = np.random.default_rng(22)
    xb, codes, bs, scale = _exact_rows(rng, 32, 256, 5)
    q, b, s = oracle.quantize_rows_nvfp4(xb)
    assert np.array_equal(s, scale)
    assert np.array_equal(b, bs)
    # -0 and +0 both decode to zero: compare decoded values
    assert np.array_equal(oracle.e2m1_to_f32(q), oracle.e2m1_to_f32(codes))


def _halfgap(v):
    a = np.abs(v)
    return np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0))


def test_quantize_rows_nvfp4_error_bounds_and_block_maxima():
    rng = np.random.default_rng(23)
    x = torch.from_numpy(rng.normal(0, 1, (48, 320)).astype(np.float32))
    x[3] *= 1e-4          # small magnitudes
    x[4, :] = 0.0         # an all-zero row
    x[5, 17] = 80.0       # one outlier: its neighbours' blocks get small scales
    x[6, 32:48] = 0.0     # an all-zero block
    xb = x.to(torch.bfloat16)
    q, bs, s = oracle.quantize_rows_nvfp4(xb)
    xv = xb.float().numpy().astype(np.float64)
    assert s[4] == 0.0 and np.all(q[4] == 0) and np.all(bs[4] == 0)
    assert np.all(bs[6, 2] == 0) and np.all(q[6, 32:48] == 0)
    bsv = oracle.e4m3_to_f32(bs).astype(np.float64)
    den = np.repeat(bsv * s[:, None].astype(np.float64), 16, axis=1)
    dq = oracle.e2m1_to_f32(q).astype(np.float64) * den
    nz = den > 0
    v = np.where(nz, xv / np.where(nz, den, 1.0), 0.0)
    # each element within half the code spacing of its value; the block maximum may exceed 6
    # by the E4M3 rounding of its block scale (at most 2^-4 relative).  The value is formed in
    # FP32 (two roundings: s * bs and x / that), which may move a near-tie onto the tie.
    bound = np.maximum(_halfgap(v), np.abs(v) - 6.0) * den + np.abs(xv) * 2.0 ** -21
    assert np.all(np.abs(dq - xv)[nz] <= bound[nz] + 1e-30)
    assert np.all(np.abs(v[nz]) <= 6.0 / (1 - 2.0 ** -4))
    # blocks with a normal, unsaturated scale put their largest element on +-6
    rows, nb = bs.shape
    mag = np.abs(oracle.e2m1_to_f32(q)).reshape(rows, nb, 16).max(axis=2)
    normal = (bsv >= 2.0 ** -6) & (bsv < 448.0)
    assert normal.sum() > 800
    assert np.all(mag[normal] == 6.0)


def _random_nvfp4(rng, rows, K):
    q = rng.integers(0, 16, (rows, K)).astype(np.uint8)
    bs = rng.integers(0x01, 0x7F, (rows, K // 16)).astype(np.uint8)  # finite, non-NaN
    return q, bs


def test_linear_nvfp4_matches_float64_on_decoded_operands():
    rng = np.random.default_rng(24)
    K = 256
    xq, xbs = _random_nvfp4(rng, 12, K)
    wq, wbs = _random_nvfp4(rng, 40, K)
    sx = rng.uniform(0.01, 2.0, 12).astype(np.float32)
    sw = rng.uniform(0.001, 0.1, 40).astype(np.float32)
    y = oracle.linear_nvfp4(xq, xbs, sx, wq, wbs, sw)
    table = np.array(E2M1_TABLE + [-m for m in E2M1_TABLE])
    X = table[xq] * np.repeat(oracle.e4m3_to_f32(xbs).astype(np.float64), 16, axis=1)
    Wv = table[wq] * np.repeat(oracle.e4m3_to_f32(wbs).astype(np.float64), 16, axis=1)
    ref = (X @ Wv.T) * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    np.testing.assert_allclose(y, ref.astype(np.float32), rtol=2 ** -23, atol=0)


def test_linear_nvfp4_equals_router_logits_on_exact_operands():
    """On rows that NVFP4 represents exactly every product and partial sum is exact in double,
    so the NVFP4 linear layer must equal the FP32-weight dot product of the router-logit
    function, bit for bit."""
    rng = np.random.default_rng(25)
    xb, xq, xbs, sx = _exact_rows(rng, 16, 256, 3)
    wb, wq, wbs, sw = _exact_rows(rng, 24, 256, 4)
    y = oracle.linear_nvfp4(xq, xbs, sx, wq, wbs, sw)
    ref = oracle.router_logits(xb, wb.float())
    assert np.array_equal(y, ref)


def _nvfp4_expert(rng, d, I, spread, center=-12):
    gb, gq, gbs, sg = _exact_rows(rng, I, d, spread, center)
    ub, uq, ubs, su = _exact_rows(rng, I, d, spread, center)
    db, dq, dbs, sd = _exact_rows(rng, d, I, spread, center)
    return (gb, ub, db), ((gq, gbs, sg), (uq, ubs, su), (dq, dbs, sd))


def test_expert_mlp_nvfp4_gate_up_equal_bf16_expert_on_exact_operands():
    rng = np.random.default_rng(26)
    d, I = 256, 64
    bf, fp4 = _nvfp4_expert(rng, d, I, 2)
    x, _, _, _ = _exact_rows(rng, 1, d, 1, -6)
    _, a_bf16 = oracle.expert_mlp(x[0], *bf, return_act=True)
    _, a_fp4 = oracle.expert_mlp_nvfp4(x[0], *fp4, return_act=True)
    assert np.array_equal(a_fp4, a_bf16)


def test_expert_mlp_nvfp4_down_uses_the_quantised_activation():
    rng = np.random.default_rng(27)
    d, I = 256, 64
    _, (gate, up, (dq, dbs, sd)) = _nvfp4_expert(rng, d, I, 2)
    x, _, _, _ = _exact_rows(rng, 1, d, 1, -6)
    y, a = oracle.expert_mlp_nvfp4(x[0], gate, up, (dq, dbs, sd), return_act=True)
    # doubling the scale of output row c doubles y_c exactly and leaves the rest
    sd2 = sd.copy()
    sd2[5] *= 2
    y2 = oracle.expert_mlp_nvfp4(x[0], gate, up, (dq, dbs, sd2))
    assert y2[5] == 2 * y[5] and np.array_equal(np.delete(y2, 5), np.delete(y, 5))
    # permuting the down projection's output rows permutes y
    perm = rng.permutation(d)
    y3 = oracle.expert_mlp_nvfp4(x[0], gate, up, (dq[perm], dbs[perm], sd[perm]))
    assert np.array_equal(y3, y[perm])
    # y is the down projection of the activation's NVFP4 values: equal (to FP32 rounding) to a
    # float64 product with the decoded activation, and different from the unquantised one
    av = oracle.bf16_to_f32(a).astype(np.float64)
    aq, abs_, sa = oracle.quantize_rows_nvfp4(torch.from_numpy(av.astype(np.float32)[None]).to(torch.bfloat16))
    a_hat = (oracle.e2m1_to_f32(aq[0]).astype(np.float64)
             * np.repeat(oracle.e4m3_to_f32(abs_[0]).astype(np.float64), 16) * float(sa[0]))
    Wd = (oracle.e2m1_to_f32(dq).astype(np.float64)
          * np.repeat(oracle.e4m3_to_f32(dbs).astype(np.float64), 16, axis=1) * sd[:, None])
    np.testing.assert_allclose(y, (Wd @ a_hat).astype(np.float32), rtol=2 ** -22, atol=1e-30)
    assert not np.allclose(y, Wd @ av, rtol=1e-3, atol=0)


def test_moe_tokens_nvfp4_is_weighted_sum_of_nvfp4_experts():
    rng = np.random.default_rng(28)
    d, I, E, k, T = 256, 64, 4, 2, 5
    experts = {e: _nvfp4_expert(rng, d, I, 2)[1] for e in range(E)}
    h = torch.from_numpy(rng.normal(0, 1, (T, d)).astype(np.float32)).to(torch.bfloat16)
    idx = np.array([[0, 1], [1, 3], [0, 2], [2, 3], [1, 2]], np.int32)
    w = rng.uniform(0.5, 2.0, (T, k)).astype(np.float32)
    out = oracle.moe_tokens_nvfp4(np.arange(T), h, idx, w, experts)
    for t in range(T):
        ys = [oracle.expert_mlp_nvfp4(h[t], *experts[e]).astype(np.float64) for e in idx[t]]
        ref = sum(float(w[t, j]) * ys[j] for j in range(k))
        assert np.array_equal(out[t], ref.astype(np.float32))


def test_quantize_rows_nvfp4_symmetries():
    """Exact symmetries of the reading: a power-of-two factor on a row moves only its row scale;
    negating a row flips only the code signs; permuting whole 16-element blocks permutes the
    codes and block scales with them."""
    rng = np.random.default_rng(29)
    x = rng.normal(0, 1, (16, 256)).astype(np.float32)
    x[2, :16] *= 1e-3                   # a block far below the row maximum
    xb = torch.from_numpy(x).to(torch.bfloat16)
    q, bs, s = oracle.quantize_rows_nvfp4(xb)
    for k in (-7, 3, 11):
        q2, bs2, s2 = oracle.quantize_rows_nvfp4((xb.float() * 2.0 ** k).to(torch.bfloat16))
        assert np.array_equal(q2, q) and np.array_equal(bs2, bs)
        assert np.array_equal(s2, (s.astype(np.float64) * 2.0 ** k).astype(np.float32))
    qn, bsn, sn = oracle.quantize_rows_nvfp4(-xb)
    assert np.array_equal(bsn, bs) and np.array_equal(sn, s)
    assert np.array_equal(oracle.e2m1_to_f32(qn), -oracle.e2m1_to_f32(q))
    perm = rng.permutation(16)
    xp = xb.reshape(16, 16, 16)[:, perm].reshape(16, 256)
    qp, bsp, sp = oracle.quantize_rows_nvfp4(xp)
    assert np.array_equal(sp, s) and np.array_equal(bsp, bs[:, perm])
    assert np.array_equal(qp, q.reshape(16, 16, 16)[:, perm].reshape(16, 256))
