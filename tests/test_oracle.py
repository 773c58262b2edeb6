"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: byte counts
printed on the pages, closed forms, exact rational arithmetic, constructed
blocks with known answers, and invariants of the definition
w = (q - zp) * scale.  A plausible slip in the oracle (a swapped nibble, a
wrong block index, a transposed operand, round-half-away instead of
half-to-even, a dropped zero point) fails at least one of them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_sizes.json")
MB = 1e6


def _pack_rows(q):
    """Independent restatement of the nibble order: element 2j low, 2j+1 high."""
    q = np.asarray(q, dtype=np.uint8)
    return (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)


def _unpack_rows(p):
    p = np.asarray(p, dtype=np.uint8)
    out = np.zeros((p.shape[0], p.shape[1] * 2), np.int64)
    out[:, 0::2] = p & 15
    out[:, 1::2] = p >> 4
    return out


# ---------------------------------------------------------------- page byte counts

def _model_bytes(linears, bs, scale_dtype, has_zp):
    total = 0
    for lin in linears:
        p, s, z = oracle.packed_sizes(lin.N, lin.K, bs, scale_dtype, has_zp)
        total += p + s + z
    return total


def test_page_byte_counts_pin_layout():
    g = json.load(open(GOLDEN))
    # int8 table and its fp32 scales
    assert round(151936 * 1024 / MB, 1) == g["int8_embed_table"]["printed_mb"]
    assert round(151936 * 4 / MB, 1) == g["embed_scales"]["printed_mb"]
    # 0.6B decoder, block 64, fp32 scales, 4-bit zero points packed two per byte
    lin = workloads.qwen3_0p6b()
    w = _model_bytes(lin, 64, np.float32, True)
    assert w == 339_897_344
    assert round(w / MB) == g["decoder_0p6b_block64_without_embedding"]["printed_mb"]
    emb = 151936 * 1024 * 4
    assert round((w + emb) / MB) == g["decoder_0p6b_block64_with_fp32_embedding"]["printed_mb"]
    # the alternative layouts do NOT give the printed figure
    assert round(_model_bytes(lin, 64, np.float16, True) / MB) != 340     # fp16 scales
    zp_u8 = sum(l.N * (l.K // 64) for l in lin)                          # one byte per zp
    assert round((w - sum(oracle.packed_sizes(l.N, l.K, 64)[2] for l in lin) + zp_u8) / MB) != 340


def test_page_compression_ratio_block32_fp16_scales():
    g = json.load(open(GOLDEN))
    lin = workloads.qwen3_1p7b()
    fp16 = sum(l.N * l.K * 2 for l in lin)
    q4 = _model_bytes(lin, 32, np.float16, True)
    assert round(fp16 / q4, 1) == g["decoder_1p7b_compression"]["ratio"]
    assert q4 == 994_635_776


def test_packed_sizes_small_cases():
    assert oracle.packed_sizes(3, 64, 32, np.float32, True) == (96, 24, 3)
    assert oracle.packed_sizes(3, 96, 32, np.float16, True) == (144, 18, 6)   # odd nb: ceil
    assert oracle.packed_sizes(5, 64, 64, np.float16, False) == (160, 10, 0)
    with pytest.raises(ValueError):
        oracle.packed_sizes(4, 48, 32)


# ---------------------------------------------------------------- dequantization

@pytest.mark.parametrize("scale", [1.0, 0.5, 0.037109375, 1e-3, 3.0e4, 2.0 ** -20])
def test_dequant_exhaustive_q_zp(scale):
    # one row per (q, zp) pair; every element of the row holds q
    pairs = [(q, z) for q in range(16) for z in range(16)]
    N, K, bs = len(pairs), 64, 32
    q = np.array([[p[0]] * K for p in pairs])
    zp_nib = np.array([[p[1], p[1]] for p in pairs])
    packed = _pack_rows(q)
    zp = _pack_rows(zp_nib)
    for sdt in (np.float32, np.float16):
        s = np.full((N, K // bs), scale, sdt)
        w = oracle.dequantize(packed, s, zp, K, bs)
        sv = float(sdt(scale))
        expect = np.array([[(p[0] - p[1]) * sv] * K for p in pairs])
        assert np.array_equal(w, expect)


def test_dequant_nibble_and_zp_order():
    # element k of the row holds q = k % 16; block b has zp = (3 * b) % 16 and scale 2^b
    N, K, bs = 2, 128, 32
    nb = K // bs
    q = np.tile(np.arange(K) % 16, (N, 1))
    zpn = np.tile((3 * np.arange(nb)) % 16, (N, 1))
    s = np.tile(2.0 ** np.arange(nb), (N, 1)).astype(np.float32)
    w = oracle.dequantize(_pack_rows(q), s, _pack_rows(zpn), K, bs)
    for k in range(K):
        b = k // bs
        assert w[0, k] == (k % 16 - (3 * b) % 16) * 2.0 ** b


def test_dequant_zp_defaults_to_8():
    rng = np.random.default_rng(5)
    N, K, bs = 7, 96, 32
    packed = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    s = rng.random((N, K // bs), dtype=np.float32)
    explicit = np.full((N, (K // bs + 1) // 2), 0x88, np.uint8)
    assert np.array_equal(oracle.dequantize(packed, s, None, K, bs),
                          oracle.dequantize(packed, s, explicit, K, bs))


def test_dequant_rounded_outputs_are_single_roundings():
    rng = np.random.default_rng(6)
    N, K, bs = 16, 128, 32
    packed = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    zp = rng.integers(0, 256, (N, 2), dtype=np.uint8)
    s32 = (rng.random((N, K // bs)) * 0.1).astype(np.float32)
    exact = oracle.dequantize(packed, s32, zp, K, bs, np.float64)
    assert np.array_equal(oracle.dequantize(packed, s32, zp, K, bs, np.float32), exact.astype(np.float32))
    assert np.array_equal(oracle.dequantize(packed, s32, zp, K, bs, np.float16), exact.astype(np.float16))


# ---------------------------------------------------------------- RTN quantization

def test_rtn_constructed_exact_block():
    # values k * 0.5 for k = -7..8, each twice: scale 0.5, zp 7, q = k + 7, error 0
    v = np.repeat(np.arange(-7, 9) * 0.5, 2).astype(np.float32)[None, :]
    packed, s, zp = oracle.quantize_rtn(v, 32)
    assert s[0, 0] == 0.5
    assert (zp[0, 0] & 15) == 7 and (zp[0, 0] >> 4) == 0
    assert list(packed[0]) == [0x11 * j for j in range(16)]
    assert np.array_equal(oracle.dequantize(packed, s, zp, 32, 32)[0], v[0].astype(np.float64))


def test_rtn_ties_round_half_to_even():
    # lo = 0, hi = 15 -> scale 1, zp 0; x.5 values must round to even
    v = np.zeros((1, 32), np.float32)
    v[0, 0] = 15.0
    halves = np.arange(0.5, 15.0, 1.0)
    v[0, 1:1 + len(halves)] = halves
    packed, s, zp = oracle.quantize_rtn(v, 32)
    assert s[0, 0] == 1.0 and (zp[0, 0] & 15) == 0
    q = _unpack_rows(packed)[0]
    for i, h in enumerate(halves):
        lo = int(np.floor(h))
        assert q[1 + i] == (lo if lo % 2 == 0 else lo + 1)
    assert q[0] == 15


def test_rtn_tie_is_broken_after_adding_zp():
    # lo = -7, hi = 8 -> scale 1, zp 7.  v = 0.5 -> 7.5 -> 8 (even); rounding v
    # first and adding zp afterwards would give 7.
    v = np.zeros((1, 32), np.float32)
    v[0, 0], v[0, 1], v[0, 2], v[0, 3] = -7.0, 8.0, 0.5, -0.5
    packed, s, zp = oracle.quantize_rtn(v, 32)
    assert s[0, 0] == 1.0 and (zp[0, 0] & 15) == 7
    q = _unpack_rows(packed)[0]
    assert q[2] == 8 and q[3] == 6


def _blocks(rng, kind, n, bs):
    if kind == "normal":
        return rng.normal(0, 0.02, (n, bs))
    if kind == "positive":
        return rng.uniform(0.1, 0.5, (n, bs))
    if kind == "negative":
        return -rng.uniform(0.01, 3.0, (n, bs))
    if kind == "outliers":
        w = rng.normal(0, 0.02, (n, bs))
        return np.where(rng.random((n, bs)) < 0.05, w * 8, w)
    if kind == "tiny":
        return rng.normal(0, 1e-30, (n, bs))
    if kind == "sparse":
        w = rng.normal(0, 1.0, (n, bs))
        return np.where(rng.random((n, bs)) < 0.7, 0.0, w)
    raise KeyError(kind)


@pytest.mark.parametrize("kind", ["normal", "positive", "negative", "outliers", "tiny", "sparse"])
@pytest.mark.parametrize("bs", [32, 64])
def test_rtn_roundtrip_error_at_most_half_scale(kind, bs):
    rng = np.random.default_rng(hash((kind, bs)) % 2 ** 32)
    W = _blocks(rng, kind, 64, 4 * bs).astype(np.float32)
    packed, s, zp = oracle.quantize_rtn(W, bs)
    w = oracle.dequantize(packed, s, zp, W.shape[1], bs)
    smax = np.repeat(s.astype(np.float64), bs, axis=1)
    err = np.abs(w - W.astype(np.float64))
    assert np.all(err <= smax * (0.5 + 1e-5))
    # the range spans exactly 15 steps of the scale (up to one fp32 rounding)
    Wb = W.reshape(64, -1, bs).astype(np.float64)
    span = np.maximum(Wb.max(-1), 0) - np.minimum(Wb.min(-1), 0)
    assert np.allclose(s * 15.0, span, rtol=1e-6, atol=0)


def test_rtn_all_zero_block():
    W = np.zeros((2, 64), np.float32)
    W[1, 32:] = np.linspace(-1, 1, 32)
    packed, s, zp = oracle.quantize_rtn(W, 32)
    assert s[0, 0] == 0 and s[0, 1] == 0 and s[1, 0] == 0
    assert np.all(packed[0] == 0) and np.all(packed[1, :16] == 0)
    assert (zp[0, 0] == 0) and (zp[1, 0] & 15) == 0
    assert np.all(oracle.dequantize(packed, s, zp, 64, 32)[0] == 0)


@pytest.mark.parametrize("bs", [32, 64])
def test_rtn_idempotent_on_representable_blocks(bs):
    # power-of-two scale, every block holds q = 0 and q = 15: quantize(dequantize) is the identity
    rng = np.random.default_rng(11)
    N, K = 32, 4 * bs
    q = rng.integers(0, 16, (N, K))
    q[:, ::bs] = 0
    q[:, 1::bs] = 15
    z = rng.integers(0, 16, (N, K // bs))
    s = (2.0 ** rng.integers(-12, -2, (N, K // bs))).astype(np.float32)
    zpk = np.zeros((N, (K // bs + 1) // 2 * 2), np.int64)
    zpk[:, : K // bs] = z
    W = oracle.dequantize(_pack_rows(q), s, _pack_rows(zpk), K, bs, np.float32)
    for sdt in (np.float32, np.float16):
        p2, s2, zp2 = oracle.quantize_rtn(W, bs, scale_dtype=sdt)
        assert np.array_equal(_unpack_rows(p2), q)
        assert np.array_equal(s2.astype(np.float64), s.astype(np.float64))
        assert np.array_equal(_unpack_rows(zp2)[:, : K // bs], z)


def test_rtn_fp16_scale_is_the_rounded_fp32_scale():
    rng = np.random.default_rng(12)
    W = rng.normal(0, 0.02, (16, 256)).astype(np.float32)
    p32, s32, z32 = oracle.quantize_rtn(W, 32, scale_dtype=np.float32)
    p16, s16, z16 = oracle.quantize_rtn(W, 32, scale_dtype=np.float16)
    assert np.array_equal(p32, p16) and np.array_equal(z32, z16)
    assert np.array_equal(s16, s32.astype(np.float16))     # numpy's own fp32 -> fp16 rounding


@pytest.mark.parametrize("bs", [32, 64])
def test_rtn_symmetric_variant_bound(bs):
    # reading R8 (no zero points, zp = 8): parity unpinned by the pages; only its bound is checked
    rng = np.random.default_rng(13)
    W = rng.normal(0, 0.02, (16, 4 * bs)).astype(np.float32)
    W[0, :bs] = 0.0
    packed, s, zp = oracle.quantize_rtn(W, bs, has_zp=False)
    assert zp is None
    w = oracle.dequantize(packed, s, None, W.shape[1], bs)
    smax = np.repeat(s.astype(np.float64), bs, axis=1)
    assert np.all(np.abs(w - W) <= smax * (0.5 + 1e-5))
    assert np.all(_unpack_rows(packed)[0, :bs] == 8)


# ---------------------------------------------------------------- the matmul

def _exact_matmul(X, packed, scales, zp, K, bs):
    """Exact rational Y = X . dequant(W)^T from the stored bits (independent unpack)."""
    M, N = X.shape[0], packed.shape[0]
    q = _unpack_rows(packed)
    z = _unpack_rows(zp) if zp is not None else None
    Y = [[Fraction(0)] * N for _ in range(M)]
    for n in range(N):
        w = []
        for k in range(K):
            b = k // bs
            zz = int(z[n, b]) if z is not None else 8
            w.append((int(q[n, k]) - zz) * Fraction(float(scales[n, b])))
        for m in range(M):
            Y[m][n] = sum(Fraction(float(X[m, k])) * w[k] for k in range(K))
    return Y


@pytest.mark.parametrize("bs,has_zp,sdt", [(32, True, np.float32), (64, True, np.float16),
                                            (32, False, np.float16)])
def test_matmul_brute_force_exact(bs, has_zp, sdt):
    rng = np.random.default_rng(21)
    M, K, N = 4, 64, 8
    packed = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    zp = rng.integers(0, 256, (N, (K // bs + 1) // 2), dtype=np.uint8) if has_zp else None
    scales = (rng.random((N, K // bs)) * 0.1 + 0.01).astype(sdt)
    X = rng.normal(0, 1, (M, K)).astype(np.float16)
    Y = oracle.matmul(X, packed, scales, zp, K, bs)
    E = _exact_matmul(X, packed, scales, zp, K, bs)
    for m in range(M):
        for n in range(N):
            assert abs(Fraction(Y[m, n]) - E[m][n]) <= Fraction(1, 2 ** 40)


def test_matmul_blocks_with_q_equal_zp_contribute_zero():
    rng = np.random.default_rng(22)
    M, K, N, bs = 3, 128, 5, 32
    nb = K // bs
    z = rng.integers(0, 16, (N, nb))
    q = np.repeat(z, bs, axis=1)
    packed, zp = _pack_rows(q), _pack_rows(z)
    scales = rng.random((N, nb)).astype(np.float32)
    X = rng.normal(0, 1, (M, K))
    assert np.all(oracle.matmul(X, packed, scales, zp, K, bs) == 0.0)
    # one block at zero contribution: changing X inside it leaves Y unchanged
    q2 = rng.integers(0, 16, (N, K))
    q2[:, bs:2 * bs] = np.repeat(z[:, 1:2], bs, axis=1)
    X2 = X.copy()
    X2[:, bs:2 * bs] = rng.normal(0, 5, (M, bs))
    A = oracle.matmul(X, _pack_rows(q2), scales, zp, K, bs)
    B = oracle.matmul(X2, _pack_rows(q2), scales, zp, K, bs)
    assert np.allclose(A, B, rtol=1e-12, atol=1e-12)


def test_matmul_block64_equals_paired_block32():
    rng = np.random.default_rng(23)
    M, K, N = 2, 256, 6
    packed = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    s64 = rng.random((N, K // 64)).astype(np.float32)
    z64 = rng.integers(0, 16, (N, K // 64))
    s32 = np.repeat(s64, 2, axis=1)
    z32 = np.repeat(z64, 2, axis=1)
    X = rng.normal(0, 1, (M, K))
    A = oracle.matmul(X, packed, s64, _pack_rows(z64), K, 64)
    B = oracle.matmul(X, packed, s32, _pack_rows(z32), K, 32)
    assert np.array_equal(A, B)
    assert np.array_equal(oracle.dequantize(packed, s64, _pack_rows(z64), K, 64),
                          oracle.dequantize(packed, s32, _pack_rows(z32), K, 32))


def test_matmul_column_subset_and_transpose_orientation():
    rng = np.random.default_rng(24)
    M, K, N, bs = 3, 96, 40, 32
    packed = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    zp = rng.integers(0, 256, (N, 2), dtype=np.uint8)
    s = rng.random((N, K // bs)).astype(np.float32)
    X = rng.normal(0, 1, (M, K))
    full = oracle.matmul(X, packed, s, zp, K, bs)
    assert full.shape == (M, N)
    cols = [39, 0, 17, 17, 5]
    assert np.array_equal(oracle.matmul(X, packed, s, zp, K, bs, cols=cols), full[:, cols])
    # Y = X . W^T: a unit row of X picks column k of every weight row
    W = oracle.dequantize(packed, s, zp, K, bs)
    E = np.zeros((1, K))
    E[0, 7] = 1.0
    assert np.array_equal(oracle.matmul(E, packed, s, zp, K, bs)[0], W[:, 7])
    with pytest.raises(ValueError):
        oracle.matmul(X, packed, s, zp, K, bs, cols=[N])


# ---------------------------------------------------------------- embedding gather

def test_embed_power_of_two_scales_exact_and_bad_ids():
    rng = np.random.default_rng(31)
    V, D, T = 50, 64, 20
    table = rng.integers(-128, 128, (V, D), dtype=np.int64).astype(np.int8)
    scales = (2.0 ** rng.integers(-10, -3, V)).astype(np.float32)
    ids = rng.integers(0, V, T).astype(np.int32)
    ids[3], ids[7] = -1, V
    out, st = oracle.embed_gather(table, scales, ids, np.float16)
    assert st == 1
    for t in range(T):
        if t in (3, 7):
            assert np.all(out[t] == 0)
        else:
            assert np.array_equal(out[t].astype(np.float64),
                                  table[ids[t]].astype(np.float64) * float(scales[ids[t]]))
    out32, st32 = oracle.embed_gather(table, scales, ids[:3], np.float32)
    assert st32 == 0


def test_embed_fp16_is_rounded_from_the_fp32_product():
    rng = np.random.default_rng(32)
    V, D, T = 40, 128, 30
    table = rng.integers(-128, 128, (V, D), dtype=np.int64).astype(np.int8)
    scales = rng.uniform(0.001, 0.05, V).astype(np.float32)
    ids = rng.integers(0, V, T).astype(np.int32)
    o32, _ = oracle.embed_gather(table, scales, ids, np.float32)
    o16, _ = oracle.embed_gather(table, scales, ids, np.float16)
    prod = table[ids].astype(np.float32) * scales[ids][:, None]      # numpy's fp32 product
    assert np.array_equal(o32, prod)
    assert np.array_equal(o16, prod.astype(np.float16))


def test_swiglu_closed_forms():
    # silu(x) = x * sigmoid(x): zero at 0, 1/(1 + 1/e) at 1, odd part x, limits x and 0
    x = np.array([0.0, 1.0, -1.0, 2.5, -2.5, 40.0, -40.0])
    ones = np.ones_like(x)
    s = oracle.swiglu(x, ones)
    assert s[0] == 0.0
    assert abs(s[1] - 1.0 / (1.0 + np.exp(-1.0))) < 1e-15
    assert abs(s[1] - 0.7310585786300049) < 1e-15
    assert np.allclose(s[1::2][:3] - s[2::2][:3], x[1::2][:3], rtol=0, atol=1e-14)
    assert abs(s[5] - 40.0) < 1e-15 and abs(s[6]) < 1e-15
    # the up factor multiplies
    assert np.allclose(oracle.swiglu(x, 3.0 * ones), 3.0 * s, rtol=1e-15, atol=0)


# ---- GPTQ ("Mega-ASR -- INT4 ONNX (GPTQ-calibrated)", "Conversion details":
# algo=GPTQ; "GPTQ calibration") -------------------------------------------------

def _codes(packed, K):
    """Unpacked 4-bit codes [N, K] (low nibble first)."""
    p = np.asarray(packed, np.uint8)
    out = np.empty((p.shape[0], K), np.int64)
    out[:, 0::2] = p & 15
    out[:, 1::2] = p >> 4
    return out


def test_gptq_hessian_is_the_exact_gram_matrix():
    rng = np.random.default_rng(0)
    X = rng.integers(-7, 8, (9, 6)).astype(np.float64)
    H = oracle.gptq_hessian(X)
    ref = [[sum(int(X[t, i]) * int(X[t, j]) for t in range(9)) for j in range(6)] for i in range(6)]
    assert np.array_equal(H, np.array(ref, np.float64))


def test_gptq_prepare_diagonal_closed_form():
    d = np.array([4.0, 0.0, 9.0, 2.25])            # feature 1 never active: dead
    U, dead = oracle.gptq_prepare(np.diag(d), percdamp=0.01)
    dd = np.array([4.0, 1.0, 9.0, 2.25])
    damp = 0.01 * dd.mean()
    assert np.array_equal(dead, [0, 1, 0, 0])
    assert np.allclose(U, np.diag(1.0 / np.sqrt(dd + damp)), rtol=1e-15, atol=0)


def test_gptq_prepare_factor_inverts_the_damped_hessian():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((200, 48)) @ rng.standard_normal((48, 48))
    H = oracle.gptq_hessian(X)
    U, dead = oracle.gptq_prepare(H, percdamp=0.05)
    assert not dead.any()
    Hd = H + 0.05 * np.mean(np.diag(H)) * np.eye(48)
    assert np.allclose(np.triu(U), U) and np.all(np.diag(U) > 0)     # upper, positive diagonal
    assert np.allclose(U.T @ U @ Hd, np.eye(48), atol=1e-9)          # U^T U = Hd^-1


@pytest.mark.parametrize("bs,has_zp,sdt", [(32, True, np.float16), (64, True, np.float32),
                                           (32, False, np.float16), (64, False, np.float32)])
def test_gptq_with_a_diagonal_hessian_is_rtn(bs, has_zp, sdt):
    # uncorrelated inputs: U is diagonal, no error flows to later columns, and
    # every block is quantized from its original values -- exactly RTN
    rng = np.random.default_rng(bs + has_zp)
    K, N = 4 * bs, 7
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    U, dead = oracle.gptq_prepare(np.diag(rng.uniform(0.5, 3.0, K)))
    g = oracle.gptq_quantize(W, U.astype(np.float32), bs, has_zp, sdt, dead)
    r = oracle.quantize_rtn(W, bs, has_zp, sdt)
    assert np.array_equal(g[0], r[0])
    assert np.array_equal(g[1].view(np.uint8), r[1].view(np.uint8))
    if has_zp:
        assert np.array_equal(g[2], r[2])


def _gptq_by_downdates(W, H, bs, has_zp, percdamp=0.01):
    """GPTQ written independently of the oracle: float64, with the explicit
    inverse Hessian of the not-yet-quantized columns, downdated after each
    column (w_F -= (w_i - q_i) H_F^-1[i, F] / H_F^-1[i, i]); the quantizer's
    decisions in float32 as the method's.  Returns the codes [N, K]."""
    K = H.shape[0]
    Hd = np.array(H, np.float64)
    d = np.diag(Hd).copy()
    d[d == 0] = 1.0
    Hd[np.arange(K), np.arange(K)] = d + percdamp * d.mean()
    Hinv = np.linalg.inv(Hd)
    coef = np.zeros((K, K))
    for i in range(K):
        coef[i, i + 1:] = Hinv[i, i + 1:] / Hinv[i, i]
        Hinv = Hinv - np.outer(Hinv[:, i], Hinv[i, :]) / Hinv[i, i]
    f32 = np.float32
    codes = np.zeros(W.shape, np.int64)
    for n in range(W.shape[0]):
        w = W[n].astype(np.float64)
        for i in range(K):
            if i % bs == 0:
                v = w[i:i + bs].astype(f32)
                if has_zp:
                    lo, hi = min(f32(0), v.min()), max(f32(0), v.max())
                    s = f32(f32(hi - lo) / f32(15))
                    z = int(np.clip(np.rint(f32(-lo) / s), 0, 15)) if s != 0 else 0
                else:
                    s = f32(np.abs(v).max() / f32(7))
                    z = 8
            wi = f32(w[i])
            if s == 0:
                q = 0 if has_zp else 8
            elif has_zp:
                q = int(np.clip(np.rint(f32(f32(wi / s) + f32(z))), 0, 15))
            else:
                q = int(np.clip(np.rint(f32(wi / s)) + 8, 0, 15))
            codes[n, i] = q
            w[i + 1:] -= (w[i] - (q - z) * float(s)) * coef[i, i + 1:]
    return codes


@pytest.mark.parametrize("seed,bs,has_zp", [(0, 32, True), (1, 64, True), (2, 32, False), (3, 32, True)])
def test_gptq_matches_an_independent_formulation(seed, bs, has_zp):
    rng = np.random.default_rng(seed)
    K, N = 3 * bs, 6
    X = rng.standard_normal((400, K)) @ rng.standard_normal((K, K)) * 0.3 + rng.standard_normal((400, K))
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    H = oracle.gptq_hessian(X)
    U, dead = oracle.gptq_prepare(H)
    packed, _, _ = oracle.gptq_quantize(W, U.astype(np.float32), bs, has_zp, np.float32, dead)
    assert np.array_equal(_codes(packed, K), _gptq_by_downdates(W, H, bs, has_zp))


def test_gptq_lowers_the_proxy_loss_below_rtn():
    # correlated calibration inputs: GPTQ's error feedback must beat plain
    # rounding on ||(W - W^) X^T||^2, the loss it minimizes
    rng = np.random.default_rng(7)
    K, N, bs = 128, 32, 32
    X = rng.standard_normal((1024, K)) @ rng.standard_normal((K, K))
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    U, dead = oracle.gptq_prepare(oracle.gptq_hessian(X))
    g = oracle.gptq_quantize(W, U.astype(np.float32), bs, True, np.float32, dead)
    r = oracle.quantize_rtn(W, bs, True, np.float32)

    def loss(q):
        Wq = oracle.dequantize(q[0], q[1], q[2], K, bs)
        return float(np.sum(((W.astype(np.float64) - Wq) @ X.T) ** 2))

    assert loss(g) < 0.8 * loss(r)


def test_gptq_dead_features_get_zero_weights():
    rng = np.random.default_rng(8)
    K, N, bs = 64, 5, 32
    X = rng.standard_normal((300, K))
    X[:, [3, 40]] = 0.0                      # two input features never active
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    U, dead = oracle.gptq_prepare(oracle.gptq_hessian(X))
    assert dead[3] == 1 and dead[40] == 1 and dead.sum() == 2
    p, s, z = oracle.gptq_quantize(W, U.astype(np.float32), bs, True, np.float32, dead)
    Wq = oracle.dequantize(p, s, z, K, bs)
    assert np.all(Wq[:, [3, 40]] == 0.0)
