"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test checks the oracle against hand-worked values (tests/golden), a
library routine (numpy's binary16 decoder, numpy's float64 matmul on tiny
inputs), a closed form, or an invariant of the mathematics, chosen so that a
plausible mistake (a dropped term, a wrong sign, a wrong byte or nibble index,
a transposed operand) fails at least one of them.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from dequant_gemv_q4_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hex(s):
    return np.frombuffer(bytes.fromhex(s.replace(" ", "")), dtype=np.uint8)


def _q4k_golden_block(spec):
    blk = np.zeros(144, np.uint8)
    blk[0:2] = _hex(spec["d_hex"])[::-1]       # hex is written big-endian, bytes are LE
    blk[2:4] = _hex(spec["dmin_hex"])[::-1]
    blk[4:16] = _hex(spec["scales_hex"])
    if "qs_fill" in spec:
        blk[16:] = spec["qs_fill"]
    else:
        b = np.arange(128)
        blk[16:] = (b % 16) + 16 * (b // 16)
    return blk


def _expected(spec):
    if "expected" in spec:
        return np.array(spec["expected"], np.float64)
    if "expected_runs" in spec:
        return np.concatenate([np.full(n, v, np.float64) for v, n in spec["expected_runs"]])
    vals = []
    for (num, den), n in spec["expected_runs_fraction"]:
        vals += [float(Fraction(num, den))] * n
    return np.array(vals, np.float64)


# --- binary16 decoder ------------------------------------------------------------

def test_fp16_decoder_matches_numpy_for_every_bit_pattern():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([oracle.fp16_to_double(int(h)) for h in pats])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])
    # the signed zeros are distinct bit patterns
    assert np.signbit(oracle.fp16_to_double(0x8000)) and not np.signbit(oracle.fp16_to_double(0))


# --- Q4_K scale/min packing ----------------------------------------------------------

# The packing written as data: for each field, the (byte, bit) that holds each
# of its six bits, least significant first.  scale_j / min_j for j < 4 are bits
# 0..5 of byte j / j+4; for j >= 4 the low four bits come from byte j+4 (its
# low nibble for scales, high nibble for mins) and the top two bits from bits
# 6..7 of byte j-4 (scales) or byte j (mins).
FIELD_BITS = {}
for _j in range(4):
    FIELD_BITS[("scale", _j)] = [(_j, b) for b in range(6)]
    FIELD_BITS[("min", _j)] = [(_j + 4, b) for b in range(6)]
for _j in range(4, 8):
    FIELD_BITS[("scale", _j)] = [(_j + 4, b) for b in range(4)] + [(_j - 4, 6), (_j - 4, 7)]
    FIELD_BITS[("min", _j)] = [(_j + 4, b) for b in range(4, 8)] + [(_j, 6), (_j, 7)]


def test_scale_min_fields_cover_all_96_bits_once():
    used = [pos for bits in FIELD_BITS.values() for pos in bits]
    assert len(used) == 96 and len(set(used)) == 96


@pytest.mark.parametrize("field", sorted(FIELD_BITS))
def test_scale_min_single_field_exhaustive(field):
    kind, j = field
    for v in range(64):
        s = np.zeros(12, np.uint8)
        for bit, (byte, pos) in enumerate(FIELD_BITS[field]):
            if (v >> bit) & 1:
                s[byte] |= np.uint8(1 << pos)
        sc, mn = oracle.q4k_scale_min(s)
        want_sc = [v if (kind == "scale" and i == j) else 0 for i in range(8)]
        want_mn = [v if (kind == "min" and i == j) else 0 for i in range(8)]
        assert (sc, mn) == (want_sc, want_mn), (field, v)


def test_scale_min_packing_is_a_bijection_on_random_bytes():
    rng = np.random.default_rng(123)
    for _ in range(500):
        s = rng.integers(0, 256, 12, dtype=np.uint8)
        sc, mn = oracle.q4k_scale_min(s)
        rebuilt = np.zeros(12, np.uint8)
        for (kind, j), bits in FIELD_BITS.items():
            v = sc[j] if kind == "scale" else mn[j]
            assert 0 <= v < 64
            for bit, (byte, pos) in enumerate(bits):
                if (v >> bit) & 1:
                    rebuilt[byte] |= np.uint8(1 << pos)
        assert np.array_equal(rebuilt, s)


# --- hand-worked blocks ------------------------------------------------------------

Q4K_GOLDEN = json.load(open(os.path.join(GOLDEN, "q4k_handworked.json")))["blocks"]
Q8_GOLDEN = json.load(open(os.path.join(GOLDEN, "q8_0_handworked.json")))["blocks"]


@pytest.mark.parametrize("spec", Q4K_GOLDEN, ids=[b["name"] for b in Q4K_GOLDEN])
def test_q4k_handworked_block(spec):
    blk = _q4k_golden_block(spec)
    sc, mn = oracle.q4k_scale_min(blk[4:16])
    assert sc == spec["scale"] and mn == spec["min"]
    w = oracle.q4k_block(blk)
    assert np.array_equal(w, _expected(spec))
    # the same block through the whole-matrix entry points, at a row offset
    mat = np.concatenate([np.zeros(144, np.uint8), blk]).reshape(1, 288)
    full = oracle.q4k_dequant(mat, 1, 512)
    assert np.array_equal(full[0, 256:], _expected(spec))
    f32 = oracle.q4k_dequant_f32(mat, 1, 512)
    assert np.array_equal(f32[0, 256:], _expected(spec).astype(np.float32))


@pytest.mark.parametrize("spec", Q8_GOLDEN, ids=[b["name"] for b in Q8_GOLDEN])
def test_q8_0_handworked_block(spec):
    blk = np.zeros(34, np.uint8)
    blk[0:2] = _hex(spec["d_hex"])[::-1]
    blk[2:] = _hex(spec["q_hex"])
    want = (np.array(spec["expected"], np.float64) if "expected" in spec
            else np.full(32, spec["expected_fill"], np.float64))
    assert np.array_equal(oracle.q8_0_block(blk), want)
    mat = np.concatenate([blk, blk]).reshape(1, 68)
    assert np.array_equal(oracle.q8_0_dequant(mat, 1, 64)[0], np.concatenate([want, want]))
    # the fp32 dequant (the bit-exact reference of the GPU's debug dequant): every
    # hand-worked weight here is exact in fp32, so it must come back unchanged
    f32 = oracle.q8_0_dequant_f32(mat, 1, 64)[0]
    assert f32.dtype == np.float32
    assert np.array_equal(f32, np.concatenate([want, want]).astype(np.float32))


def test_nibble_order_rejects_the_low_nibbles_first_reading():
    # Under the other reading of the quant layout (all 128 low nibbles are
    # weights 0..127), weights 32..63 would be the low nibbles of bytes 32..63.
    spec = next(b for b in Q4K_GOLDEN if b["name"] == "nibble_order")
    w = oracle.q4k_block(_q4k_golden_block(spec))
    other = np.arange(32, 64) % 16
    assert not np.array_equal(w[32:64], other)


def test_q4k_quant_single_nibble_positions():
    # setting only the low nibble of byte 32c+r (r < 32) must move exactly weight 64c+r;
    # only the high nibble: exactly weight 64c+32+r.
    for c in range(4):
        for r in (0, 7, 31):
            qs = np.zeros(128, np.uint8)
            qs[32 * c + r] = 0x09
            got = [oracle.q4k_quant(qs, i) for i in range(256)]
            want = [0] * 256
            want[64 * c + r] = 9
            assert got == want
            qs[32 * c + r] = 0x90
            got = [oracle.q4k_quant(qs, i) for i in range(256)]
            want = [0] * 256
            want[64 * c + 32 + r] = 9
            assert got == want


# --- GEMV: brute force, closed forms, invariants ----------------------------------------

@pytest.mark.parametrize("N,K,B", [(8, 256, 1), (3, 512, 2), (5, 768, 3)])
def test_q4k_gemv_matches_dense_brute_force(N, K, B):
    rng = np.random.default_rng(N * 1000 + K + B)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, B, K)
    dense = oracle.q4k_dequant(w, N, K)
    y, a = oracle.q4k_gemv(w, N, K, x)
    ref = x.astype(np.float64) @ dense.T                         # (B, N)
    absref = np.abs(x.astype(np.float64)) @ np.abs(dense).T
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-13)
    assert np.allclose(a, absref, rtol=1e-13, atol=1e-13)
    # row selection returns the same numbers in the requested order
    rows = np.array([N - 1, 0])
    ys, as_ = oracle.q4k_gemv(w, N, K, x, rows=rows)
    assert np.array_equal(ys, y[:, rows]) and np.array_equal(as_, a[:, rows])


@pytest.mark.parametrize("N,K,B", [(8, 32, 1), (4, 1024, 2), (3, 96, 4)])
def test_q8_0_gemv_matches_dense_brute_force(N, K, B):
    rng = np.random.default_rng(N + K + B)
    w = synth.q8_0_matrix(rng, N, K)
    x = synth.activations(rng, B, K)
    dense = oracle.q8_0_dequant(w, N, K)
    y, a = oracle.q8_0_gemv(w, N, K, x)
    assert np.allclose(y, x.astype(np.float64) @ dense.T, rtol=1e-13, atol=1e-13)
    assert np.allclose(a, np.abs(x.astype(np.float64)) @ np.abs(dense).T, rtol=1e-13, atol=1e-13)


def _unit_q4k_matrix(N, nb, q_byte, m_val=0, dmin=0.0):
    """d = 1, every scale 1, every min m_val, every quant byte q_byte."""
    sc_bytes = np.array([1, 1, 1, 1, m_val, m_val, m_val, m_val,
                         1 | (m_val << 4), 1 | (m_val << 4), 1 | (m_val << 4), 1 | (m_val << 4)],
                        np.uint8)
    assert m_val < 16
    nblk = N * nb
    return synth.q4k_pack(np.ones(nblk, np.float16), np.full(nblk, dmin, np.float16),
                          np.tile(sc_bytes, (nblk, 1)),
                          np.full((nblk, 128), q_byte, np.uint8)).reshape(N, -1)


def test_q4k_gemv_closed_form_all_ones():
    # d=1, scale=1, min=0, q=1 everywhere: W is all ones, y = sum(x) exactly for integer x.
    N, K = 4, 1024
    w = _unit_q4k_matrix(N, K // 256, 0x11)
    x = np.arange(K, dtype=np.float32) % 7 - 3
    y, a = oracle.q4k_gemv(w, N, K, x)
    assert np.all(y == float(np.sum(x.astype(np.int64))))
    assert np.all(a == float(np.sum(np.abs(x.astype(np.int64)))))


def test_q4k_gemv_closed_form_cancelling_scale_and_min():
    # d=1, scale=1, dmin=1, min=1, q=1: every weight is 1*1*1 - 1*1 = 0 exactly.
    N, K = 3, 512
    w = _unit_q4k_matrix(N, K // 256, 0x11, m_val=1, dmin=1.0)
    x = synth.activations(np.random.default_rng(5), 1, K)
    y, a = oracle.q4k_gemv(w, N, K, x)
    assert np.all(y == 0.0) and np.all(a == 0.0)


def test_gemv_linearity_row_independence_and_k_additivity():
    rng = np.random.default_rng(77)
    N, K = 6, 512
    w = synth.q4k_matrix(rng, N, K)
    x1 = np.round(synth.activations(rng, 1, K) * 8) / 8       # dyadic: sums stay exact-ish
    x2 = np.round(synth.activations(rng, 1, K) * 8) / 8
    y1, _ = oracle.q4k_gemv(w, N, K, x1)
    y2, _ = oracle.q4k_gemv(w, N, K, x2)
    y12, _ = oracle.q4k_gemv(w, N, K, 2 * x1 - 0.5 * x2)
    assert np.allclose(y12, 2 * y1 - 0.5 * y2, rtol=1e-12, atol=1e-12)
    # row independence: changing row 2 alone changes y[2] alone
    w2 = w.copy()
    w2[2, 16 + 5] ^= 0x0F
    y1b, _ = oracle.q4k_gemv(w2, N, K, x1)
    changed = np.nonzero(y1b[0] != y1[0])[0]
    assert list(changed) == [2]
    # K-additivity: [W1 | W2] [x1; x2] = W1 x1 + W2 x2 at a super-block boundary
    wa, wb = w[:, :144], w[:, 144:]
    ya, _ = oracle.q4k_gemv(np.ascontiguousarray(wa), N, 256, x1[:, :256])
    yb, _ = oracle.q4k_gemv(np.ascontiguousarray(wb), N, 256, x1[:, 256:])
    assert np.allclose(y1, ya + yb, rtol=1e-13, atol=1e-13)


def test_batch_rows_are_independent_gemvs():
    rng = np.random.default_rng(3)
    N, K = 5, 256
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 3, K)
    y, a = oracle.q4k_gemv(w, N, K, x)
    for b in range(3):
        yb, ab = oracle.q4k_gemv(w, N, K, x[b])
        assert np.array_equal(y[b], yb[0]) and np.array_equal(a[b], ab[0])


# --- SwiGLU and argmax ------------------------------------------------------------------

def test_swiglu_identities():
    g = np.array([0.0, 1.5, -2.25, 30.0, -40.0, 1e-3])
    one = np.ones_like(g)
    s = oracle.swiglu(g, one)
    s_neg = oracle.swiglu(-g, one)
    # silu(g) - silu(-g) = g(sigma(g) + sigma(-g)) = g
    assert np.allclose(s - s_neg, g, rtol=1e-15, atol=1e-15)
    assert s[0] == 0.0                                  # silu(0) = 0
    assert abs(s[3] - 30.0) < 1e-11                     # silu(g) -> g for large g
    assert abs(s[4]) < 1e-15                            # silu(g) -> 0 for very negative g
    u = np.array([2.0, -3.0, 0.5, 1.0, 1.0, 4.0])
    assert np.allclose(oracle.swiglu(g, u), s * u, rtol=1e-15, atol=0)
    # W_up = W_gate: silu(g)g + silu(-g)(-g) = g^2 (sigma(g) + sigma(-g)) = g^2
    assert np.allclose(oracle.swiglu(g, g) + oracle.swiglu(-g, -g), g * g, rtol=1e-14, atol=1e-15)


def test_argmax_lowest_index_on_ties():
    assert oracle.argmax([1.0, 3.0, 3.0, 2.0]) == 1
    assert oracle.argmax([-5.0, -1.0, -1.0]) == 1
    assert oracle.argmax([7.0]) == 0
    assert oracle.argmax([0.0, -0.0, 0.0]) == 0
    v = np.zeros(1000)
    v[999] = 1e-30
    assert oracle.argmax(v) == 999


# --- structure-of-arrays repack -----------------------------------------------------------

@pytest.mark.parametrize("N,K", [(3, 4096), (2, 5120), (2, 1024), (1, 256)])
def test_soa_repack_is_a_row_permutation_and_decodes_identically(N, K):
    rng = np.random.default_rng(K + N)
    w = synth.q4k_matrix(rng, N, K)
    soa = oracle.q4k_repack_soa(w, N, K)
    assert soa.shape == w.shape
    for n in range(N):
        assert np.array_equal(np.sort(soa[n]), np.sort(w[n]))
    assert np.array_equal(oracle.q4k_dequant(soa, N, K, layout="soa"), oracle.q4k_dequant(w, N, K))
    x = synth.activations(rng, 1, K)
    assert np.array_equal(oracle.q4k_gemv(soa, N, K, x, layout="soa")[0],
                          oracle.q4k_gemv(w, N, K, x)[0])


def test_soa_positions_hand_derived():
    # one row of 6 super-blocks: a full group of 4 and a partial group of 2.
    N, K = 1, 6 * 256
    w = np.zeros((1, 6 * 144), np.uint8)
    w[0, 1 * 144 + 0] = 11            # block 1, header byte 0
    w[0, 0 * 144 + 16 + 16] = 22      # block 0, quant byte 16 (slice 1, byte 0)
    w[0, 5 * 144 + 16 + 127] = 33     # block 5 (group 1, t=1, g=2), quant byte 127 (slice 7, byte 15)
    soa = oracle.q4k_repack_soa(w, N, K)
    # group 0: 4 headers (64 B), then slice s of block t at 64 + 64*s + 16*t
    assert soa[0, 16] == 11
    assert soa[0, 64 + 64 * 1 + 0] == 22
    # group 1 starts at byte 4*144 = 576: 2 headers (32 B), slice s of block t at 32 + 32*s + 16*t
    assert soa[0, 576 + 32 + 32 * 7 + 16 * 1 + 15] == 33
    assert int(np.count_nonzero(soa)) == 3


# --- Q/gate de-interleave (Doppler split_qg.wgsl) -------------------------------------

def test_split_qg_hand_derived():
    # two heads of head_dim 2: row = [Q0 Q0 G0 G0 Q1 Q1 G1 G1]
    y = np.array([[10, 11, 20, 21, 12, 13, 22, 23]], np.float64)
    q, g = oracle.split_qg(y, 2)
    assert q.tolist() == [[10, 11, 12, 13]]
    assert g.tolist() == [[20, 21, 22, 23]]
    # head_dim = N/2: one head, Q is the first half, G the second
    q1, g1 = oracle.split_qg(y, 4)
    assert q1.tolist() == [[10, 11, 20, 21]] and g1.tolist() == [[12, 13, 22, 23]]


def test_split_qg_is_a_per_row_permutation_inverted_by_interleaving():
    rng = np.random.default_rng(5)
    B, heads, hd = 3, 5, 8
    y = rng.standard_normal((B, 2 * heads * hd))
    q, g = oracle.split_qg(y, hd)
    # re-interleave by a different route: stack per head and flatten
    back = np.stack([q.reshape(B, heads, hd), g.reshape(B, heads, hd)], axis=2).reshape(B, -1)
    assert np.array_equal(back, y)
    for b in range(B):
        assert np.array_equal(np.sort(np.concatenate([q[b], g[b]])), np.sort(y[b]))


def test_split_qg_rejects_rows_that_are_not_whole_heads():
    with pytest.raises(Exception):
        oracle.split_qg(np.zeros((1, 12)), 4)


# --- W4A16 prefill ------------------------------------------------------------------

def _fp16_midpoints():
    """Every finite positive binary16 value, the midpoints between neighbours
    (exact in fp32) and the fp32 values one ulp either side of each midpoint."""
    pats = np.arange(0x7C00, dtype=np.uint16)
    vals = pats.view(np.float16).astype(np.float32)
    mids = ((vals[:-1].astype(np.float64) + vals[1:].astype(np.float64)) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (vals[:-1].astype(np.float64) + vals[1:]) / 2)
    up = np.nextafter(mids, np.float32(np.inf))
    down = np.nextafter(mids, np.float32(0))
    return np.concatenate([vals, mids, up, down, np.float32([65504, 65519.996, 65520, 65536, 1e30])])


def test_fp16_rounding_matches_numpy_on_values_midpoints_and_random_floats():
    rng = np.random.default_rng(11)
    rnd = (rng.standard_normal(400000) * np.exp2(rng.integers(-30, 18, 400000))).astype(np.float32)
    f = np.concatenate([_fp16_midpoints(), rnd, np.float32([0.0, np.inf, np.nan])])
    f = np.concatenate([f, -f])
    got = oracle.float_to_fp16(f)
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    nan = np.isnan(f)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.all((got[nan] & 0x7C00) == 0x7C00) and np.all((got[nan] & 0x3FF) != 0)


def test_fp16_rounding_hand_worked_ties():
    # 1 + 2^-11 is half-way between 1 and 1 + 2^-10: ties to the even significand (1.0);
    # 1 + 3*2^-11 is half-way between 1 + 2^-10 and 1 + 2^-9: ties up to 1 + 2^-9.
    one = 0x3C00
    got = oracle.float_to_fp16(np.float32([1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2.0 ** -25,
                                           3 * 2.0 ** -25, 65519.0, 65520.0]))
    assert list(got) == [one, one + 2, 0x0000, 0x0002, 0x7BFF, 0x7C00]


def test_q4k_dequant_f16_is_the_fp32_weight_rounded_to_binary16():
    rng = np.random.default_rng(12)
    N, K = 5, 768
    w = synth.q4k_matrix(rng, N, K)
    got = oracle.q4k_dequant_f16(w, N, K)
    ref = oracle.q4k_dequant_f32(w, N, K).astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)
    soa = oracle.q4k_repack_soa(w, N, K)
    assert np.array_equal(oracle.q4k_dequant_f16(soa, N, K, layout="soa"), got)


def test_q4k_prefill_hand_worked_weight_rounding():
    # d = 1 + 2^-10 (0x3C01), scale 63, q 15, min 0: w = 945 * (1 + 2^-10) = 945.9228515625,
    # exact in fp32; binary16 spacing in [512, 1024) is 0.5, so W16 = 946.  With x = 1 at
    # that weight and 0 elsewhere the prefill result is 946 (the exact GEMV gives 945.92...).
    blk = np.zeros(144, np.uint8)
    blk[0:2] = [0x01, 0x3C]
    blk[4] = 63                              # sub-block 0: scale 63, min 0
    blk[16] = 0x0F                           # weight 0: q = 15
    w = blk.reshape(1, 144)
    x16 = np.zeros((1, 256), np.float16)
    x16[0, 0] = 1.0
    y, a = oracle.q4k_prefill(w, 1, 256, x16)
    assert y[0, 0] == 946.0 and a[0, 0] == 946.0
    yg, _ = oracle.q4k_gemv(w, 1, 256, x16.astype(np.float32))
    assert yg[0, 0] == 945.9228515625


@pytest.mark.parametrize("N,K,M", [(8, 256, 1), (3, 512, 5), (4, 768, 17)])
def test_q4k_prefill_matches_dense_brute_force(N, K, M):
    rng = np.random.default_rng(N * 100 + K + M)
    w = synth.q4k_matrix(rng, N, K)
    x16 = synth.activations_f16(rng, M, K)
    w16 = oracle.q4k_dequant_f16(w, N, K).view(np.float16).astype(np.float64)
    xd = x16.astype(np.float64)
    y, a = oracle.q4k_prefill(w, N, K, x16)
    assert y.shape == (M, N)
    assert np.allclose(y, xd @ w16.T, rtol=1e-13, atol=1e-13)
    assert np.allclose(a, np.abs(xd) @ np.abs(w16).T, rtol=1e-13, atol=1e-13)
    rows = np.array([N - 1, 0])
    ys, as_ = oracle.q4k_prefill(w, N, K, x16, rows=rows)
    assert np.array_equal(ys, y[:, rows]) and np.array_equal(as_, a[:, rows])
    soa = oracle.q4k_repack_soa(w, N, K)
    assert np.array_equal(oracle.q4k_prefill(soa, N, K, x16, layout="soa")[0], y)


def test_q4k_prefill_equals_the_gemv_when_weights_and_x_are_binary16_exact():
    # d = 1, scale 1, min 0: every weight is its quant (exact in binary16); x is binary16, so
    # the prefill and the fp32-input GEMV compute the same exact products.
    N, K, M = 3, 512, 4
    rng = np.random.default_rng(13)
    nblk = N * K // 256
    sc = np.array([1, 1, 1, 1, 0, 0, 0, 0, 1, 1, 1, 1], np.uint8)
    w = synth.q4k_pack(np.ones(nblk, np.float16), np.zeros(nblk, np.float16),
                       np.tile(sc, (nblk, 1)),
                       rng.integers(0, 256, (nblk, 128), dtype=np.uint8)).reshape(N, -1)
    x16 = synth.activations_f16(rng, M, K)
    y, _ = oracle.q4k_prefill(w, N, K, x16)
    yg, _ = oracle.q4k_gemv(w, N, K, x16.astype(np.float32))
    assert np.array_equal(y, yg)


def test_q8_0_fp32_dequant_is_exact_for_every_scale_and_quant():
    # d has 11 significant bits and q 8, so d*q (<= 19 bits, exponent within
    # fp32's range) is exact in fp32: the fp32 dequant must equal the exact one
    # for every fp16 scale pattern (finite) against the extreme quants
    d_bits = np.arange(0, 0x7C00, dtype=np.uint16)           # every finite non-negative fp16
    d_bits = np.concatenate([d_bits, d_bits | 0x8000])
    q = np.array([-128, -127, -1, 0, 1, 127], np.int8)
    blocks = np.zeros((d_bits.size, 34), np.uint8)
    blocks[:, 0:2] = d_bits.view(np.uint8).reshape(-1, 2)
    blocks[:, 2:] = np.resize(q.view(np.uint8), 32)
    N = d_bits.size
    exact = oracle.q8_0_dequant(blocks, N, 32)
    f32 = oracle.q8_0_dequant_f32(blocks, N, 32)
    assert np.array_equal(f32.astype(np.float64), exact)
    d = d_bits.view(np.float16).astype(np.float64)
    assert np.array_equal(exact, d[:, None] * np.resize(q.astype(np.float64), 32)[None, :])
