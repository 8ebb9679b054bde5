"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bars (from the method's definition):
  * dequantized weights and the SoA repack: bit-exact;
  * GEMV outputs: |y_gpu - y_ref| <= 1e-4 * sum_k |w_nk x_k| + 1e-6, with y_ref
    and the sum accumulated in double over the exact weights;
  * SwiGLU: the GEMV bound propagated through silu (oracle.swiglu_tolerance);
  * argmax: exactly the oracle's index (lowest index on ties), asserted only
    when the oracle's top-2 margin exceeds the two logits' tolerances.
Inputs are the seeded synthetic workloads (dequant_gemv_q4_b200.synth).
"""

import concurrent.futures
import os

import numpy as np
import pytest

import oracle
from dequant_gemv_q4_b200 import synth

torch = pytest.importorskip("torch")
import dequant_gemv_q4_b200 as dq  # noqa: E402

pytestmark = pytest.mark.gpu

THREADS = max(1, min(16, os.cpu_count() or 1))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    dq.load_library()
    yield
    assert dq.dq_device_error(clear=True) == 0


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def oracle_rows(fn, N, rows, **kw):
    """Run an oracle GEMV over `rows` in THREADS threads (ctypes drops the GIL)."""
    rows = np.asarray(rows, dtype=np.int64)
    parts = np.array_split(rows, THREADS)
    with concurrent.futures.ThreadPoolExecutor(THREADS) as ex:
        res = list(ex.map(lambda r: fn(rows=r, **kw), [p for p in parts if p.size]))
    return np.concatenate([r[0] for r in res], axis=1), np.concatenate([r[1] for r in res], axis=1)


def assert_within(y_gpu, y_ref, a_ref, what=""):
    y_gpu = np.asarray(y_gpu, dtype=np.float64).reshape(y_ref.shape)
    err = np.abs(y_gpu - y_ref)
    tol = oracle.gemv_tolerance(a_ref)
    ratio = err / tol
    assert np.all(np.isfinite(y_gpu)), what + ": non-finite output"
    assert ratio.max() <= 1.0, "%s: %d of %d outputs out of tolerance, worst err/tol %.3g" % (
        what, int((ratio > 1).sum()), ratio.size, ratio.max())


# --- dequantization and repack: bit-exact -----------------------------------------------

@pytest.mark.parametrize("N,K,seed", [(4096, 1024, 1), (37, 5120, 11), (5, 256, 12), (3, 12288, 13)])
@pytest.mark.parametrize("layout", ["aos", "soa"])
def test_q4k_dequant_bit_exact(N, K, seed, layout):
    w = synth.q4k_matrix(np.random.default_rng(seed), N, K)
    if layout == "soa":
        w = oracle.q4k_repack_soa(w, N, K)
    want = oracle.q4k_dequant_f32(w, N, K, layout=layout)
    got = host(dq.q4k_dequant(dev(w), N, K, layout=layout))
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_q4k_dequant_row_slice_of_lm_head_rows():
    # rows are independent: a row slice is a pointer offset (here: rows 1000..1063)
    N, K = 2048, 4096
    w = synth.q4k_matrix(np.random.default_rng(4), N, K)
    wd = dev(w)
    row_bytes = K // 256 * 144
    sl = wd.view(-1)[1000 * row_bytes:1064 * row_bytes]
    got = host(dq.q4k_dequant(sl, 64, K))
    want = oracle.q4k_dequant_f32(w[1000:1064], 64, K)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_q4k_dequant_handworked_special_blocks():
    # zero quants (w = -dmin*min), q=15/scale=63/min=0 (945*d), subnormal d and dmin
    blocks = [
        synth.q4k_pack([1.0], [0.25], [np.array([1, 2, 3, 4, 5, 6, 7, 8, 0, 0, 0, 0], np.uint8)],
                       [np.zeros(128, np.uint8)]),
        synth.q4k_pack([0.5], [1.0], [np.array([255] * 4 + [0] * 4 + [15] * 4, np.uint8)],
                       [np.full(128, 255, np.uint8)]),
        synth.q4k_pack(np.array([1], np.uint16).view(np.float16), np.array([512], np.uint16).view(np.float16),
                       [np.full(12, 255, np.uint8)], [np.full(128, 15, np.uint8)]),
    ]
    w = np.concatenate(blocks).reshape(3, 144)
    got = host(dq.q4k_dequant(dev(w), 3, 256))
    want = oracle.q4k_dequant_f32(w, 3, 256)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert np.all(got[1] == np.float32(945 * 0.5))


@pytest.mark.parametrize("N,K,seed", [(1024, 1024, 0), (7, 96, 1), (3, 32, 2)])
def test_q8_0_dequant_bit_exact(N, K, seed):
    w = synth.q8_0_matrix(np.random.default_rng(seed), N, K)
    got = host(dq.q8_0_dequant(dev(w), N, K))
    want = oracle.q8_0_dequant_f32(w, N, K)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("N,K", [(4096, 1024), (3, 5120), (5, 256), (2, 12288)])
def test_repack_soa_bit_exact(N, K):
    w = synth.q4k_matrix(np.random.default_rng(N + K), N, K)
    got = host(dq.q4k_repack_soa(dev(w), N, K))
    assert np.array_equal(got, oracle.q4k_repack_soa(w, N, K))


# --- the five workloads -------------------------------------------------------------------

def test_q8_0_gemv_1024x1024():
    wl = synth.WORKLOADS["q8_0_gemv_1024x1024"]
    inp = synth.make_inputs(wl)
    y = host(dq.q8_0_gemv(dev(inp["w"]), dev(inp["x"]), wl.N, wl.K))
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q8_0_gemv(inp["w"], wl.N, wl.K, inp["x"], rows=rows),
                               wl.N, np.arange(wl.N))
    assert_within(y, y_ref, a_ref, "q8_0 1024x1024")


@pytest.mark.parametrize("layout", ["aos", "soa"])
def test_q4k_gemv_4096x1024(layout):
    wl = synth.WORKLOADS["q4k_gemv_4096x1024"]
    inp = synth.make_inputs(wl)
    w = inp["w"] if layout == "aos" else oracle.q4k_repack_soa(inp["w"], wl.N, wl.K)
    y = host(dq.q4k_gemv(dev(w), dev(inp["x"]), wl.N, wl.K, layout=layout))
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q4k_gemv(inp["w"], wl.N, wl.K, inp["x"], rows=rows),
                               wl.N, np.arange(wl.N))
    assert_within(y, y_ref, a_ref, "q4k 4096x1024 " + layout)


def test_q4k_swiglu_12288x4096():
    wl = synth.WORKLOADS["q4k_swiglu_12288x4096"]
    inp = synth.make_inputs(wl)
    out = host(dq.q4k_swiglu_gemv(dev(inp["w_gate"]), dev(inp["w_up"]), dev(inp["x"]), wl.N, wl.K))
    rows = np.arange(wl.N)
    g, ag = oracle_rows(lambda rows: oracle.q4k_gemv(inp["w_gate"], wl.N, wl.K, inp["x"], rows=rows), wl.N, rows)
    u, au = oracle_rows(lambda rows: oracle.q4k_gemv(inp["w_up"], wl.N, wl.K, inp["x"], rows=rows), wl.N, rows)
    ref = oracle.swiglu(g, u)
    tol = oracle.swiglu_tolerance(g, u, ag, au)
    err = np.abs(out.reshape(ref.shape).astype(np.float64) - ref)
    assert np.all(err <= tol), "worst err/tol %.3g" % (err / tol).max()


@pytest.mark.parametrize("B", [1, 2, 4, 8])
def test_q4k_down_4096x12288(B):
    wl = synth.WORKLOADS["q4k_down_4096x12288"]
    inp = synth.make_inputs(wl, B=B)
    y = host(dq.q4k_gemv(dev(inp["w"]), dev(inp["x"]), wl.N, wl.K))
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q4k_gemv(inp["w"], wl.N, wl.K, inp["x"], rows=rows),
                               wl.N, np.arange(wl.N))
    assert_within(y, y_ref, a_ref, "q4k down B=%d" % B)


def test_q4k_lm_head_248320x4096_with_argmax():
    wl = synth.WORKLOADS["q4k_lmhead_248320x4096"]
    inp = synth.make_inputs(wl)
    y, idx = dq.q4k_gemv(dev(inp["w"]), dev(inp["x"]), wl.N, wl.K, argmax=True)
    y = host(y)[0]
    idx = int(host(idx)[0])
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q4k_gemv(inp["w"], wl.N, wl.K, inp["x"], rows=rows),
                               wl.N, np.arange(wl.N))
    y_ref, a_ref = y_ref[0], a_ref[0]
    assert_within(y, y_ref, a_ref, "lm head")
    want = oracle.argmax(y_ref)
    order = np.argsort(-y_ref, kind="stable")
    first, second = order[0], order[1]
    tol = oracle.gemv_tolerance(a_ref)
    margin = y_ref[first] - y_ref[second]
    assert margin > tol[first] + tol[second], "ambiguous argmax: top-2 margin within tolerance"
    assert idx == want
    assert idx == int(np.argmax(y))   # and consistent with the logits it returned


# --- edge cases -----------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,B", [(1, 256, 1), (5, 256, 3), (17, 1024, 1), (4097, 1024, 2), (33, 5120, 1),
                                   (9, 12288, 5), (130, 4096, 7), (3, 768, 8), (64, 65536, 1), (16, 262144, 2),
                                   # K split unevenly (2 + 1 chunks) inside clusters of two CTAs
                                   (9728, 2560, 1)])
@pytest.mark.parametrize("layout", ["aos", "soa"])
def test_q4k_gemv_ragged_and_split_shapes(N, K, B, layout):
    rng = np.random.default_rng(N * 7 + K + B)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, B, K)
    wl = w if layout == "aos" else oracle.q4k_repack_soa(w, N, K)
    y = host(dq.q4k_gemv(dev(wl), dev(x), N, K, layout=layout))
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q4k_gemv(w, N, K, x, rows=rows), N, np.arange(N))
    assert_within(y, y_ref, a_ref, "N=%d K=%d B=%d %s" % (N, K, B, layout))


@pytest.mark.parametrize("N,K,B", [(7, 256, 1), (100, 4096, 3), (24, 65536, 1), (1, 1024, 8)])
def test_q4k_swiglu_ragged_and_split_shapes(N, K, B):
    rng = np.random.default_rng(N + K + B)
    wg = synth.q4k_matrix(rng, N, K)
    wu = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, B, K)
    out = host(dq.q4k_swiglu_gemv(dev(wg), dev(wu), dev(x), N, K))
    g, ag = oracle.q4k_gemv(wg, N, K, x)
    u, au = oracle.q4k_gemv(wu, N, K, x)
    ref = oracle.swiglu(g, u)
    tol = oracle.swiglu_tolerance(g, u, ag, au)
    assert np.all(np.abs(out.reshape(ref.shape) - ref) <= tol)


@pytest.mark.parametrize("N,K,B", [(5, 32, 1), (33, 96, 2), (300, 4096, 4), (7, 8192, 8), (1, 64, 3)])
def test_q8_0_gemv_ragged_shapes(N, K, B):
    rng = np.random.default_rng(N + K + B)
    w = synth.q8_0_matrix(rng, N, K)
    x = synth.activations(rng, B, K)
    y = host(dq.q8_0_gemv(dev(w), dev(x), N, K))
    y_ref, a_ref = oracle.q8_0_gemv(w, N, K, x)
    assert_within(y, y_ref, a_ref, "q8_0 N=%d K=%d B=%d" % (N, K, B))


def _unit_matrix(N, nb, q_byte, m_val=0, dmin=0.0):
    sc = np.array([1, 1, 1, 1, m_val, m_val, m_val, m_val] + [1 | (m_val << 4)] * 4, np.uint8)
    n = N * nb
    return synth.q4k_pack(np.ones(n, np.float16), np.full(n, dmin, np.float16), np.tile(sc, (n, 1)),
                          np.full((n, 128), q_byte, np.uint8)).reshape(N, -1)


@pytest.mark.parametrize("K", [256, 4096, 12288])
def test_exact_integer_case_is_bit_exact(K):
    # d=1, scale=1, min=0: integer weights q in [0,15]; small integer x keep
    # every partial sum an integer below 2^24, so fp32 must equal the exact sum.
    rng = np.random.default_rng(K)
    N = 50
    nblk = N * K // 256
    sc = np.tile(np.array([1, 1, 1, 1, 0, 0, 0, 0, 1, 1, 1, 1], np.uint8), (nblk, 1))
    w = synth.q4k_pack(np.ones(nblk, np.float16), np.zeros(nblk, np.float16), sc,
                       rng.integers(0, 256, (nblk, 128), dtype=np.uint8)).reshape(N, -1)
    x = rng.integers(-3, 4, (2, K)).astype(np.float32)
    y = host(dq.q4k_gemv(dev(w), dev(x), N, K))
    y_ref, _ = oracle.q4k_gemv(w, N, K, x)
    assert np.array_equal(y.astype(np.float64), y_ref)


def test_zero_quants_and_cancelling_weights():
    K, N = 4096, 40
    x = synth.activations(np.random.default_rng(9), 1, K)
    # all quants 0, min 3, dmin 0.5: every weight is -1.5
    w0 = _unit_matrix(N, K // 256, 0x00, m_val=3, dmin=0.5)
    y0 = host(dq.q4k_gemv(dev(w0), dev(x), N, K))
    y_ref, a_ref = oracle.q4k_gemv(w0, N, K, x)
    assert_within(y0, y_ref, a_ref, "zero quants")
    # q=1, scale=1, d=1, min=1, dmin=1: every weight is exactly 0, so y must be exactly 0
    wz = _unit_matrix(N, K // 256, 0x11, m_val=1, dmin=1.0)
    yz = host(dq.q4k_gemv(dev(wz), dev(x), N, K))
    assert np.all(yz == 0.0)


def test_argmax_ties_take_the_lowest_index():
    N, K = 5000, 1024
    rng = np.random.default_rng(21)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 1, K)
    y_ref, _ = oracle.q4k_gemv(w, N, K, x)
    top = int(np.argmax(y_ref[0]))
    # copy the winning row to a lower and a higher index: three equal maxima
    lo, hi = top // 2, min(N - 1, top + 1234)
    w2 = w.copy()
    w2[lo] = w[top]
    w2[hi] = w[top]
    y, idx = dq.q4k_gemv(dev(w2), dev(x), N, K, argmax=True)
    y = host(y)[0]
    assert y[lo] == y[top] == y[hi]
    assert int(host(idx)[0]) == lo == oracle.argmax(oracle.q4k_gemv(w2, N, K, x)[0][0])
    # all rows identical: index 0
    w3 = np.tile(w[top], (N, 1))
    _, idx3 = dq.q4k_gemv(dev(w3), dev(x), N, K, argmax=True)
    assert int(host(idx3)[0]) == 0


def test_argmax_through_split_k():
    # few rows, long K: the plan splits K and the argmax runs in the reduction
    N, K = 40, 131072
    rng = np.random.default_rng(31)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 1, K)
    y, idx = dq.q4k_gemv(dev(w), dev(x), N, K, argmax=True)
    y_ref, a_ref = oracle.q4k_gemv(w, N, K, x)
    assert_within(host(y), y_ref, a_ref, "split-K argmax")
    assert int(host(idx)[0]) == oracle.argmax(y_ref[0])


def test_soa_and_aos_outputs_are_bitwise_equal():
    N, K = 1000, 12288
    rng = np.random.default_rng(41)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 2, K)
    wd = dev(w)
    y_aos = host(dq.q4k_gemv(wd, dev(x), N, K))
    y_soa = host(dq.q4k_gemv(dq.q4k_repack_soa(wd, N, K), dev(x), N, K, layout="soa"))
    assert np.array_equal(y_aos.view(np.uint32), y_soa.view(np.uint32))


def test_errors_launch_nothing_and_leave_the_stream_usable():
    lib = dq.load_library()
    N, K = 64, 1024
    w = dev(synth.q4k_matrix(np.random.default_rng(1), N, K))
    x = dev(synth.activations(np.random.default_rng(2), 1, K))
    y = torch.full((N,), 12345.0, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    import ctypes
    vp = ctypes.c_void_p
    # K not a multiple of 256, B out of range, misaligned x, bad layout, missing workspace
    assert lib.q4k_gemv(vp(w.data_ptr()), 0, vp(x.data_ptr()), vp(y.data_ptr()), N, K + 8, 1, None, None, 0, vp(s)) == 2
    assert lib.q4k_gemv(vp(w.data_ptr()), 0, vp(x.data_ptr()), vp(y.data_ptr()), N, K, 9, None, None, 0, vp(s)) == 2
    assert lib.q4k_gemv(vp(w.data_ptr()), 0, vp(x.data_ptr() + 4), vp(y.data_ptr()), N, K, 1, None, None, 0, vp(s)) == 3
    assert lib.q4k_gemv(vp(w.data_ptr()), 3, vp(x.data_ptr()), vp(y.data_ptr()), N, K, 1, None, None, 0, vp(s)) == 5
    idx = torch.zeros(1, dtype=torch.int64, device="cuda")
    assert lib.q4k_gemv(vp(w.data_ptr()), 0, vp(x.data_ptr()), vp(y.data_ptr()), N, K, 1, vp(idx.data_ptr()),
                        None, 0, vp(s)) == 4
    torch.cuda.synchronize()
    assert torch.all(y == 12345.0).item()          # nothing was written
    y2 = dq.q4k_gemv(w, x, N, K)                     # a valid call still works
    torch.cuda.synchronize()
    assert torch.isfinite(y2).all().item()


@pytest.mark.parametrize("N,K", [(40000, 4096), (16000, 12288)])
@pytest.mark.parametrize("layout", ["aos", "soa"])
def test_q4k_gemv_long_matrices(N, K, layout):
    # enough rows that batch 1 runs without K splits, several tiles per warp
    # (the LM-head plan); the smaller shapes above split K
    rng = np.random.default_rng(N + K)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 1, K)
    wl = w if layout == "aos" else oracle.q4k_repack_soa(w, N, K)
    y = host(dq.q4k_gemv(dev(wl), dev(x), N, K, layout=layout))
    rows = np.unique(np.concatenate([np.arange(0, N, 7), [N - 1]]))
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q4k_gemv(w, N, K, x, rows=rows), N, rows)
    assert_within(y[:, rows], y_ref, a_ref, "N=%d K=%d %s" % (N, K, layout))


# --- the batch-1 fixed-point path: its own error bound, special values, copy paths ------

def _fx_bound(wd, x):
    """The batch-1 kernel's own rounding bound: sum over super-blocks of
    2^(e_sb - F_bits) * sum |w|, e_sb the exponent of the block's largest |x|
    (2^e <= max < 2^(e+1)); F_bits is 22 for blocks whose largest |x| is at most
    6 times their rms (three limbs) and 30 otherwise (four limbs)."""
    N, K = wd.shape
    xb = np.abs(x.astype(np.float64)).reshape(K // 256, 256)
    mx = xb.max(axis=1)
    rms = np.sqrt((xb ** 2).mean(axis=1))
    bits = np.where(mx <= 6 * rms, 22, 30)
    _, E = np.frexp(mx)
    unit = np.where(mx > 0, np.ldexp(1.0, E - 1 - bits), 0.0)
    wsum = np.abs(wd.astype(np.float64)).reshape(N, K // 256, 256).sum(axis=2)
    return wsum @ unit


def test_fixed_point_activations_within_their_stated_bound():
    # wide dynamic range inside super-blocks: outliers, tiny values, a zero block,
    # subnormals; the result must stay within the kernel's own rounding bound
    # and within the GEMV contract
    N, K = 640, 4096
    rng = np.random.default_rng(31)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 1, K)[0].astype(np.float32)
    x[7] = 3.0e4
    x[300] = -1.0e4
    x[1000:1010] = 1e-7
    x[2 * 256:3 * 256] = 0.0
    x[5 * 256:6 * 256] *= np.float32(1e-40)          # subnormal activations
    y = host(dq.q4k_gemv(dev(w), dev(x[None, :]), N, K))[0].astype(np.float64)
    y_ref, a_ref = oracle.q4k_gemv(w, N, K, x[None, :])
    y_ref = y_ref[0]
    wd = oracle.q4k_dequant(w, N, K)
    bound = _fx_bound(wd, x) + 2.0 ** -24 * np.abs(y_ref) + 1e-30
    err = np.abs(y - y_ref)
    assert np.all(np.isfinite(y))
    assert np.all(err <= bound), "worst err/bound %.3g" % (err / bound).max()
    assert_within(y[None, :], y_ref[None, :], a_ref, "wide-range x")


@pytest.mark.parametrize("scale", [1e-30, 1e30, 1e34])
def test_extreme_activation_scales(scale):
    # the per-super-block exponent covers the fp32 range: the contract holds as is
    N, K = 256, 2048
    rng = np.random.default_rng(34)
    w = synth.q4k_matrix(rng, N, K)
    x = (synth.activations(rng, 1, K) * np.float32(scale)).astype(np.float32)
    y = host(dq.q4k_gemv(dev(w), dev(x), N, K))
    y_ref, a_ref = oracle.q4k_gemv(w, N, K, x)
    assert_within(y, y_ref, a_ref, "x scaled by %g" % scale)


@pytest.mark.parametrize("bad", [np.inf, -np.inf, np.nan])
def test_non_finite_activations_give_nan_rows(bad):
    N, K = 64, 1024
    rng = np.random.default_rng(32)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 1, K)
    x[0, 300] = bad
    y = host(dq.q4k_gemv(dev(w), dev(x), N, K))
    assert np.all(np.isnan(y))


def test_per_row_copy_path_is_bitwise_equal_to_tma():
    # DQGEMV_NO_TMA=1 moves the same slots with one bulk copy per row
    import subprocess
    import sys
    N, K = 1000, 5120
    rng = np.random.default_rng(33)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 1, K)
    y_tma = host(dq.q4k_gemv(dev(w), dev(x), N, K))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import sys, numpy as np, torch\n"
        "sys.path.insert(0, %r)\n"
        "import dequant_gemv_q4_b200 as dq\n"
        "from dequant_gemv_q4_b200 import synth\n"
        "rng = np.random.default_rng(33)\n"
        "w = synth.q4k_matrix(rng, %d, %d); x = synth.activations(rng, 1, %d)\n"
        "y = dq.q4k_gemv(torch.from_numpy(w).cuda(), torch.from_numpy(x).cuda(), %d, %d)\n"
        "torch.cuda.synchronize(); sys.stdout.buffer.write(y.cpu().numpy().tobytes())\n"
    ) % (root, N, K, K, N, K)
    env = dict(os.environ, DQGEMV_NO_TMA="1")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, timeout=300)
    assert out.returncode == 0, out.stderr.decode()[-2000:]
    y_rows = np.frombuffer(out.stdout, dtype=np.float32).reshape(1, N)
    assert np.array_equal(y_rows.view(np.uint32), y_tma.view(np.uint32))


# --- fused Q/gate de-interleave (Doppler split_qg.wgsl) ---------------------------------

@pytest.mark.parametrize("N,K,B,hd,layout", [
    (4096, 1024, 1, 128, "aos"),     # the q-projection-with-gate workload, 16 heads of 128
    (4096, 1024, 1, 128, "soa"),
    (512, 12288, 1, 64, "aos"),      # K splits (reduced in a CTA cluster)
    (1040, 4096, 3, 8, "aos"),       # batch 3: the fp32 kernel
    (200, 65536, 2, 50, "aos"),      # many K splits, a second-kernel reduction
])
def test_q4k_gemv_split_qg_is_the_plain_gemv_deinterleaved(N, K, B, hd, layout):
    rng = np.random.default_rng(N + K + B)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, B, K)
    wl = w if layout == "aos" else oracle.q4k_repack_soa(w, N, K)
    wd, xd = dev(wl), dev(x)
    y = host(dq.q4k_gemv(wd, xd, N, K, layout=layout))
    q, g = dq.q4k_gemv_split_qg(wd, xd, N, K, hd, layout=layout)
    q, g = host(q), host(g)
    q_ref, g_ref = oracle.split_qg(y.astype(np.float64), hd)
    # the same arithmetic, only stored in the split order
    assert np.array_equal(q.astype(np.float64), q_ref) and np.array_equal(g.astype(np.float64), g_ref)
    # and against the oracle's exact GEMV, split by the oracle
    y_ref, a_ref = oracle.q4k_gemv(w, N, K, x)
    tq, tg = oracle.split_qg(oracle.gemv_tolerance(a_ref), hd)
    yq, yg = oracle.split_qg(y_ref, hd)
    assert np.all(np.abs(q - yq) <= tq) and np.all(np.abs(g - yg) <= tg)


# --- capture of a decode step's GEMV sequence in a CUDA graph ---------------------------

def test_ffn_and_qproj_sequence_replays_from_a_cuda_graph():
    # q-projection with the Q/gate split, then the FFN: SwiGLU (gate/up 12288 x 4096)
    # feeding the down projection (4096 x 12288); captured once, replayed twice
    rng = np.random.default_rng(41)
    H, F, NQ, KQ = 4096, 12288, 4096, 1024
    wq = synth.q4k_matrix(rng, NQ, KQ)
    wg = synth.q4k_matrix(rng, F, H)
    wu = synth.q4k_matrix(rng, F, H)
    wdn = synth.q4k_matrix(rng, H, F)
    xq = dev(synth.activations(rng, 1, KQ))
    x = dev(synth.activations(rng, 1, H))
    dwq, dwg, dwu, dwd = dev(wq), dev(wg), dev(wu), dev(wdn)
    q = torch.empty((1, NQ // 2), device="cuda")
    gq = torch.empty((1, NQ // 2), device="cuda")
    h = torch.empty((1, F), device="cuda")
    out = torch.empty((1, H), device="cuda")
    wsz = max(dq.dq_workspace_bytes(dq.DQ_OP_Q4K_GEMV, NQ, KQ, 1), dq.dq_workspace_bytes(dq.DQ_OP_Q4K_SWIGLU, F, H, 1),
              dq.dq_workspace_bytes(dq.DQ_OP_Q4K_GEMV, H, F, 1), 16)
    ws = torch.empty(wsz, dtype=torch.uint8, device="cuda")

    def step():
        dq.q4k_gemv_split_qg(dwq, xq, NQ, KQ, 128, q=q, g=gq, workspace=ws)
        dq.q4k_swiglu_gemv(dwg, dwu, x, F, H, out=h, workspace=ws)
        dq.q4k_gemv(dwd, h, H, F, y=out, workspace=ws)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step()                                  # warm-up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step()
    for tensor in (q, gq, h, out):
        tensor.fill_(float("nan"))
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    qv, gv, hv, ov = host(q), host(gq), host(h), host(out)

    yq_ref, aq = oracle.q4k_gemv(wq, NQ, KQ, host(xq))
    qr, gr = oracle.split_qg(yq_ref, 128)
    tq, tg = oracle.split_qg(oracle.gemv_tolerance(aq), 128)
    assert np.all(np.abs(qv - qr) <= tq) and np.all(np.abs(gv - gr) <= tg)
    xh = host(x)
    g_ref, a_g = oracle_rows(lambda rows: oracle.q4k_gemv(wg, F, H, xh, rows=rows), F, np.arange(F))
    u_ref, a_u = oracle_rows(lambda rows: oracle.q4k_gemv(wu, F, H, xh, rows=rows), F, np.arange(F))
    assert np.all(np.abs(hv - oracle.swiglu(g_ref, u_ref)) <= oracle.swiglu_tolerance(g_ref, u_ref, a_g, a_u))
    # the down projection of the GPU's own SwiGLU output
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q4k_gemv(wdn, H, F, hv, rows=rows), H, np.arange(H))
    assert_within(ov, y_ref, a_ref, "down projection replayed from the graph")


# --- grouped batch-1 GEMV (QKV-style projections in one launch) --------------------------

@pytest.mark.parametrize("Ns,K,layout", [
    ((4096, 1024, 1024), 4096, "aos"),   # Q, K, V of a hidden-4096 layer with 8 KV heads of 128
    ((4096, 1024, 1024), 4096, "soa"),
    ((1000, 24, 7, 333), 5120, "aos"),   # ragged row counts, four matrices
    ((40, 72), 65536, "aos"),            # long K: split into many parts
    ((3000,), 1024, "aos"),              # a group of one
])
def test_q4k_gemv_group_matches_separate_oracle_gemvs(Ns, K, layout):
    rng = np.random.default_rng(sum(Ns) + K)
    ws = [synth.q4k_matrix(rng, n, K) for n in Ns]
    x = synth.activations(rng, 1, K)
    wls = ws if layout == "aos" else [oracle.q4k_repack_soa(w, n, K) for w, n in zip(ws, Ns)]
    ys = dq.q4k_gemv_group([dev(w) for w in wls], dev(x[0]), list(Ns), K, layout=layout)
    for m, (w, n) in enumerate(zip(ws, Ns)):
        y = host(ys[m])
        y_ref, a_ref = oracle.q4k_gemv(w, n, K, x)
        assert_within(y[None, :], y_ref, a_ref, "group matrix %d" % m)


# --- W4A16 prefill on the tensor cores ---------------------------------------------------
# y = x16 W16^T, W16 the binary16 rounding of the fp32 weights; bar: the GEMV rule against the
# oracle's double sum over the same binary16 operands.

@pytest.mark.parametrize("N,K,M,layout", [
    (128, 256, 1, "aos"),      # one tile, one token (16-column MMA, 15 padding columns)
    (200, 512, 5, "aos"),      # ragged rows (128 + 72)
    (200, 512, 5, "soa"),
    (300, 1024, 33, "aos"),    # ragged tokens (T = 48)
    (256, 768, 130, "soa"),    # SoA rows of 3 blocks: the partial group only
    (130, 1280, 64, "soa"),    # SoA rows of 5 blocks: a full group and a partial one
    (384, 512, 700, "aos"),    # three token tiles of 240
    (1000, 2048, 256, "aos"),  # eight row tiles, K split in two
    (64, 4096, 17, "aos"),     # one tile, K split sixteen ways
])
def test_q4k_prefill_matches_oracle(N, K, M, layout):
    rng = np.random.default_rng(N + K + M)
    w = synth.q4k_matrix(rng, N, K)
    x16 = synth.activations_f16(rng, M, K)
    wl = w if layout == "aos" else oracle.q4k_repack_soa(w, N, K)
    y = host(dq.q4k_prefill_gemm(dev(wl), dev(x16), N, K, layout=layout))
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q4k_prefill(w, N, K, x16, rows=rows), N, np.arange(N))
    assert_within(y, y_ref, a_ref, "prefill %dx%d M=%d %s" % (N, K, M, layout))


@pytest.mark.parametrize("N,K", [(4096, 12288), (12288, 4096)])
def test_q4k_prefill_full_size_sampled_rows(N, K):
    # the down projection and one gate/up matrix at M = 128 tokens, in the launch
    # configuration bench.py times; the oracle computes 96 sampled rows
    M = 128
    rng = np.random.default_rng(N * 7 + K)
    w = synth.q4k_matrix(rng, N, K)
    x16 = synth.activations_f16(rng, M, K)
    y = host(dq.q4k_prefill_gemm(dev(w), dev(x16), N, K))
    rows = np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, 94)]))
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q4k_prefill(w, N, K, x16, rows=rows), N, rows)
    assert_within(y[:, rows], y_ref, a_ref, "prefill %dx%d sampled" % (N, K))


def test_q4k_prefill_exact_integer_case_is_bit_exact():
    # d = 1, scale 1, min 0: W16 = q in [0, 15]; x small integers: every partial sum is an
    # integer below 2^24, so the fp32 tensor-core sum is exact and must equal the oracle
    N, K, M = 256, 4096, 48
    nb = K // 256
    rng = np.random.default_rng(21)
    sc = np.array([1, 1, 1, 1, 0, 0, 0, 0, 1, 1, 1, 1], np.uint8)
    w = synth.q4k_pack(np.ones(N * nb, np.float16), np.zeros(N * nb, np.float16), np.tile(sc, (N * nb, 1)),
                       rng.integers(0, 256, (N * nb, 128), dtype=np.uint8)).reshape(N, -1)
    x16 = rng.integers(-3, 4, (M, K)).astype(np.float16)
    y = host(dq.q4k_prefill_gemm(dev(w), dev(x16), N, K))
    y_ref, _ = oracle.q4k_prefill(w, N, K, x16)
    assert np.array_equal(y.astype(np.float64), y_ref)


def test_q4k_prefill_is_deterministic_and_soa_equals_aos():
    N, K, M = 520, 4096, 96      # few tiles: K is split and the partials are reduced
    rng = np.random.default_rng(22)
    w = synth.q4k_matrix(rng, N, K)
    x16 = dev(synth.activations_f16(rng, M, K))
    assert dq.dq_workspace_bytes(dq.DQ_OP_Q4K_PREFILL, N, K, M) > 0
    y1 = host(dq.q4k_prefill_gemm(dev(w), x16, N, K))
    y2 = host(dq.q4k_prefill_gemm(dev(w), x16, N, K))
    y3 = host(dq.q4k_prefill_gemm(dev(oracle.q4k_repack_soa(w, N, K)), x16, N, K, layout="soa"))
    assert np.array_equal(y1.view(np.uint32), y2.view(np.uint32))
    assert np.array_equal(y1.view(np.uint32), y3.view(np.uint32))


# --- fused residual add (FFN block down projection) ----------------------------------------

@pytest.mark.parametrize("N,K,B,inplace", [
    (4096, 12288, 1, False),   # the down projection, K split in clusters
    (4096, 12288, 1, True),    # y += W x
    (1000, 4096, 3, False),    # batch 3
    (300, 65536, 1, True),     # long K: split-K reduction kernel
    (77, 1024, 2, True),
])
def test_q4k_gemv_residual_is_the_gemv_plus_the_residual(N, K, B, inplace):
    rng = np.random.default_rng(N + K + B)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, B, K)
    r = synth.activations(rng, B, N, scale=4.0)
    rd = dev(r)
    y = dq.q4k_gemv_residual(dev(w), dev(x), rd, N, K, y=rd if inplace else None)
    got = host(y).reshape(B, N).astype(np.float64)
    plain = host(dq.q4k_gemv(dev(w), dev(x), N, K)).reshape(B, N)
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q4k_gemv(w, N, K, x, rows=rows), N, np.arange(N))
    want = y_ref + r.astype(np.float64)
    # the GEMV rule, plus one fp32 rounding of the sum
    tol = oracle.gemv_tolerance(a_ref) + np.abs(want) * 2.0 ** -23
    assert np.all(np.abs(got - want) <= tol)
    # and exactly the fp32 sum of q4k_gemv's own output and the residual
    assert np.array_equal(got.astype(np.float32), (plain + r).astype(np.float32))


@pytest.mark.parametrize("H,F,B,mode", [
    (4096, 12288, 1, "residual_x"),   # the decode shape, y = x + FFN(x)
    (4096, 12288, 1, "inplace"),      # x = x + FFN(x) in place
    (1024, 4096, 3, "none"),          # batch 3, no residual
    (512, 1536, 2, "residual_x"),
    (2560, 9728, 1, "residual_x"),    # K not a multiple of the 1024-wide chunk
])
def test_q4k_ffn_block_matches_the_separate_calls_and_the_oracle(H, F, B, mode):
    rng = np.random.default_rng(H + F + B)
    wg, wu = synth.q4k_matrix(rng, F, H), synth.q4k_matrix(rng, F, H)
    wd = synth.q4k_matrix(rng, H, F)
    x = synth.activations(rng, B, H)
    dwg, dwu, dwd, dx = dev(wg), dev(wu), dev(wd), dev(x)
    # the separate calls
    h = dq.q4k_swiglu_gemv(dwg, dwu, dx, F, H)
    sep = host(dq.q4k_gemv_residual(dwd, h, dx, H, F) if mode != "none" else dq.q4k_gemv(dwd, h, H, F))
    ws = torch.empty(dq.dq_workspace_bytes(dq.DQ_OP_Q4K_FFN, H, F, B), dtype=torch.uint8, device="cuda")
    if mode == "inplace":
        xin = dev(x)
        y = dq.q4k_ffn_block(dwg, dwu, dwd, xin, H, F, residual=xin, y=xin, workspace=ws)
    else:
        y = dq.q4k_ffn_block(dwg, dwu, dwd, dx, H, F, residual=dx if mode == "residual_x" else None, workspace=ws)
    got = host(y).reshape(B, H)
    # h, the GPU's own SwiGLU output, is left at the start of the workspace
    hv = host(ws[:4 * B * F].view(torch.float32)).reshape(B, F)
    # two launches: exactly the separate calls
    assert np.array_equal(got.view(np.uint32), sep.reshape(B, H).view(np.uint32))
    # the oracle: SwiGLU within its bound, then the down projection of the GPU's own h
    g_ref, a_g = oracle_rows(lambda rows: oracle.q4k_gemv(wg, F, H, x, rows=rows), F, np.arange(F))
    u_ref, a_u = oracle_rows(lambda rows: oracle.q4k_gemv(wu, F, H, x, rows=rows), F, np.arange(F))
    assert np.all(np.abs(hv - oracle.swiglu(g_ref, u_ref)) <= oracle.swiglu_tolerance(g_ref, u_ref, a_g, a_u))
    y_ref, a_ref = oracle_rows(lambda rows: oracle.q4k_gemv(wd, H, F, hv, rows=rows), H, np.arange(H))
    want = y_ref + (x.astype(np.float64) if mode != "none" else 0.0)
    tol = oracle.gemv_tolerance(a_ref) + np.abs(want) * 2.0 ** -23
    assert np.all(np.abs(got - want) <= tol)
