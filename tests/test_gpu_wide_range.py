"""Batch-1 Q4_K GEMV on activations of any finite range, against the oracle.

The batch-1 kernels round each activation to a fixed point shared by its
super-block of 256.  Alongside every output row they carry an upper bound on
the error that rounding caused (the block's total rounding residue times the
largest weight magnitude the block's header allows) and a lower bound on
sum_k |w_k x_k| (the sum of the super-blocks' |partial sums|); a row whose
bound cannot show the contract |y - y_ref| <= 1e-4 * sum_k |w_nk x_k| + 1e-6
is recomputed exactly in fp64.  The result must meet the contract element by
element on every finite input.  The hard inputs are outliers that meet a
weight that is exactly 0 (q = 0 and min = 0): the rows holding that zero do not
see the outlier in their tolerance, but a fixed point scaled to the outlier
blurs every other activation of the block.  These tests put outliers of
1e6 .. 1e30 on such columns, spread huge ranges over whole blocks, and cover
every batch-1 output form: plain (both layouts), SwiGLU, K splits added in a
cluster and in the reduction kernel, grouped matrices, the fused Q/gate split
and argmax.
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
OUTLIERS = [1e6, -1e7, 1e20, -1e30]


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


def oracle_gemv(w, N, K, x):
    rows = np.arange(N, dtype=np.int64)
    parts = [p for p in np.array_split(rows, THREADS) if p.size]
    with concurrent.futures.ThreadPoolExecutor(THREADS) as ex:
        res = list(ex.map(lambda r: oracle.q4k_gemv(w, N, K, x, rows=r), parts))
    return np.concatenate([r[0] for r in res], axis=1), np.concatenate([r[1] for r in res], axis=1)


def assert_within(y_gpu, y_ref, a_ref, what=""):
    y_gpu = np.asarray(y_gpu, dtype=np.float64).reshape(y_ref.shape)
    assert np.all(np.isfinite(y_gpu)), what + ": non-finite output"
    ratio = np.abs(y_gpu - y_ref) / oracle.gemv_tolerance(a_ref)
    assert ratio.max() <= 1.0, "%s: %d of %d outputs out of tolerance, worst err/tol %.3g" % (
        what, int((ratio > 1).sum()), ratio.size, ratio.max())


def zero_weight_at(w, N, K, col, rows):
    """Make weight (n, col) exactly 0 for n in `rows`: its quant nibble and the
    min of its sub-block become 0 (GGML Q4_K bytes, get_scale_min_k4 packing)."""
    w = w.copy().reshape(N, K // 256, 144)
    kb, i = divmod(col, 256)
    c, r = divmod(i, 64)
    byte = 16 + 32 * c + r % 32
    j = i // 32
    for n in rows:
        blk = w[n, kb]
        blk[byte] &= 0xF0 if r < 32 else 0x0F
        s = blk[4:16]
        if j < 4:
            s[j + 4] &= 0xC0            # min j: low six bits of scale byte j + 4
        else:
            s[j + 4] &= 0x0F            # min j: high nibble of byte j + 4 ...
            s[j] &= 0x3F                # ... and bits 6..7 of byte j
    return w.reshape(N, -1)


def outlier_case(seed, N, K, cols, value, zero_rows=None):
    """Seeded matrix and x ~ N(0,1) with `value` at each column in `cols`; the
    weights of every other row (or of `zero_rows`) at those columns are 0."""
    rng = np.random.default_rng(seed)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 1, K)
    rows = np.arange(0, N, 2) if zero_rows is None else zero_rows
    for c in cols:
        w = zero_weight_at(w, N, K, c, rows)
        x[0, c] = np.float32(value)
    return w, x


def test_zero_weight_helper_zeroes_exactly_those_weights():
    N, K = 6, 512
    w = synth.q4k_matrix(np.random.default_rng(5), N, K)
    for col in (0, 31, 32, 63, 64, 200, 255, 256 + 130, 511):
        wz = zero_weight_at(w, N, K, col, [1, 4])
        d = oracle.q4k_dequant(wz, N, K)
        assert d[1, col] == 0.0 and d[4, col] == 0.0
        assert np.array_equal(d[[0, 2, 3, 5]], oracle.q4k_dequant(w, N, K)[[0, 2, 3, 5]])


def test_counterexample_64x256_outlier_on_the_most_zero_column():
    # a seeded 64 x 256 matrix; the outlier sits in the column holding the most
    # exactly-zero weights (q = 0 with min = 0)
    rng = np.random.default_rng(0)
    N, K = 64, 256
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 1, K)
    zeros = (oracle.q4k_dequant(w, N, K) == 0.0).sum(axis=0)
    col = int(np.argmax(zeros))
    assert zeros[col] >= 1
    for v in (1e6, 1e7, -1e7, 1e20, 1e30):
        xv = x.copy()
        xv[0, col] = np.float32(v)
        y = host(dq.q4k_gemv(dev(w), dev(xv), N, K))
        y_ref, a_ref = oracle.q4k_gemv(w, N, K, xv)
        assert_within(y, y_ref, a_ref, "64x256 outlier %g at column %d" % (v, col))


@pytest.mark.parametrize("value", OUTLIERS)
@pytest.mark.parametrize("layout", ["aos", "soa"])
def test_plain_gemv_outliers_on_zero_weights(value, layout):
    N, K = 1000, 4096
    w, x = outlier_case(11, N, K, [5, 700, 2049, 4095], value)
    wl = w if layout == "aos" else oracle.q4k_repack_soa(w, N, K)
    y = host(dq.q4k_gemv(dev(wl), dev(x), N, K, layout=layout))
    y_ref, a_ref = oracle_gemv(w, N, K, x)
    assert_within(y, y_ref, a_ref, "plain %g %s" % (value, layout))


@pytest.mark.parametrize("value", OUTLIERS)
def test_swiglu_outliers_on_zero_weights(value):
    N, K = 300, 4096
    cols = [17, 1500]
    wg, x = outlier_case(12, N, K, cols, value)
    wu, _ = outlier_case(13, N, K, cols, value)
    # silu(g) * u stays finite only where g is moderate: zero the outlier's
    # weights in every gate row, and in every other up row
    for c in cols:
        wg = zero_weight_at(wg, N, K, c, np.arange(N))
    out = host(dq.q4k_swiglu_gemv(dev(wg), dev(wu), dev(x), N, K))
    g, ag = oracle_gemv(wg, N, K, x)
    u, au = oracle_gemv(wu, N, K, x)
    ref = oracle.swiglu(g, u)
    tol = oracle.swiglu_tolerance(g, u, ag, au)
    err = np.abs(out.reshape(ref.shape).astype(np.float64) - ref)
    assert np.all(np.isfinite(out))
    assert np.all(err <= tol), "worst err/tol %.3g" % (err / tol).max()


@pytest.mark.parametrize("value", OUTLIERS)
def test_cluster_split_outliers_on_zero_weights(value):
    # the down-projection shape: K splits added inside CTA clusters
    N, K = 4096, 12288
    w, x = outlier_case(14, N, K, [3, 5000, 12287], value)
    y = host(dq.q4k_gemv(dev(w), dev(x), N, K))
    y_ref, a_ref = oracle_gemv(w, N, K, x)
    assert_within(y, y_ref, a_ref, "cluster split %g" % value)


@pytest.mark.parametrize("value", OUTLIERS)
def test_reduction_kernel_split_outliers_and_argmax(value):
    # few rows, long K: splits added by the reduction kernel, argmax there too
    N, K = 24, 65536
    w, x = outlier_case(15, N, K, [100, 40000], value)
    y, idx = dq.q4k_gemv(dev(w), dev(x), N, K, argmax=True)
    y = host(y)
    y_ref, a_ref = oracle.q4k_gemv(w, N, K, x)
    assert_within(y, y_ref, a_ref, "reduction split %g" % value)
    tol = oracle.gemv_tolerance(a_ref[0])
    order = np.argsort(-y_ref[0], kind="stable")
    if y_ref[0, order[0]] - y_ref[0, order[1]] > tol[order[0]] + tol[order[1]]:
        assert int(host(idx)[0]) == oracle.argmax(y_ref[0])


@pytest.mark.parametrize("value", OUTLIERS)
def test_group_and_split_qg_outliers_on_zero_weights(value):
    K = 4096
    cols = [9, 3000]
    Ns = [1000, 24, 7]
    mats = []
    for m, n in enumerate(Ns):
        wm, x = outlier_case(16 + m, n, K, cols, value)
        mats.append(wm)
    ys = dq.q4k_gemv_group([dev(m) for m in mats], dev(x[0]), Ns, K)
    for m, n in enumerate(Ns):
        y_ref, a_ref = oracle.q4k_gemv(mats[m], n, K, x)
        assert_within(host(ys[m])[None, :], y_ref, a_ref, "group matrix %d, %g" % (m, value))
    # the q-projection-with-gate shape, 16 heads of 128
    N, KQ, hd = 4096, 1024, 128
    w, xq = outlier_case(20, N, KQ, [1, 777], value)
    q, g = dq.q4k_gemv_split_qg(dev(w), dev(xq), N, KQ, hd)
    y_ref, a_ref = oracle_gemv(w, N, KQ, xq)
    tq, tg = oracle.split_qg(oracle.gemv_tolerance(a_ref), hd)
    yq, yg = oracle.split_qg(y_ref, hd)
    assert np.all(np.abs(host(q) - yq) <= tq) and np.all(np.abs(host(g) - yg) <= tg)


def test_log_uniform_activations_in_every_block():
    # |x| spread log-uniformly over 1e-30 .. 1e30 with random signs: most
    # activations of each block are far below its largest one
    N, K = 512, 2048
    rng = np.random.default_rng(21)
    w = synth.q4k_matrix(rng, N, K)
    x = (np.sign(rng.standard_normal((1, K))) * 10.0 ** rng.uniform(-30, 30, (1, K))).astype(np.float32)
    for col in range(0, K, 97):
        w = zero_weight_at(w, N, K, col, np.arange(0, N, 3))
    y = host(dq.q4k_gemv(dev(w), dev(x), N, K))
    y_ref, a_ref = oracle_gemv(w, N, K, x)
    assert_within(y, y_ref, a_ref, "log-uniform x")


@pytest.mark.parametrize("nexc", [1, 2, 4, 5, 40, 255])
def test_tiny_activations_beside_one_huge_one(nexc):
    # one block: a large activation on a weight that is zero in half the rows,
    # and `nexc` tiny ones; the rest of the block is zero
    N, K = 64, 256
    rng = np.random.default_rng(100 + nexc)
    w = synth.q4k_matrix(rng, N, K)
    x = np.zeros((1, K), np.float32)
    x[0, 128] = 1e9
    pos = rng.choice([k for k in range(K) if k != 128], size=nexc, replace=False)
    x[0, pos] = (rng.standard_normal(nexc) * 1e-3).astype(np.float32)
    w = zero_weight_at(w, N, K, 128, np.arange(0, N, 2))
    y = host(dq.q4k_gemv(dev(w), dev(x), N, K))
    y_ref, a_ref = oracle.q4k_gemv(w, N, K, x)
    assert_within(y, y_ref, a_ref, "%d tiny activations" % nexc)


def test_subnormal_activations_beside_normal_ones():
    N, K = 256, 1024
    rng = np.random.default_rng(22)
    w = synth.q4k_matrix(rng, N, K)
    x = synth.activations(rng, 1, K)
    x[0, ::3] *= np.float32(1e-40)       # subnormal, far below the blocks' largest |x|
    y = host(dq.q4k_gemv(dev(w), dev(x), N, K))
    y_ref, a_ref = oracle.q4k_gemv(w, N, K, x)
    assert_within(y, y_ref, a_ref, "subnormal mix")


def test_post_swiglu_activations_into_the_down_projection():
    # the down projection's real input: silu(g) * u of a gate/up pair, whose
    # negative-g tail spans many decades below each block's largest value
    H, F = 1024, 4096
    rng = np.random.default_rng(23)
    wg = synth.q4k_matrix(rng, F, H)
    wu = synth.q4k_matrix(rng, F, H)
    wd = synth.q4k_matrix(rng, H, F)
    x = synth.activations(rng, 1, H)
    g, _ = oracle.q4k_gemv(wg, F, H, x)
    u, _ = oracle.q4k_gemv(wu, F, H, x)
    h = oracle.swiglu(g, u).astype(np.float32)
    assert np.abs(h).min() < 1e-6 * np.abs(h).max()
    y = host(dq.q4k_gemv(dev(wd), dev(h), H, F))
    y_ref, a_ref = oracle_gemv(wd, H, F, h)
    assert_within(y, y_ref, a_ref, "down projection of silu(g) * u")
