"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait of the GEMV kernels for their own asynchronous copies is bounded by
the global timer.  dq_test_lost_copy runs a batch-1 q4k_gemv in which one warp
arms the mbarrier of its first slot but issues no copy into it, with every
wait limited to 1 ms.  The kernel must return, the device error flag must read
1 (wait timeout), the rows of the other tiles must still be right, and the
next ordinary call must be correct with the flag back at 0.
"""

import numpy as np
import pytest

import oracle
from dequant_gemv_q4_b200 import synth

torch = pytest.importorskip("torch")
import dequant_gemv_q4_b200 as dq  # noqa: E402

pytestmark = pytest.mark.gpu

ERR_WAIT_TIMEOUT = 1


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    dq.load_library()
    yield
    assert dq.dq_device_error(clear=True) == 0


@pytest.mark.parametrize("N,K", [(4096, 4096), (4096, 12288)])   # no K split; K split in clusters
def test_a_lost_copy_times_out_sets_the_flag_and_the_next_call_is_clean(N, K):
    import ctypes
    lib = dq.load_library()
    assert dq.dq_device_error(clear=True) == 0
    rng = np.random.default_rng(N + K)
    w_np = synth.q4k_matrix(rng, N, K)
    x_np = synth.activations(rng, 1, K)
    w = torch.from_numpy(w_np).cuda()
    x = torch.from_numpy(x_np).cuda()
    y = torch.full((1, N), float("nan"), device="cuda")
    need = dq.dq_workspace_bytes(dq.DQ_OP_Q4K_GEMV, N, K, 1)
    ws = torch.empty(max(16, need), dtype=torch.uint8, device="cuda")
    vp = ctypes.c_void_p
    s = torch.cuda.current_stream().cuda_stream
    st = lib.dq_test_lost_copy(vp(w.data_ptr()), vp(x.data_ptr()), vp(y.data_ptr()), N, K, 1_000_000,
                               vp(ws.data_ptr()), ws.numel(), vp(s))
    assert st == 0
    torch.cuda.synchronize()                     # the kernel returned
    assert dq.dq_device_error(clear=True) == ERR_WAIT_TIMEOUT
    # only the tiles of the warp that lost its slot may be wrong: a handful of
    # 16-row tiles out of 256
    y_ref, a_ref = oracle.q4k_gemv(w_np, N, K, x_np)
    got = y.cpu().numpy().astype(np.float64)
    good = np.abs(got - y_ref) <= oracle.gemv_tolerance(a_ref)
    assert good.sum() >= 0.95 * N, "%d of %d rows wrong" % (N - good.sum(), N)
    # the context is usable and the next call is clean
    y2 = dq.q4k_gemv(w, x, N, K)
    torch.cuda.synchronize()
    assert np.all(np.abs(y2.cpu().numpy().astype(np.float64) - y_ref) <= oracle.gemv_tolerance(a_ref))
    assert dq.dq_device_error(clear=True) == 0
