"""q4k_gemv_noalloc: the Q4_K GEMV entry point that allocates nothing.

Some callers cannot allocate device memory: code that runs where no device
allocator is reachable, or that must keep its memory fixed once set up (a
decode loop with a pre-planned budget).  For them the library keeps its own
fixed scratch array in device memory instead of taking a workspace argument.
These tests call that entry point through the C ABI, twice in a row, and
check each output (logits and argmax) against the ordinary q4k_gemv entry point
within the GEMV tolerance (1e-4 * sum|w*x| + 1e-6, sum taken by the oracle).
"""

import ctypes

import numpy as np
import pytest

import oracle
from dequant_gemv_q4_b200 import synth

torch = pytest.importorskip("torch")
import dequant_gemv_q4_b200 as dq  # noqa: E402

pytestmark = pytest.mark.gpu

DQ_ERR_WORKSPACE = 4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    dq.load_library()
    yield


def _call_noalloc(lib, w, x, y, N, K, B, idx=None):
    vp = ctypes.c_void_p
    s = torch.cuda.current_stream().cuda_stream
    return lib.q4k_gemv_noalloc(vp(w.data_ptr()), 0, vp(x.data_ptr()), vp(y.data_ptr()), N, K, B,
                                vp(idx.data_ptr()) if idx is not None else None, vp(s))


@pytest.mark.parametrize("N,K,B,argmax", [
    (5000, 4096, 1, True),       # argmax candidates in the scratch array
    (64, 65536, 1, True),        # split-K partials + argmax through the reduction
    (512, 12288, 8, False),      # split-K partials for B = 8
])
def test_noalloc_matches_q4k_gemv_twice(N, K, B, argmax):
    lib = dq.load_library()
    rng = np.random.default_rng(N + K + B)
    w_np = synth.q4k_matrix(rng, N, K)
    x_np = synth.activations(rng, B, K)
    w = torch.from_numpy(w_np).cuda()
    x = torch.from_numpy(x_np).cuda()
    need = dq.dq_workspace_bytes(dq.DQ_OP_Q4K_GEMV, N, K, B, argmax)
    assert 0 < need <= lib.dq_noalloc_scratch_bytes()
    ref = dq.q4k_gemv(w, x, N, K, argmax=argmax)
    y_ref, i_ref = (ref if argmax else (ref, None))
    _, a_ref = oracle.q4k_gemv(w_np, N, K, x_np)
    tol = oracle.gemv_tolerance(a_ref)
    for _ in range(2):
        y = torch.full((B, N), float("nan"), device="cuda")
        idx = torch.full((1,), -7, dtype=torch.int64, device="cuda") if argmax else None
        assert _call_noalloc(lib, w, x, y, N, K, B, idx) == 0
        torch.cuda.synchronize()
        err = np.abs(y.cpu().numpy().astype(np.float64) - y_ref.cpu().numpy().reshape(B, N))
        assert np.all(err <= tol)
        if argmax:
            assert int(idx.item()) == int(i_ref.item())


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = dq.load_library()
    # B = 8, K = 65536 splits K sixteen ways; the partial sums of N = 16384 rows
    # need 8 MiB, twice the fixed scratch: rejected before anything launches.
    N, K, B = 16384, 65536, 8
    assert dq.dq_workspace_bytes(dq.DQ_OP_Q4K_GEMV, N, K, B) > lib.dq_noalloc_scratch_bytes()
    w = torch.zeros(4096, dtype=torch.uint8, device="cuda")     # never read
    x = torch.zeros(B * K, dtype=torch.float32, device="cuda")
    y = torch.full((16,), 3.0, device="cuda")
    assert _call_noalloc(lib, w, x, y, N, K, B) == DQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(y == 3.0).item()
