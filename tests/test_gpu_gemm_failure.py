"""The GEMM's bounded-wait failure path, exercised without a fault: a test build of the library
(libfp4q_failtest.so, the same sources with FP4Q_GEMM_FAIL_FIRST_WAIT) makes the MMA thread
treat its first wait as timed out.  The call must return, report FP4Q_DEVSTAT_TIMEOUT in the
status word once the stream is done (the producer's own wait for a free ring slot then runs out
as well, after its bounded polls), and leave the context usable: the product library's next GEMM
on the same device is correct."""
import ctypes as C
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle as O
import fp4_block_scaled_nvfp4_b200 as fq
from fp4_block_scaled_nvfp4_b200 import synth

TEST_LIB = os.path.join(os.path.dirname(fq.__file__), "libfp4q_failtest.so")


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if not os.path.exists(TEST_LIB):
        pytest.fail("libfp4q_failtest.so is not built (__graft_entry__.build() builds it)")
    fq.lib()


def _operand(cfg, rows, cols):
    w = synth.make(cfg, rows=rows, cols=cols)
    xd = torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda()
    return fq.quantize(xd, "nvfp4", "sweep_mse", tiled_scales=True), w


def test_timed_out_wait_returns_status_and_leaves_the_device_usable():
    M, N, K = 256, 512, 2048      # 8 K stages per tile: the producer fills the 4-slot ring and waits
    (qa, wa), (qb, wb) = _operand("cfg3", M, K), _operand("cfg2", N, K)
    L = C.CDLL(TEST_LIB)
    P, i64 = C.c_void_p, C.c_int64
    L.fp4q_nvfp4_gemm.restype = C.c_int
    L.fp4q_nvfp4_gemm.argtypes = [P, P, P, P, P, P, i64, i64, i64, P, i64, P, P]
    L.fp4q_last_cuda_error.restype = C.c_int
    d = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    ws = fq.new_workspace()
    ptr = lambda t: C.c_void_p(t.data_ptr())
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.fp4q_nvfp4_gemm(ptr(qa[0]), ptr(qa[1]), ptr(qa[2]), ptr(qb[0]), ptr(qb[1]), ptr(qb[2]), M, N, K, ptr(d),
                           N, ptr(ws), stream)
    assert rc == fq.OK, f"rc {rc}, CUDA error {L.fp4q_last_cuda_error()}"
    torch.cuda.synchronize()
    assert fq.read_device_status(ws) == fq.DEVSTAT_TIMEOUT
    assert torch.equal(d, torch.full_like(d, 7.0))     # no tile was written
    # the same device, the product library: a correct product and a clean status
    ws2 = fq.new_workspace()
    out = fq.nvfp4_gemm(qa, qb, workspace=ws2)
    torch.cuda.synchronize()
    assert fq.read_device_status(ws2) == fq.DEVSTAT_OK
    ra = O.nvfp4_quantize(O.widen_bf16(wa["x"]), "sweep_mse")
    rb = O.nvfp4_quantize(O.widen_bf16(wb["x"]), "sweep_mse")
    ref = O.nvfp4_gemm(ra["codes"], ra["scales"], ra["S"], rb["codes"], rb["scales"], rb["S"])
    da = O.dequantize(ra["codes"], ra["scales"], ra["S"], "nvfp4").astype(np.float64)
    db = O.dequantize(rb["codes"], rb["scales"], rb["S"], "nvfp4").astype(np.float64)
    mag = np.abs(da) @ np.abs(db).T
    assert np.all(np.abs(out.cpu().numpy().astype(np.float64) - ref) <= 2e-5 * mag + 1e-30)
