"""The block-scaled NVFP4 GEMM (fp4q_nvfp4_gemm, tcgen05 tensor cores) consuming the quantizer's
codes and tiled scales, against the oracle's float64 product of the same operands: every product
of two element values is exact, so the difference is the fp32 accumulation alone, bounded here by
2e-5 of sum |a||b| per output."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle as O
import fp4_block_scaled_nvfp4_b200 as fq
from fp4_block_scaled_nvfp4_b200 import synth


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def _operand(cfg, rows, cols, obj):
    w = synth.make(cfg, rows=rows, cols=cols)
    xd = torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda()
    q = fq.quantize(xd, "nvfp4", obj, tiled_scales=True)
    r = O.nvfp4_quantize(O.widen_bf16(w["x"]), obj)
    return q, r


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 384, 1024), (128, 256, 4096)])
def test_nvfp4_gemm_matches_the_oracle_product(M, N, K):
    (qa, ra), (qb, rb) = _operand("cfg3", M, K, "sweep_mse"), _operand("cfg2", N, K, "sweep_mse")
    ws = fq.new_workspace()
    d = fq.nvfp4_gemm(qa, qb, workspace=ws)
    torch.cuda.synchronize()
    assert fq.read_device_status(ws) == fq.DEVSTAT_OK
    assert fq.last_launch_count() == 1
    # the operands are the oracle's bit for bit (checked elsewhere); the product from its tables
    assert np.array_equal(qa[0].cpu().numpy(), ra["codes"]) and np.array_equal(qb[0].cpu().numpy(), rb["codes"])
    ref = O.nvfp4_gemm(ra["codes"], ra["scales"], ra["S"], rb["codes"], rb["scales"], rb["S"])
    da = O.dequantize(ra["codes"], ra["scales"], ra["S"], "nvfp4").astype(np.float64)
    db = O.dequantize(rb["codes"], rb["scales"], rb["S"], "nvfp4").astype(np.float64)
    mag = np.abs(da) @ np.abs(db).T
    got = d.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= 2e-5 * mag + 1e-30), float(np.max(err / (mag + 1e-30)))


@pytest.mark.parametrize("M,N,K", [(256, 256, 512), (4096, 2432, 512), (2048, 4096, 768), (4096, 4096, 512)])
def test_nvfp4_gemm_several_tiles_per_cta(M, N, K):
    # one tile, and more tiles than two per SM: the two overlapping accumulators alternate,
    # 128-wide last tiles (N = 2432) mix with 256-wide ones, and the operand ring wraps across
    # tiles (K = 768 is three stages per tile)
    (qa, ra), (qb, rb) = _operand("cfg3", M, K, "sweep_mse"), _operand("cfg4", N, K, "absmax")
    ws = fq.new_workspace()
    d = fq.nvfp4_gemm(qa, qb, workspace=ws)
    torch.cuda.synchronize()
    assert fq.read_device_status(ws) == fq.DEVSTAT_OK
    ref = O.nvfp4_gemm(ra["codes"], ra["scales"], ra["S"], rb["codes"], rb["scales"], rb["S"])
    da = O.dequantize(ra["codes"], ra["scales"], ra["S"], "nvfp4").astype(np.float64)
    db = O.dequantize(rb["codes"], rb["scales"], rb["S"], "nvfp4").astype(np.float64)
    mag = np.abs(da) @ np.abs(db).T
    err = np.abs(d.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= 2e-5 * mag + 1e-30), float(np.max(err / (mag + 1e-30)))


def test_nvfp4_gemm_other_objectives_and_padding_rows():
    # AbsMax and 4/6 operands, and an output with a row pitch wider than N
    (qa, ra), (qb, rb) = _operand("cfg3", 128, 512, "absmax"), _operand("cfg4", 128, 512, "four_over_six")
    d = torch.full((128, 160), 7.0, device="cuda")
    fq.nvfp4_gemm(qa, qb, out=d[:, :128])
    torch.cuda.synchronize()
    ref = O.nvfp4_gemm(ra["codes"], ra["scales"], ra["S"], rb["codes"], rb["scales"], rb["S"])
    da = O.dequantize(ra["codes"], ra["scales"], ra["S"], "nvfp4").astype(np.float64)
    db = O.dequantize(rb["codes"], rb["scales"], rb["S"], "nvfp4").astype(np.float64)
    got = d.cpu().numpy()
    assert np.all(np.abs(got[:, :128] - ref) <= 2e-5 * (np.abs(da) @ np.abs(db).T) + 1e-30)
    assert np.all(got[:, 128:] == 7.0)


def _mx_operand(cfg, rows, cols, had, sweep=False):
    w = synth.make(cfg, rows=rows, cols=cols)
    xd = torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda()
    if had:
        q = fq.hadamard_quantize(xd, mx_sweep=sweep, tiled_scales=True)
    else:
        q = fq.quantize(xd, "mxfp4", mx_sweep=sweep, tiled_scales=True)
    x = O.widen_bf16(w["x"])
    r = O.mxfp4_quantize(x, hadamard=had, sweep="sweep" if sweep else "rule")
    return q, r, x


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 384, 1024), (4096, 2432, 512)])
@pytest.mark.parametrize("had", [False, True])
def test_mxfp4_gemm_matches_the_oracle_product(M, N, K, had):
    (qa, ra, xa), (qb, rb, xb) = _mx_operand("cfg5", M, K, had), _mx_operand("cfg4", N, K, had, sweep=True)
    assert np.array_equal(qa[0].cpu().numpy(), ra["codes"]) and np.array_equal(qb[0].cpu().numpy(), rb["codes"])
    ws = fq.new_workspace()
    d = fq.mxfp4_gemm(qa, qb, workspace=ws)
    torch.cuda.synchronize()
    assert fq.read_device_status(ws) == fq.DEVSTAT_OK
    assert fq.last_launch_count() == 1
    ref = O.mxfp4_gemm(ra["codes"], ra["scales"], rb["codes"], rb["scales"])
    da = O.dequantize(ra["codes"], ra["scales"], 0.0, "mxfp4").astype(np.float64)
    db = O.dequantize(rb["codes"], rb["scales"], 0.0, "mxfp4").astype(np.float64)
    mag = np.abs(da) @ np.abs(db).T
    got = d.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2e-5 * mag + 1e-30), float(np.max(np.abs(got - ref) / (mag + 1e-30)))
    # the rotations cancel in the product: either way it approximates the unrotated product
    exact = xa.astype(np.float64) @ xb.astype(np.float64).T
    assert np.linalg.norm(got - exact) <= 0.25 * np.linalg.norm(exact)


@pytest.mark.parametrize("mx", [False, True])
def test_full_size_gemm_sampled(mx):
    # the bench's GEMM at full size (8192 x 14336 x 4096: activation-workload rows times
    # weight-workload rows, quantized by the library), checked on 32 x 96 sampled outputs
    # against the oracle's product of the same rows and columns, quantized by the oracle
    M, N, K = 8192, 14336, 4096
    wa, wb = synth.make("cfg3", rows=M, cols=K), synth.make("cfg2", rows=N, cols=K)
    xa = torch.from_numpy(wa["x"].view(np.int16)).view(torch.bfloat16).cuda()
    xb = torch.from_numpy(wb["x"].view(np.int16)).view(torch.bfloat16).cuda()
    ws = fq.new_workspace()
    if mx:
        qa, qb = fq.hadamard_quantize(xa, tiled_scales=True)[:2], fq.hadamard_quantize(xb, tiled_scales=True)[:2]
        d = fq.mxfp4_gemm(qa, qb, workspace=ws)
    else:
        qa = fq.quantize(xa, "nvfp4", "sweep_mse", tiled_scales=True)
        qb = fq.quantize(xb, "nvfp4", "sweep_mse", tiled_scales=True)
        d = fq.nvfp4_gemm(qa, qb, workspace=ws)
    torch.cuda.synchronize()
    assert fq.read_device_status(ws) == fq.DEVSTAT_OK
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(M, 32, replace=False))
    cols = np.sort(rng.choice(N, 96, replace=False))
    xa_r, xb_c = O.widen_bf16(wa["x"][rows]), O.widen_bf16(wb["x"][cols])
    if mx:
        ra, rb = O.mxfp4_quantize(xa_r, hadamard=True), O.mxfp4_quantize(xb_c, hadamard=True)
        ref = O.mxfp4_gemm(ra["codes"], ra["scales"], rb["codes"], rb["scales"])
        da = O.dequantize(ra["codes"], ra["scales"], 0.0, "mxfp4").astype(np.float64)
        db = O.dequantize(rb["codes"], rb["scales"], 0.0, "mxfp4").astype(np.float64)
    else:
        Sa, sta = O.tensor_scale(O.widen_bf16(wa["x"]))
        Sb, stb = O.tensor_scale(O.widen_bf16(wb["x"]))
        assert sta == stb == 0
        assert np.float32(qa[2].cpu().item()).view(np.uint32) == np.float32(Sa).view(np.uint32)
        assert np.float32(qb[2].cpu().item()).view(np.uint32) == np.float32(Sb).view(np.uint32)
        ra, rb = O.nvfp4_quantize(xa_r, "sweep_mse", S=Sa), O.nvfp4_quantize(xb_c, "sweep_mse", S=Sb)
        ref = O.nvfp4_gemm(ra["codes"], ra["scales"], Sa, rb["codes"], rb["scales"], Sb)
        da = O.dequantize(ra["codes"], ra["scales"], Sa, "nvfp4").astype(np.float64)
        db = O.dequantize(rb["codes"], rb["scales"], Sb, "nvfp4").astype(np.float64)
    # the operands agree bit for bit on the sampled rows
    assert np.array_equal(qa[0][torch.from_numpy(rows).cuda()].cpu().numpy(), ra["codes"])
    assert np.array_equal(qb[0][torch.from_numpy(cols).cuda()].cpu().numpy(), rb["codes"])
    got = d[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].cpu().numpy().astype(np.float64)
    mag = np.abs(da) @ np.abs(db).T
    assert np.all(np.abs(got - ref) <= 2e-5 * mag + 1e-30), float(np.max(np.abs(got - ref) / (mag + 1e-30)))


@pytest.mark.parametrize("M,N,K", [(256, 384, 1024), (128, 256, 512)])
def test_gemm_bf16_output(M, N, K):
    # bf16 D: each value is the fp32 result RN(acc * RN(S_a S_b)) rounded to bf16 (nearest even),
    # checked against the fp32 launch of the same operands rounded by the oracle's bf16 rounding
    (qa, ra), (qb, rb) = _operand("cfg3", M, K, "sweep_mse"), _operand("cfg2", N, K, "sweep_mse")
    ws = fq.new_workspace()
    d32 = fq.nvfp4_gemm(qa, qb, workspace=ws)
    d16 = fq.nvfp4_gemm(qa, qb, workspace=ws, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert fq.read_device_status(ws) == fq.DEVSTAT_OK
    want = O.f32_to_bf16(d32.cpu().numpy())
    got = d16.view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    assert np.array_equal(got, want)
    # the MXFP4 GEMM with rotated operands rounds its fp32 result the same way
    xa = torch.from_numpy(synth.make("cfg3", rows=M, cols=K)["x"].view(np.int16)).view(torch.bfloat16).cuda()
    xb = torch.from_numpy(synth.make("cfg2", rows=N, cols=K)["x"].view(np.int16)).view(torch.bfloat16).cuda()
    a = fq.hadamard_quantize(xa, tiled_scales=True)
    b = fq.hadamard_quantize(xb, tiled_scales=True)
    m32 = fq.mxfp4_gemm(a, b, workspace=ws)
    m16 = fq.mxfp4_gemm(a, b, workspace=ws, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert np.array_equal(m16.view(torch.int16).cpu().numpy().view(np.uint16).ravel(),
                          O.f32_to_bf16(m32.cpu().numpy()))
