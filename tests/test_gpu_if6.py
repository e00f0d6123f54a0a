"""IF6 (FP6 E2M3 vs scaled INT6 per 16-element block, indicator in the scale byte's sign bit)
on the B200 against the oracle: 6-bit codes, scale bytes and S bit-exact, dequantized values
bit-exact (fp32 and bf16), on weight- and activation-shaped tensors, ragged shapes and edge
blocks.  Adaptive Block-Scaled Data Types (gist.science/ko/paper/2603.28765), Methodology:
the IF4 construction extended to 6-bit elements."""
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


def _dev(w):
    if w["dtype"] == "bf16":
        return torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(w["x"])).cuda()


def _check(xd, x, S=None):
    ws = fq.new_workspace()
    gs = None if S is None else torch.tensor([S], dtype=torch.float32, device="cuda")
    codes, scales, g = fq.quantize(xd, "if6", global_scale=gs, workspace=ws)
    torch.cuda.synchronize()
    r = O.if6_quantize(x, S=S)
    assert fq.read_device_status(ws) == r["status"]
    assert np.float32(g.cpu().numpy()[0]).view(np.uint32) == np.float32(r["S"]).view(np.uint32)
    assert np.array_equal(scales.cpu().numpy(), r["scales"])
    assert np.array_equal(codes.cpu().numpy(), r["codes"])
    for bf in (False, True):
        out = fq.dequantize(codes, scales, g, "if6", out_dtype=torch.bfloat16 if bf else torch.float32)
        torch.cuda.synchronize()
        ref = O.if6_dequantize(r["codes"], r["scales"], r["S"], out_bf16=bf)
        got = out.view(torch.int16).cpu().numpy().view(np.uint16) if bf else out.cpu().numpy()
        assert np.array_equal(got.view(np.uint16 if bf else np.uint32), ref.view(np.uint16 if bf else np.uint32))
    return r


@pytest.mark.parametrize("cfg,rows,cols", [("cfg4", 24, 14336), ("cfg4", 3, 48), ("cfg3", 17, 2048), ("cfg2", 8, 4096),
                                           ("cfg1", None, None)])
def test_if6_parity(cfg, rows, cols):
    w = synth.make(cfg, rows=rows, cols=cols)
    x = O.widen_bf16(w["x"]) if w["dtype"] == "bf16" else np.asarray(w["x"], np.float32)
    r = _check(_dev(w), x)
    assert 0 < np.mean(r["scales"] >> 7) < 1          # both element types occur


def test_if6_edge_blocks_and_given_scale():
    x = np.zeros((4, 64), np.float32)
    x[0, :16] = [7.5, 0.125, 3.75, -1.875, 0.5, 6, 0.625, -0.375] + [0] * 8     # FP6 grid at s = 1
    K = np.float32(15) / np.float32(62)
    x[0, 16:32] = [7.5, K, 2 * K, 4 * K, 8 * K, 16 * K] + [0] * 10              # INT6 points
    x[1, 7] = 1920.0                                                            # S = 1
    x[2, 40:48] = -0.0
    x[3, 3] = 1e-30                                                             # a block far below S
    r = _check(torch.from_numpy(x).cuda(), x)
    assert r["S"] == 1.0 and r["scales"][0, 0] == 0x38 and r["scales"][0, 1] == 0xB8
    _check(torch.from_numpy(x).cuda(), x, S=0.37)


def test_if6_full_size_sampled():
    w = synth.make("cfg4")
    xd = _dev(w)
    ws = fq.new_workspace()
    codes, scales, g = fq.quantize(xd, "if6", workspace=ws)
    torch.cuda.synchronize()
    assert fq.read_device_status(ws) == 0
    x = O.widen_bf16(w["x"])
    S, st = O.tensor_scale(x)
    S6 = float(np.float32(np.float32(np.abs(x).max()) / np.float32(1920.0)))
    assert float(g.cpu()[0]) == S6
    rows = np.sort(np.random.default_rng(6).choice(w["rows"], size=48, replace=False))
    r = O.if6_quantize(x[rows], S=S6)
    assert np.array_equal(scales.cpu().numpy()[rows], r["scales"])
    assert np.array_equal(codes.cpu().numpy()[rows], r["codes"])


def test_if6_padded_rows_and_nonfinite():
    # a row pitch larger than the width (the kernel's padded-row addressing), bit-exact against
    # the oracle on the unpadded values; then a NaN: status NONFINITE and zero-filled outputs
    w = synth.make("cfg4", rows=10, cols=1024)
    x = O.widen_bf16(w["x"])
    full = _dev(w)
    padded = torch.zeros((10, 1024 + 48), dtype=torch.bfloat16, device="cuda")
    padded[:, :1024] = full
    view = padded[:, :1024]
    assert view.stride(0) == 1024 + 48
    ws = fq.new_workspace()
    codes, scales, g = fq.quantize(view, "if6", workspace=ws)
    torch.cuda.synchronize()
    r = O.if6_quantize(x)
    assert fq.read_device_status(ws) == r["status"] == 0
    assert np.float32(g.cpu().numpy()[0]).view(np.uint32) == np.float32(r["S"]).view(np.uint32)
    assert np.array_equal(scales.cpu().numpy(), r["scales"])
    assert np.array_equal(codes.cpu().numpy(), r["codes"])
    bad = full.clone()
    bad[3, 100] = float("nan")
    codes, scales, g = fq.quantize(bad, "if6", workspace=ws)
    torch.cuda.synchronize()
    assert fq.read_device_status(ws) == fq.DEVSTAT_NONFINITE
    assert not codes.any() and not scales.any()


@pytest.mark.parametrize("cfg,rows,cols", [("cfg4", 40, 14336), ("cfg1", None, None)])
def test_if6_global_scale_entry_point(cfg, rows, cols):
    # fp4q_if6_global_scale alone gives the S that an IF6 quantize computes, and passing it back
    # reproduces that call's codes and scales
    w = synth.make(cfg, rows=rows, cols=cols)
    x = O.widen_bf16(w["x"]) if w["dtype"] == "bf16" else np.asarray(w["x"], np.float32)
    xd = _dev(w)
    ws = fq.new_workspace()
    g = fq.global_scale(xd, workspace=ws, fmt="if6")
    torch.cuda.synchronize()
    assert np.float32(g.cpu().numpy()[0]).view(np.uint32) == np.float32(O.if6_tensor_scale(x)).view(np.uint32)
    c0, s0, g0 = fq.quantize(xd, "if6", workspace=ws)
    c1, s1, _ = fq.quantize(xd, "if6", global_scale=g, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(g.view(torch.int32), g0.view(torch.int32))
    assert torch.equal(c0, c1) and torch.equal(s0, s1)
    # a non-finite element gives S = NaN and the NONFINITE status; the next call (a zero tensor)
    # overwrites the status word with its own
    z = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    z[2, 9] = float("nan")
    gn = fq.global_scale(z, workspace=ws, fmt="if6")
    torch.cuda.synchronize()
    assert torch.isnan(gn).all() and fq.read_device_status(ws) & fq.DEVSTAT_NONFINITE
    z[2, 9] = 0
    gz = fq.global_scale(z, workspace=ws, fmt="if6")
    torch.cuda.synchronize()
    assert float(gz.item()) == 0.0
    assert fq.read_device_status(ws) == O.if6_quantize(np.zeros((4, 64), np.float32))["status"]
