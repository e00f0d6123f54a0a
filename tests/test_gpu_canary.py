"""Guard bytes around every output buffer (the stand-in for a memory checker, which this pool
does not offer): the outputs of quantize and dequantize are written into the middle of larger
buffers filled with a known pattern, on a ragged shape (130 rows: not a multiple of the
128-row scale tile nor of a warp), and the pattern outside must be untouched afterwards.  The
results must also equal those of a call into buffers of the exact size."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import fp4_block_scaled_nvfp4_b200 as fq

G = 64           # guard bytes (a multiple of 16, so the outputs stay 16-byte aligned)
CANARY = 0xA5
FCANARY = 12345.0


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


def _guarded_u8(n, fill_inside=None):
    buf = torch.full((n + 2 * G,), CANARY, dtype=torch.uint8, device="cuda")
    if fill_inside is not None:
        buf[G:G + n] = fill_inside
    return buf, buf[G:G + n]


def _guards_intact(buf, n):
    return bool((buf[:G] == CANARY).all()) and bool((buf[G + n:] == CANARY).all())


@pytest.mark.parametrize("fmt,obj,tiled,had16", [
    ("nvfp4", "sweep_mse", False, False), ("nvfp4", "sweep_wmse", False, False), ("nvfp4", "absmax", True, False),
    ("nvfp4", "four_over_six", False, True), ("if4", "absmax", False, False), ("mxfp4", "absmax", False, False),
    ("mxfp4", "absmax", True, False)])
def test_quantize_and_dequantize_stay_inside_their_buffers(fmt, obj, tiled, had16):
    rows, cols = 130, 96
    rng = np.random.default_rng(11)
    x = torch.from_numpy(rng.laplace(size=(rows, cols)).astype(np.float32)).cuda()
    imp = torch.from_numpy(np.linspace(0.1, 3.0, cols).astype(np.float32)).cuda() if obj == "sweep_wmse" else None
    nc = rows * cols // 2
    ns = fq.scale_bytes(rows, cols, fmt, tiled)
    cbuf, codes = _guarded_u8(nc)
    sbuf, scales = _guarded_u8(ns, fill_inside=0 if tiled else None)   # tiled padding starts zeroed
    gbuf = torch.full((48,), FCANARY, dtype=torch.float32, device="cuda")
    gs = gbuf[16:17]
    out = (codes.view(rows, cols // 2), scales if tiled else scales.view(rows, cols // fq.BLOCK[fmt]), gs)
    fq.quantize(x, fmt, obj, importance=imp, out=out, tiled_scales=tiled, hadamard16=had16)
    torch.cuda.synchronize()
    assert _guards_intact(cbuf, nc) and _guards_intact(sbuf, ns)
    assert bool((gbuf[:16] == FCANARY).all()) and bool((gbuf[17:] == FCANARY).all())
    ref = fq.quantize(x, fmt, obj, importance=imp, tiled_scales=tiled, hadamard16=had16)
    torch.cuda.synchronize()
    assert torch.equal(out[0], ref[0]) and torch.equal(out[1].view(-1), ref[1].view(-1))
    # dequantize into a guarded fp32 buffer
    nd = rows * cols
    dbuf = torch.full((nd + 2 * G,), FCANARY, dtype=torch.float32, device="cuda")
    xd = dbuf[G:G + nd].view(rows, cols)
    fq.dequantize(out[0], out[1], out[2] if fmt != "mxfp4" else None, fmt, inverse_hadamard=had16, out=xd,
                  tiled_scales=tiled)
    torch.cuda.synchronize()
    assert bool((dbuf[:G] == FCANARY).all()) and bool((dbuf[G + nd:] == FCANARY).all())
    xr = fq.dequantize(ref[0], ref[1], ref[2], fmt, inverse_hadamard=had16, tiled_scales=tiled)
    torch.cuda.synchronize()
    assert torch.equal(xd.view(torch.int32), xr.view(torch.int32))
