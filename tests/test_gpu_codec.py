"""The hardware conversions every quantize path relies on (cvt.rn.satfinite to E2M1 and to
E4M3FN, through fp4q_encode) against the oracle's codec over every fp32 bit pattern except the
NaNs: round to nearest with ties to even, saturation, signed zeros, subnormal inputs and
infinities.  Bit-exact."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import oracle as O
import fp4_block_scaled_nvfp4_b200 as fq

CHUNK = 1 << 26


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fq.lib()


@pytest.mark.parametrize("kind", ["e2m1", "e4m3"])
def test_hardware_codec_every_fp32_pattern(kind):
    out = torch.empty(CHUNK, dtype=torch.uint8, device="cuda")
    checked = 0
    for c in range((1 << 32) // CHUNK):
        lo = -(1 << 31) + c * CHUNK          # the chunk's bit patterns as int32
        x = torch.arange(lo, lo + CHUNK, dtype=torch.int32, device="cuda").view(torch.float32)
        got = fq.encode(x, kind, out=out).cpu().numpy()
        xh = np.arange(lo, lo + CHUNK, dtype=np.int64).astype(np.int32).view(np.float32)
        ref = O.encode(xh, kind)
        keep = ~np.isnan(xh)
        bad = np.flatnonzero((got != ref) & keep)
        assert bad.size == 0, (kind, [(hex(int(xh.view(np.uint32)[i])), int(got[i]), int(ref[i])) for i in bad[:5]])
        checked += int(keep.sum())
    assert checked == (1 << 32) - 2 * ((1 << 23) - 1)   # every pattern but the NaNs


def test_encode_tail_and_rejections():
    x = torch.tensor([0.25, 0.75, -1.25, 5.0, 7.0, -0.0, 3.5], device="cuda")
    assert fq.encode(x, "e2m1").cpu().tolist() == [0, 2, 0xA, 6, 7, 8, 6]
    assert fq.encode(torch.tensor([448.0, 464.0, 0.001953125, 1e9], device="cuda"), "e4m3").cpu().tolist() == \
        [0x7E, 0x7E, 0x01, 0x7E]
    L = fq.lib()
    assert L.fp4q_encode(None, 4, 0, None, None) == fq.ERR_INVALID_ARG
    assert L.fp4q_encode(None, 4, 2, None, None) == fq.ERR_INVALID_ARG
    assert L.fp4q_encode(None, -1, 0, None, None) == fq.ERR_SHAPE
    assert L.fp4q_encode(None, 0, 0, None, None) == fq.OK
