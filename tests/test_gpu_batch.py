"""fp4q_quantize_batch: a sequence of tensors quantized in one call, each quantize kernel also
taking the next tensor's amax.  Every tensor's codes, scale bytes and S must equal the oracle's
for that tensor alone (and so the separate fp4q_quantize calls), whatever the shapes around it:
empty tensors, row-padded views, a larger tensor after a small one (more of its amax than the
small kernel's blocks carry), a non-finite tensor in the middle, bf16 and fp32 batches."""
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


def _bf16_bits(x):
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _inputs(dtype, seed=0):
    """(host float32 values the oracle sees, device tensor) for each tensor of the batch."""
    rng = np.random.default_rng(seed)
    vals = [synth.as_f32(synth.make("cfg3", rows=17, cols=2048)),
            np.zeros((0, 64), np.float32),
            synth.as_f32(synth.make("cfg4", rows=3, cols=48)),
            synth.as_f32(synth.make("cfg2", rows=40, cols=4096)),    # stored as a row-padded view
            rng.standard_normal((8, 256)).astype(np.float32),
            synth.as_f32(synth.make("cfg3", rows=300, cols=4096, seed=7)),
            np.float32([[3.0, -0.25] + [0.0] * 14])]
    vals[4][5, 17] = np.nan                                          # this tensor is out of contract
    out = []
    for i, v in enumerate(vals):
        if dtype == "bf16":
            bits = _bf16_bits(v)
            v = (bits.astype(np.uint32) << 16).view(np.float32)
            t = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(v))
        if i == 3:   # padded rows: a view of the first cols of a wider buffer
            wide = torch.zeros((v.shape[0], v.shape[1] + 64), dtype=t.dtype)
            wide[:, :v.shape[1]] = t
            t = wide.cuda()[:, :v.shape[1]]
        else:
            t = t.cuda()
        out.append((v, t))
    return out


def _oracle(v, fmt, obj, imp, S, had16):
    if fmt == "if4":
        return O.if4_quantize(v, S=S, hadamard16=had16, sweep="sweep" if obj == "if4_sweep" else "absmax")
    return O.nvfp4_quantize(v, obj, importance=imp, S=S, hadamard16=had16)


CASES = [("nvfp4", "sweep_mse", False), ("nvfp4", "absmax", False), ("nvfp4", "four_over_six", False),
         ("nvfp4", "sweep_wmse", False), ("if4", None, False), ("if4", "if4_sweep", False),
         ("nvfp4", "sweep_mse", True), ("if4", None, True)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("fmt,obj,had16", CASES)
def test_batch_matches_the_oracle_per_tensor(dtype, fmt, obj, had16):
    ins = _inputs(dtype)
    rng = np.random.default_rng(3)
    imps = [(rng.random(v.shape[1]) * 4).astype(np.float32) for v, _ in ins] if obj == "sweep_wmse" else None
    ws = fq.new_workspace()
    res = fq.quantize_batch([t for _, t in ins], fmt, obj if fmt == "nvfp4" else "absmax",
                            importance=None if imps is None else [torch.from_numpy(w).cuda() for w in imps],
                            workspace=ws, hadamard16=had16, if4_sweep=(obj == "if4_sweep"))
    torch.cuda.synchronize()
    m = sum(1 for v, _ in ins if v.size)
    fused = not had16 and obj != "sweep_wmse"
    assert fq.last_launch_count() == (m + 1 if fused else 2 * m)
    status = 0
    for i, ((v, _), (c, s, g)) in enumerate(zip(ins, res)):
        if not v.size:
            continue
        r = _oracle(v, fmt, obj, None if imps is None else imps[i], None, had16)
        status |= r["status"]
        where = f"tensor {i} shape {v.shape}"
        assert np.float32(g.cpu().numpy()[0]).view(np.uint32) == np.float32(r["S"]).view(np.uint32), where
        assert np.array_equal(s.cpu().numpy(), r["scales"]), where
        assert np.array_equal(c.cpu().numpy(), r["codes"]), where
    assert status == fq.DEVSTAT_NONFINITE
    assert fq.read_device_status(ws) == status


@pytest.mark.parametrize("fmt", ["nvfp4", "if4"])
def test_batch_with_given_scales_and_tiled_layout(fmt):
    ins = [(v, t) for v, t in _inputs("bf16") if v.size and not np.isnan(v).any()]
    Ss = [0.37, 2.0 ** -20, 1.0, 5e-3, 0.01]
    ws = fq.new_workspace()
    gss = [torch.tensor([S], dtype=torch.float32, device="cuda") for S in Ss]
    res = fq.quantize_batch([t for _, t in ins], fmt, "sweep_mse", global_scales=gss, workspace=ws)
    torch.cuda.synchronize()
    assert fq.last_launch_count() == len(ins)
    for (v, _), (c, s, g), S in zip(ins, res, Ss):
        r = _oracle(v, fmt, "sweep_mse", None, S, False)
        assert np.array_equal(s.cpu().numpy(), r["scales"]) and np.array_equal(c.cpu().numpy(), r["codes"])
    assert fq.read_device_status(ws) == 0
    if fmt == "nvfp4":   # the tiled scale layout of block-scaled GEMMs
        outs = [fq.alloc_outputs(v.shape[0], v.shape[1], "nvfp4", tiled=True) for v, _ in ins]
        res = fq.quantize_batch([t for _, t in ins], "nvfp4", "sweep_mse", outs=outs, tiled_scales=True)
        torch.cuda.synchronize()
        for (v, _), (c, s, g) in zip(ins, res):
            r = O.nvfp4_quantize(v, "sweep_mse")
            assert np.array_equal(s.cpu().numpy(), O.tile_scales(r["scales"]))
            assert np.array_equal(c.cpu().numpy(), r["codes"])


def test_full_size_batch_equals_separate_calls():
    # three activation-sized tensors (8192 x 4096 bf16) and the same buffer twice in a row: each
    # result equals its own fp4q_quantize call bit for bit, and each S the oracle's tensor scale
    ws_ = [synth.make("cfg3", seed=s) for s in (11, 12, 13)]
    xs = [torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda() for w in ws_]
    xs = xs + [xs[0]]
    ws = fq.new_workspace()
    res = fq.quantize_batch(xs, "nvfp4", "sweep_mse", workspace=ws)
    torch.cuda.synchronize()
    assert fq.last_launch_count() == len(xs) + 1 and fq.read_device_status(ws) == 0
    for i, (x, (c, s, g)) in enumerate(zip(xs, res)):
        c0, s0, g0 = fq.quantize(x, "nvfp4", "sweep_mse", workspace=fq.new_workspace())
        torch.cuda.synchronize()
        assert torch.equal(g.view(torch.int32), g0.view(torch.int32)), i
        assert torch.equal(s, s0) and torch.equal(c, c0), i
        S_o = O.tensor_scale(O.widen_bf16(ws_[i % 3]["x"]))[0]
        assert np.float32(g.cpu().numpy()[0]).view(np.uint32) == np.float32(S_o).view(np.uint32)

