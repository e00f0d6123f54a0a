"""GPU parity of the 16-point rotated NVFP4 / IF4 path (FP4Q_F_HADAMARD16) against the oracle.

Every 16-element block is rotated by H_16 / 4 before the method runs, and S is taken over
the rotated tensor (Bridging the Gap ... Microscaling FP4, gist.science/ko/paper/2509.23202,
"Methodology", block-wise Hadamard transforms, applied to NVFP4 as to MXFP4).  Bar as in
test_gpu_parity: S, codes and scale bytes bit-exact; dequantized values (with and without the
inverse rotation) bit-exact, NaN compared as NaN.
"""
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


def to_dev(w):
    if w["dtype"] == "bf16":
        return torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(w["x"])).cuda()


def oracle_x(w, rows=None):
    x = O.widen_bf16(w["x"]) if w["dtype"] == "bf16" else np.asarray(w["x"], np.float32)
    return x if rows is None else x[rows]


def bits(v):
    return np.float32(v).view(np.uint32)


def run(xd, fmt, obj="sweep_mse", S=None):
    ws = fq.new_workspace()
    gs = None if S is None else torch.tensor([S], dtype=torch.float32, device="cuda")
    out = fq.quantize(xd, fmt, obj, global_scale=gs, workspace=ws, hadamard16=True)
    torch.cuda.synchronize()
    st = fq.read_device_status(ws)
    c, s, g = out
    return c.cpu().numpy(), s.cpu().numpy(), float(g.cpu()[0]), st, out


def oracle_run(x, fmt, obj="sweep_mse", S=None):
    if fmt == "if4":
        return O.if4_quantize(x, S=S, hadamard16=True)
    return O.nvfp4_quantize(x, obj, S=S, hadamard16=True)


def same(gc, gsc, r):
    if not np.array_equal(gsc, r["scales"]):
        bad = np.argwhere(gsc != r["scales"])
        raise AssertionError(f"{len(bad)} scale bytes differ, first {bad[:5].tolist()}")
    if not np.array_equal(gc, r["codes"]):
        bad = np.argwhere(gc != r["codes"])
        raise AssertionError(f"{len(bad)} code bytes differ, first {bad[:5].tolist()}")


def check_dequant(out, r, fmt):
    codes, scales, gs = out
    for inv in (False, True):
        for bf in (False, True):
            xd = fq.dequantize(codes, scales, gs, fmt, inverse_hadamard=inv,
                               out_dtype=torch.bfloat16 if bf else torch.float32)
            torch.cuda.synchronize()
            got = xd.view(torch.int16).cpu().numpy().view(np.uint16) if bf else xd.cpu().numpy()
            ref = O.dequantize(r["codes"], r["scales"], r["S"], fmt, inverse_hadamard=inv, out_bf16=bf)
            if bf:
                assert np.array_equal(got, ref)
            else:
                nan = np.isnan(ref)
                assert np.array_equal(np.isnan(got), nan)
                assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


CASES = [
    ("cfg3", 96, 4096, "nvfp4", "sweep_mse"), ("cfg3", 33, 1024, "nvfp4", "absmax"),
    ("cfg3", 33, 1024, "nvfp4", "four_over_six"), ("cfg3", 7, 48, "nvfp4", "sweep_mse"),
    ("cfg3", 1, 16, "nvfp4", "sweep_mse"), ("cfg1", None, None, "nvfp4", "sweep_mse"),
    ("cfg1", None, None, "nvfp4", "four_over_six"), ("cfg2", 9, 4096, "nvfp4", "sweep_mse"),
    ("cfg4", 24, 14336, "if4", None), ("cfg4", 3, 48, "if4", None), ("cfg1", None, None, "if4", None),
]


@pytest.mark.parametrize("cfg,rows,cols,fmt,obj", CASES)
def test_rotated_parity(cfg, rows, cols, fmt, obj):
    w = synth.make(cfg, rows=rows, cols=cols)
    gc, gsc, gS, st, out = run(to_dev(w), fmt, obj or "absmax")
    r = oracle_run(oracle_x(w), fmt, obj)
    assert st == r["status"] == 0
    assert bits(gS) == bits(r["S"])
    same(gc, gsc, r)
    check_dequant(out, r, fmt)
    if fmt == "if4" and gsc.size > 100:   # both paths occur (rotated blocks favour INT4)
        assert 0 < np.mean(gsc >> 7) < 1


def test_rotated_global_scale_and_given_scale():
    """fp4q_hadamard_global_scale gives the rotated tensor's S (also through a padded row
    pitch); passing it back with FP4Q_F_GLOBAL_SCALE_GIVEN reproduces the one-call result."""
    w = synth.make("cfg3", rows=40, cols=2048)
    x = oracle_x(w)
    full = to_dev(w)
    padded = torch.zeros((40, 2048 + 128), dtype=torch.bfloat16, device="cuda")
    padded[:, :2048] = full
    view = padded[:, :2048]
    S_ref, st_ref = O.tensor_scale(O.rotate16(x))
    for t in (full, view):
        ws = fq.new_workspace()
        gs = fq.global_scale(t, workspace=ws, hadamard16=True)
        torch.cuda.synchronize()
        assert bits(float(gs.cpu()[0])) == bits(S_ref) and fq.read_device_status(ws) == st_ref == 0
        assert fq.last_launch_count() == 1
    plain = fq.global_scale(full)
    assert bits(float(plain.cpu()[0])) != bits(S_ref)          # the rotation changes the amax
    for fmt, obj in (("nvfp4", "sweep_mse"), ("if4", "absmax")):
        gc, gsc, _, st, _ = run(view, fmt, obj, S=float(gs.cpu()[0]))
        assert fq.last_launch_count() == 1
        r = oracle_run(x, fmt, obj)
        assert st == 0
        same(gc, gsc, r)


def test_rotated_launch_counts():
    x = torch.randn(8, 64, device="cuda")
    fq.quantize(x, "nvfp4", "sweep_mse", hadamard16=True)
    assert fq.last_launch_count() == 2
    fq.quantize(x, "if4", hadamard16=True, global_scale=torch.ones(1, device="cuda"))
    assert fq.last_launch_count() == 1


def _edge_tensors():
    rng = np.random.default_rng(77)
    out = {}
    out["zeros"] = np.zeros((3, 64), np.float32)
    t = rng.laplace(size=(8, 256)).astype(np.float32)
    t[3, 40] = 1e4                                   # one outlier spread over its block
    t[5, 16:32] *= 1e-7
    t[6, 32:48] = 0.0
    t[7, 48:64] = np.float32(2.0 ** -140)           # fp32 subnormal inputs
    t[2, 0:16] = np.float32(3.0) * np.float32(2.0 ** -149)   # rotated then divided: subnormal rounding
    out["mixed_ranges"] = t
    s = np.zeros((2, 32), np.float32)
    s[0, 0] = np.float32(2.0 ** -125 + 2.0 ** -149)  # H x / 4 rounds in the subnormal range
    s[1, 16:32] = np.float32(2.0 ** -127)
    out["subnormal_rotation"] = s                    # S below the supported range: RANGE
    g = np.zeros((2, 64), np.float32)                # rotated grid values: exact, sweep ties
    g[0, :16] = np.array([6, 4, 3, 2, 1.5, 1, .5, 0, -6, -4, -3, -2, -1.5, -1, -.5, 0], np.float32)
    g[1, 16:32] = 6.0
    out["rotated_grid"] = O.rotate16(g)
    big = np.zeros((2, 32), np.float32)
    big[1, 0:16] = np.float32(3e38)                  # the butterflies overflow: NONFINITE
    out["overflow"] = big
    n = rng.normal(size=(4, 64)).astype(np.float32)
    n[2, 7] = np.nan
    out["nan"] = n
    return out


@pytest.mark.parametrize("name", list(_edge_tensors()))
@pytest.mark.parametrize("method", ["absmax", "four_over_six", "sweep_mse", "if4"])
def test_rotated_edge_tensors(name, method):
    x = _edge_tensors()[name]
    fmt = "if4" if method == "if4" else "nvfp4"
    gc, gsc, gS, st, _ = run(torch.from_numpy(x).cuda(), fmt, method)
    r = oracle_run(x, fmt, method)
    assert st == r["status"]
    assert bits(gS) == bits(r["S"]) or (np.isnan(gS) and np.isnan(r["S"]))
    same(gc, gsc, r)
    if name in ("overflow", "nan"):
        assert st == fq.DEVSTAT_NONFINITE and not gc.any() and not gsc.any()


def test_rotated_given_scale_subnormal_products():
    """A given S at the bottom of the range (2^-117) with inputs near 2^-122: about one rotated
    value in thirteen is subnormal, so the rotation's division by 4 rounds in the subnormal
    range, the block scales are E4M3 subnormals and every squared scale underflows to 0 (the
    sweep then keeps its lowest candidate, by the tie rule)."""
    rng = np.random.default_rng(5)
    x = (rng.uniform(-1, 1, size=(6, 128)) * 2.0 ** -122).astype(np.float32)
    S = 2.0 ** -117
    for fmt, obj in (("nvfp4", "sweep_mse"), ("nvfp4", "four_over_six"), ("if4", "absmax")):
        gc, gsc, _, st, _ = run(torch.from_numpy(x).cuda(), fmt, obj, S=S)
        r = oracle_run(x, fmt, obj, S=S)
        assert st == r["status"] == 0
        same(gc, gsc, r)
        assert np.any(gsc != 0)


@pytest.mark.parametrize("fmt,obj", [("nvfp4", "sweep_mse"), ("if4", None)])
def test_rotated_full_size_sampled(fmt, obj):
    """The 8192 x 4096 (NVFP4) and 4096 x 14336 (IF4) bf16 workloads, rotated: S over the
    whole tensor, codes and scales on 48 sampled rows."""
    w = synth.make("cfg3" if fmt == "nvfp4" else "cfg4")
    xd = to_dev(w)
    gc, gsc, gS, st, _ = run(xd, fmt, obj or "absmax")
    S, ost = O.tensor_scale(O.rotate16(oracle_x(w)))
    assert st == ost == 0 and bits(gS) == bits(S)
    rows = np.sort(np.random.default_rng(98).choice(w["rows"], size=48, replace=False))
    r = oracle_run(oracle_x(w, rows), fmt, obj, S=S)
    same(gc[rows], gsc[rows], r)
