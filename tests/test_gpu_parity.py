"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element.

Bar: codes, scale bytes (including the IF4 indicator) and S are bit-exact; dequantized
values are bit-exact (NaN compared as NaN); reconstruction MSE agrees to 1e-6 relative.
Inputs are the seeded synthetic workloads (fp4_block_scaled_nvfp4_b200.synth) at sizes the
oracle finishes in seconds (several thread-blocks' worth of quantization blocks and ragged
shapes), the full workload sizes on sampled rows, and edge tensors.
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
    """Workload -> CUDA tensor in its storage dtype."""
    if w["dtype"] == "bf16":
        return torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(w["x"])).cuda()


def oracle_x(w, rows=None):
    x = O.widen_bf16(w["x"]) if w["dtype"] == "bf16" else np.asarray(w["x"], np.float32)
    return x if rows is None else x[rows]


def run_gpu(xd, fmt, obj="sweep_mse", imp=None, S=None, ocp=False, had=False, mx_sweep=False, if4_sweep=False,
            had16=False):
    ws = fq.new_workspace()
    impd = None if imp is None else torch.from_numpy(np.ascontiguousarray(imp)).cuda()
    gs = None if S is None else torch.tensor([S], dtype=torch.float32, device="cuda")
    if had:
        codes, scales = fq.hadamard_quantize(xd, mx_ocp_floor=ocp, workspace=ws, mx_sweep=mx_sweep)
        out = (codes, scales, None)
    else:
        out = fq.quantize(xd, fmt, obj, importance=impd, global_scale=gs, mx_ocp_floor=ocp, workspace=ws,
                          mx_sweep=mx_sweep, if4_sweep=if4_sweep, hadamard16=had16)
    torch.cuda.synchronize()
    st = fq.read_device_status(ws)
    c, s, g = out
    return c.cpu().numpy(), s.cpu().numpy(), (None if g is None else float(g.cpu()[0])), st, out


def f32_bits(v):
    return np.float32(v).view(np.uint32)


def assert_same_codes(gc, gs, oc, os_):
    if not np.array_equal(gs, os_):
        bad = np.argwhere(gs != os_)
        raise AssertionError(f"{len(bad)} scale bytes differ, first {bad[:5].tolist()}: gpu {gs[tuple(bad[0])]:#x} "
                             f"oracle {os_[tuple(bad[0])]:#x}")
    if not np.array_equal(gc, oc):
        bad = np.argwhere(gc != oc)
        raise AssertionError(f"{len(bad)} code bytes differ, first {bad[:5].tolist()}")


def check_dequant(out, S, fmt, oc, os_, had=False):
    codes, scales, gs = out
    if fmt != "mxfp4" and gs is None:
        gs = torch.tensor([S], dtype=torch.float32, device="cuda")
    for bf in (False, True):
        xd = fq.dequantize(codes, scales, gs, fmt, inverse_hadamard=had,
                           out_dtype=torch.bfloat16 if bf else torch.float32)
        torch.cuda.synchronize()
        got = xd.view(torch.int16).cpu().numpy().view(np.uint16) if bf else xd.cpu().numpy()
        ref = O.dequantize(oc, os_, S if S is not None else 0.0, fmt, inverse_hadamard=had, out_bf16=bf)
        if bf:
            assert np.array_equal(got, ref)
        else:
            nan = np.isnan(ref)
            assert np.array_equal(np.isnan(got), nan)
            assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def recon_mse(x, xh):
    d = x.astype(np.float64) - xh.astype(np.float64)
    return float(np.mean(d * d))


# ------------------------------------------------------------------------------------------
# small / ragged sizes, every method
# ------------------------------------------------------------------------------------------
NV_CASES = [
    ("cfg1", None, None, "absmax"), ("cfg1", None, None, "four_over_six"), ("cfg1", None, None, "sweep_mse"),
    ("cfg3", 96, 4096, "sweep_mse"), ("cfg3", 33, 1024, "absmax"), ("cfg3", 33, 1024, "four_over_six"),
    ("cfg3", 7, 48, "sweep_mse"), ("cfg3", 1, 16, "sweep_mse"), ("cfg2", 40, 4096, "sweep_wmse"),
    ("cfg2", 5, 4096, "sweep_mse"), ("cfg4", 16, 14336, "sweep_mse"),
]


@pytest.mark.parametrize("cfg,rows,cols,obj", NV_CASES)
def test_nvfp4_parity(cfg, rows, cols, obj):
    w = synth.make(cfg, rows=rows, cols=cols)
    imp = w["importance"][: w["cols"]] if obj == "sweep_wmse" else None
    gc, gsc, gS, st, out = run_gpu(to_dev(w), "nvfp4", obj, imp=imp)
    x = oracle_x(w)
    r = O.nvfp4_quantize(x, obj, importance=imp)
    assert st == 0 and r["status"] == 0
    assert f32_bits(gS) == f32_bits(r["S"])
    assert_same_codes(gc, gsc, r["codes"], r["scales"])
    check_dequant(out, r["S"], "nvfp4", r["codes"], r["scales"])
    xh = O.dequantize(r["codes"], r["scales"], r["S"], "nvfp4")
    xg = fq.dequantize(out[0], out[1], out[2], "nvfp4").cpu().numpy()
    assert abs(recon_mse(x, xg) - recon_mse(x, xh)) <= 1e-6 * recon_mse(x, xh)


@pytest.mark.parametrize("cfg,rows,cols", [("cfg4", 24, 14336), ("cfg4", 3, 48), ("cfg3", 17, 2048), ("cfg1", None, None)])
def test_if4_parity(cfg, rows, cols):
    w = synth.make(cfg, rows=rows, cols=cols)
    gc, gsc, gS, st, out = run_gpu(to_dev(w), "if4")
    r = O.if4_quantize(oracle_x(w))
    assert st == 0 and f32_bits(gS) == f32_bits(r["S"])
    assert_same_codes(gc, gsc, r["codes"], r["scales"])
    check_dequant(out, r["S"], "if4", r["codes"], r["scales"])
    assert 0 < np.mean(gsc >> 7) < 1


@pytest.mark.parametrize("had", [False, True])
@pytest.mark.parametrize("ocp", [False, True])
@pytest.mark.parametrize("cfg,rows,cols", [("cfg5", 24, 8192), ("cfg5", 5, 96), ("cfg1", None, None)])
def test_mxfp4_parity(cfg, rows, cols, had, ocp):
    w = synth.make(cfg, rows=rows, cols=cols)
    gc, gsc, _, st, out = run_gpu(to_dev(w), "mxfp4", ocp=ocp, had=had)
    r = O.mxfp4_quantize(oracle_x(w), hadamard=had, ocp_floor=ocp)
    assert st == 0 and r["status"] == 0
    assert_same_codes(gc, gsc, r["codes"], r["scales"])
    check_dequant(out, None, "mxfp4", r["codes"], r["scales"], had=False)
    if had:
        check_dequant(out, None, "mxfp4", r["codes"], r["scales"], had=True)


@pytest.mark.parametrize("had16", [False, True])
@pytest.mark.parametrize("cfg,rows,cols", [("cfg4", 24, 14336), ("cfg4", 3, 48), ("cfg3", 17, 2048), ("cfg1", None, None)])
def test_if4_sweep_parity(cfg, rows, cols, had16):
    # IF4 x ScaleSweep (scale and type chosen together over the MSE window) against the oracle
    w = synth.make(cfg, rows=rows, cols=cols)
    gc, gsc, gS, st, out = run_gpu(to_dev(w), "if4", if4_sweep=True, had16=had16)
    x = oracle_x(w)
    r = O.if4_quantize(x, sweep="sweep", hadamard16=had16)
    a = O.if4_quantize(x, hadamard16=had16)
    assert st == 0 and f32_bits(gS) == f32_bits(r["S"])
    assert_same_codes(gc, gsc, r["codes"], r["scales"])
    check_dequant(out, r["S"], "if4", r["codes"], r["scales"], had=had16)
    assert (gsc != a["scales"]).any()


@pytest.mark.parametrize("had", [False, True])
@pytest.mark.parametrize("cfg,rows,cols", [("cfg5", 24, 8192), ("cfg5", 5, 96), ("cfg1", None, None)])
def test_mx_sweep_parity(cfg, rows, cols, had):
    # MX scale sweep (exponents e_c-2 .. e_c by block error) against the oracle, bit for bit
    w = synth.make(cfg, rows=rows, cols=cols)
    gc, gsc, _, st, out = run_gpu(to_dev(w), "mxfp4", had=had, mx_sweep=True)
    x = oracle_x(w)
    r = O.mxfp4_quantize(x, hadamard=had, sweep="sweep")
    assert st == 0 and r["status"] == 0
    assert_same_codes(gc, gsc, r["codes"], r["scales"])
    check_dequant(out, None, "mxfp4", r["codes"], r["scales"], had=had)
    rule = O.mxfp4_quantize(x, hadamard=had)["scales"].astype(int)
    moved = gsc.astype(int) - rule
    assert ((moved >= -2) & (moved <= 0)).all() and (moved != 0).any()


def test_padded_rows_and_given_scale():
    w = synth.make("cfg3", rows=16, cols=1024)
    full = torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda()
    padded = torch.zeros((16, 1024 + 64), dtype=torch.bfloat16, device="cuda")
    padded[:, :1024] = full
    view = padded[:, :1024]
    gc, gsc, gS, st, _ = run_gpu(view, "nvfp4", "sweep_mse")
    r = O.nvfp4_quantize(oracle_x(w), "sweep_mse")
    assert f32_bits(gS) == f32_bits(r["S"])
    assert_same_codes(gc, gsc, r["codes"], r["scales"])
    S = 0.37
    gc, gsc, _, st, _ = run_gpu(full, "nvfp4", "sweep_mse", S=S)
    r = O.nvfp4_quantize(oracle_x(w), "sweep_mse", S=S)
    assert st == r["status"] == 0
    assert_same_codes(gc, gsc, r["codes"], r["scales"])
    gc, gsc, _, st, _ = run_gpu(full, "if4", S=S)
    r = O.if4_quantize(oracle_x(w), S=S)
    assert_same_codes(gc, gsc, r["codes"], r["scales"])
    # IF4 and its sweep on the padded view, at the tensor's own S
    for sweep in (False, True):
        gc, gsc, gS, st, _ = run_gpu(view, "if4", if4_sweep=sweep)
        r = O.if4_quantize(oracle_x(w), sweep="sweep" if sweep else "absmax")
        assert st == r["status"] == 0 and f32_bits(gS) == f32_bits(r["S"])
        assert_same_codes(gc, gsc, r["codes"], r["scales"])
    # a given S far below the tensor's: base patterns saturate at 126, where the INT4 codes clamp
    S = float(np.float32(r["S"]) / np.float32(64))
    gc, gsc, _, st, _ = run_gpu(full, "if4", S=S)
    r = O.if4_quantize(oracle_x(w), S=S)
    assert st == r["status"]
    assert np.any((r["scales"] & 0x7F) == 0x7E)
    assert_same_codes(gc, gsc, r["codes"], r["scales"])


# ------------------------------------------------------------------------------------------
# edge tensors
# ------------------------------------------------------------------------------------------
def _edge_tensors():
    rng = np.random.default_rng(2024)
    out = {}
    out["zeros"] = np.zeros((4, 64), np.float32)
    z = np.zeros((4, 64), np.float32)
    z[1, ::3] = -0.0
    z[2, 17] = 3.0
    out["single_nonzero_signed_zeros"] = z
    t = rng.laplace(size=(8, 256)).astype(np.float32)
    t[3, 40] = 1e4                                   # the block holding the global max (p0 = 0x78)
    t[5, 16:32] *= 1e-7                              # subnormal-range base scales
    t[6, 32:48] = 0.0
    t[7, 48:64] = np.float32(2.0 ** -140)           # fp32 subnormal inputs
    out["mixed_ranges"] = t
    u = np.full((2, 32), 7.0, np.float32)
    u[1] = np.arange(32, dtype=np.float32) * 0.25 - 4   # exact E2M1 midpoints at S = 1 scale steps
    u[0, 0] = 1536.0
    out["ties"] = u
    # exact FP4/INT4 ties: one saturating outlier per block, every other |y| <= 0.25
    v = (rng.laplace(size=(8, 256)) * 0.02).astype(np.float32)
    v[:, ::16] = np.float32(102.5) * np.sign(rng.normal(size=(8, 16))).astype(np.float32)
    out["outlier_ties"] = v
    # exact sweep ties: [6*e, 0 ...] is reproduced exactly by two candidate scales
    t2 = np.zeros((4, 128), np.float32)
    t2[0, 0] = 1536.0                                   # S = 1
    for k, e in enumerate([1.0, 0.5, 2.0, 0.75, 1.25, 3.0, 0.375]):
        t2[1 + k % 3, 16 * (k + 1)] = np.float32(6 * e)
    out["sweep_ties"] = t2
    return out


@pytest.mark.parametrize("name", list(_edge_tensors()))
@pytest.mark.parametrize("method", ["absmax", "four_over_six", "sweep_mse", "sweep_wmse", "if4", "if4_sweep", "mxfp4",
                                    "mxfp4_had", "mxfp4_sweep", "mxfp4_had_sweep"])
def test_edge_tensors(name, method):
    x = _edge_tensors()[name]
    xd = torch.from_numpy(x).cuda()
    if method.startswith("mxfp4"):
        had, sw = "had" in method, method.endswith("sweep")
        gc, gsc, _, st, _ = run_gpu(xd, "mxfp4", had=had, mx_sweep=sw)
        r = O.mxfp4_quantize(x, hadamard=had, sweep="sweep" if sw else "rule")
    elif method.startswith("if4"):
        sw = method.endswith("sweep")
        gc, gsc, gS, st, _ = run_gpu(xd, "if4", if4_sweep=sw)
        r = O.if4_quantize(x, sweep="sweep" if sw else "absmax")
        assert f32_bits(gS) == f32_bits(r["S"])
    else:
        imp = np.linspace(0.01, 5, x.shape[1]).astype(np.float32) if method == "sweep_wmse" else None
        gc, gsc, gS, st, _ = run_gpu(xd, "nvfp4", method, imp=imp)
        r = O.nvfp4_quantize(x, method, importance=imp)
        assert f32_bits(gS) == f32_bits(r["S"])
    assert st == r["status"]
    assert_same_codes(gc, gsc, r["codes"], r["scales"])


def test_exact_roundtrip_every_representable_value():
    # with S = 1, a block whose maximum is 6 e(p) and whose other elements are the signed grid
    # values times e(p) selects pattern p under AbsMax and the sweep, and dequantizes bit-exactly:
    # every E2M1 x E4M3 value for the patterns AbsMax reaches (1 .. 0x78)
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0]
    blocks = []
    for p in range(1, 0x79):
        e = O.lib().fp4q_o_e4m3_value(p)
        vals = [6 * e] + [s * g * e for g in grid for s in (1, -1)] + [0.0]
        blocks.append(np.array(vals[:16], np.float32))
    x = np.concatenate(blocks).reshape(1, -1)
    for obj in ("absmax", "sweep_mse"):
        gc, gsc, gS, st, out = run_gpu(torch.from_numpy(x).cuda(), "nvfp4", obj)
        assert st == 0 and gS == 1.0
        if obj == "absmax":
            assert list(gsc[0]) == list(range(1, 0x79))
        xg = fq.dequantize(out[0], out[1], out[2], "nvfp4").cpu().numpy()
        assert np.array_equal(xg.view(np.uint32), x.view(np.uint32))


def test_bad_data_sets_status_and_zero_fills():
    x = np.random.default_rng(1).normal(size=(4, 64)).astype(np.float32)
    x[2, 7] = np.nan
    for fmt, obj in [("nvfp4", "sweep_mse"), ("if4", None)]:
        gc, gsc, gS, st, _ = run_gpu(torch.from_numpy(x).cuda(), fmt, obj or "absmax")
        assert st == fq.DEVSTAT_NONFINITE and np.isnan(gS)
        assert not gc.any() and not gsc.any()
    gc, gsc, _, st, _ = run_gpu(torch.from_numpy(x).cuda(), "mxfp4")
    r = O.mxfp4_quantize(x)
    assert st == fq.DEVSTAT_NONFINITE == r["status"]
    assert_same_codes(gc, gsc, r["codes"], r["scales"])
    tiny = np.full((2, 32), 1e-35, np.float32)
    gc, gsc, gS, st, _ = run_gpu(torch.from_numpy(tiny).cuda(), "nvfp4", "absmax")
    assert st == fq.DEVSTAT_RANGE and not gc.any()
    # the status word is per call: a clean call afterwards reports OK on the same workspace
    ws = fq.new_workspace()
    fq.quantize(torch.from_numpy(x).cuda(), "nvfp4", "absmax", workspace=ws)
    assert fq.read_device_status(ws) == fq.DEVSTAT_NONFINITE
    fq.quantize(torch.from_numpy(tiny * 0 + 1).cuda(), "nvfp4", "absmax", workspace=ws)
    assert fq.read_device_status(ws) == fq.DEVSTAT_OK
    assert not ws[4:].cpu().numpy().any()          # counters and scratch words are clean again


def test_launch_counts():
    x = torch.randn(8, 64, device="cuda")
    fq.quantize(x, "nvfp4", "sweep_mse")
    assert fq.last_launch_count() == 2
    fq.quantize(x, "nvfp4", "sweep_mse", global_scale=torch.ones(1, device="cuda"))
    assert fq.last_launch_count() == 1
    fq.quantize(x, "mxfp4")
    assert fq.last_launch_count() == 1


# ------------------------------------------------------------------------------------------
# full workload sizes, sampled rows
# ------------------------------------------------------------------------------------------
FULL = [("cfg2", "nvfp4", "sweep_wmse"), ("cfg3", "nvfp4", "sweep_mse"), ("cfg4", "if4", None), ("cfg4", "if4", "if4_sweep"),
        ("cfg5", "mxfp4", None), ("cfg5", "mxfp4_had", None), ("cfg5", "mxfp4", "mx_sweep"),
        ("cfg5", "mxfp4_had", "mx_sweep")]


@pytest.mark.parametrize("cfg,fmt,obj", FULL)
def test_full_size_sampled(cfg, fmt, obj):
    w = synth.make(cfg)
    xd = to_dev(w)
    rng = np.random.default_rng(99)
    rows = np.sort(rng.choice(w["rows"], size=48, replace=False))
    if fmt.startswith("mxfp4"):
        had, sw = fmt.endswith("had"), obj == "mx_sweep"
        gc, gsc, _, st, _ = run_gpu(xd, "mxfp4", had=had, mx_sweep=sw)
        r = O.mxfp4_quantize(oracle_x(w, rows), hadamard=had, sweep="sweep" if sw else "rule")
    else:
        imp = w.get("importance")
        gc, gsc, gS, st, _ = run_gpu(xd, fmt, obj or "absmax", imp=imp, if4_sweep=(obj == "if4_sweep"))
        S, ost = O.tensor_scale(oracle_x(w))
        assert ost == 0 and f32_bits(gS) == f32_bits(S)
        if fmt == "if4":
            r = O.if4_quantize(oracle_x(w, rows), S=S, sweep="sweep" if obj == "if4_sweep" else "absmax")
        else:
            r = O.nvfp4_quantize(oracle_x(w, rows), obj, importance=imp, S=S)
    assert st == 0
    assert_same_codes(gc[rows], gsc[rows], r["codes"], r["scales"])
