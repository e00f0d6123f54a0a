"""The row-sharded quantization (dist.sharded_quantize) on the B200 over an NCCL process group.
Every run on this pool has one GPU, so the group has one rank: the all-reduce-MAX of S goes
through NCCL on the device, and the result must equal the single call bit for bit.  The
two-rank exchange itself is covered on CPU by test_dist_gloo.py."""
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import fp4_block_scaled_nvfp4_b200 as fq
from fp4_block_scaled_nvfp4_b200 import dist as fdist
from fp4_block_scaled_nvfp4_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import datetime
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    yield dist
    dist.destroy_process_group()


@pytest.mark.parametrize("fmt,obj,had16", [("nvfp4", "sweep_mse", False), ("nvfp4", "sweep_mse", True),
                                           ("if4", "absmax", False), ("if6", "absmax", False),
                                           ("mxfp4", "absmax", False)])
def test_sharded_quantize_over_nccl_matches_the_single_call(nccl_group, fmt, obj, had16):
    w = synth.make("cfg3", rows=256, cols=4096)
    x = torch.from_numpy(w["x"].view(np.int16)).view(torch.bfloat16).cuda()
    c1, s1, g1 = fdist.sharded_quantize(x, fmt, obj, hadamard16=had16)
    c0, s0, g0 = fq.quantize(x, fmt, obj, hadamard16=had16)
    torch.cuda.synchronize()
    assert torch.equal(c1, c0) and torch.equal(s1, s0)
    if fmt != "mxfp4":
        assert torch.equal(g1.view(torch.int32), g0.view(torch.int32))
    # the reduction carries a NaN scale through as NaN
    s_nan = fdist.reduce_global_scale(torch.tensor([float("nan")], device="cuda"))
    assert torch.isnan(s_nan).all()
