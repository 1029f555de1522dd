"""One process, two GPUs: kernels whose dynamic shared memory exceeds the 48 KB
default are prepared on every device the process uses (the attribute is a
property of a device), and give bitwise the same results on each (PR #468's
device-guard check: bitwise-equal results on cuda:1).  Skipped with one GPU."""
import pytest
import torch

from gpu_util import run
from rollout_parity_b200 import workloads

pytestmark = pytest.mark.gpu


def bits(t):
    return t.view(torch.int32 if t.dtype == torch.float32 else torch.int16)


@pytest.mark.parametrize("op,rows,width", [("norm", 1024, 8192), ("gated", 300, 5120),
                                           ("gated", 4096, 128)])
def test_same_bits_on_two_devices(cuda_lib, op, rows, width):
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two GPUs in one process")
    host = workloads.make(op, rows, width, "bf16", seed=width)
    outs = []
    for dev in ("cuda:0", "cuda:1"):
        with torch.cuda.device(dev):
            out = run(cuda_lib, host.to(dev))
            torch.cuda.synchronize()
            outs.append({k: None if v is None else v.cpu() for k, v in out.items()})
    for k in ("y", "rstd", "dx", "dz", "dw"):
        if outs[0][k] is not None:
            assert torch.equal(bits(outs[0][k]), bits(outs[1][k])), k
