"""Several host threads, each on its own CUDA stream, calling the library at the
same time: every call gives bitwise the outputs of the same call made alone.  The
host side keeps no per-call state outside the call (the launch counter is per
thread, the kernel preparation caches are atomic), the kernels touch only their
own buffers, and every launch goes to the stream the call names."""
import threading

import pytest
import torch

from gpu_util import run
from rollout_parity_b200 import workloads

pytestmark = pytest.mark.gpu

# one shape per kernel family: narrow stripe, register-path k_bwd, lean k_bwd
# (fp16, sigmoid, offset 1), the H = 256 stripe, 512-thread teams; ragged rows
CASES = [
    dict(op="gated", rows=4133, width=128, dtype="bf16"),
    dict(op="norm", rows=3000, width=2048, dtype="bf16"),
    dict(op="general", rows=777, width=5120, dtype="f16", act="sigmoid", weight_offset=1.0),
    dict(op="norm", rows=20000, width=256, dtype="bf16"),
    dict(op="gated", rows=300, width=8192, dtype="bf16"),
]
KEYS = ("y", "rstd", "dx", "dz", "dw")


def bits(t):
    return t.view(torch.int32 if t.dtype == torch.float32 else torch.int16)


def test_threads_on_streams_give_the_serial_bits(cuda_lib):
    dev = torch.device("cuda:0")
    wls = [workloads.make(seed=31 + i, **c).to(dev) for i, c in enumerate(CASES)]
    want = []
    for wl in wls:
        out = run(cuda_lib, wl)
        torch.cuda.synchronize()
        want.append({k: None if out[k] is None else out[k].clone() for k in KEYS})

    reps = 6
    got = [[None] * reps for _ in wls]
    errors = []
    start = threading.Barrier(len(wls))

    def worker(i):
        try:
            s = torch.cuda.Stream(dev)
            start.wait(timeout=60)
            with torch.cuda.stream(s):
                for r in range(reps):
                    got[i][r] = run(cuda_lib, wls[i])
            s.synchronize()
        except Exception as e:          # reported on the main thread
            errors.append((i, repr(e)))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(wls))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads), "a worker did not finish"
    assert not errors, errors
    torch.cuda.synchronize()
    for i, c in enumerate(CASES):
        for r in range(reps):
            for k in KEYS:
                if want[i][k] is None:
                    assert got[i][r][k] is None, (c, k)
                    continue
                assert torch.equal(bits(got[i][r][k]), bits(want[i][k])), (c, r, k)


def test_one_stream_per_call_in_turn(cuda_lib):
    """Independent calls alternating between two streams of one thread (nothing
    orders one stream's calls after the other's): each gives the serial bits."""
    dev = torch.device("cuda:0")
    wl = workloads.make("gated", 2049, 128, "bf16", seed=5).to(dev)
    ref = run(cuda_lib, wl)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    outs = []
    for j in range(6):
        s = streams[j % 2]
        with torch.cuda.stream(s):
            outs.append(run(cuda_lib, wl))
    torch.cuda.synchronize()
    for out in outs:
        for k in KEYS:
            if ref[k] is not None:
                assert torch.equal(bits(out[k]), bits(ref[k])), k


@pytest.mark.parametrize("case", [CASES[0], CASES[1], CASES[2]],
                         ids=["stripe", "k_bwd", "lean-f16"])
def test_graph_replay_gives_the_eager_bits(cuda_lib, case):
    """The calls captured into a CUDA graph (as bench.py replays them) and the
    graph replayed give the bits of the calls made eagerly."""
    dev = torch.device("cuda:0")
    wl = workloads.make(seed=77, **case).to(dev)
    ref = run(cuda_lib, wl)
    torch.cuda.synchronize()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        out = run(cuda_lib, wl)
    for _ in range(3):
        for k in KEYS:
            if out[k] is not None:
                out[k].fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for k in KEYS:
            if ref[k] is not None:
                assert torch.equal(bits(out[k]), bits(ref[k])), (case, k)
