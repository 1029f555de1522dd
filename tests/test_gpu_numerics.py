"""GPU checks of the elementwise building blocks against IEEE arithmetic."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _all_floats_1_to_2(dev):
    bits = torch.arange(0x3F800000, 0x40000001, dtype=torch.int64, device=dev).to(torch.int32)
    return bits.view(torch.float32)


@pytest.mark.parametrize("steps", [1, 2])
def test_sigmoid_reciprocal_is_ieee_on_every_input(cuda_lib, steps):
    # the sigmoid's reciprocal of 1 + exp(-|z|), refined from the hardware
    # approximation by Newton steps (the kernels use one), must equal IEEE 1/d
    # for every float d in [1, 2]
    lib = cuda_lib.load()
    dev = torch.device("cuda:0")
    d = _all_floats_1_to_2(dev)
    out = torch.empty_like(d)
    want = torch.div(torch.ones_like(d), d)          # IEEE division, round to nearest
    st = torch.cuda.current_stream(dev).cuda_stream
    assert lib.rn_test_rcp_1to2(d.numel(), d.data_ptr(), out.data_ptr(), steps, st) == 0
    torch.cuda.synchronize()
    bad = (out.view(torch.int32) != want.view(torch.int32)).sum().item()
    assert bad == 0, f"{bad} of {d.numel()} reciprocals differ from IEEE division"


def test_rcp_entry_point_rejects_bad_arguments(cuda_lib):
    lib = cuda_lib.load()
    assert lib.rn_test_rcp_1to2(-1, None, None, 2, None) != 0
    assert lib.rn_test_rcp_1to2(16, None, None, 2, None) != 0
    x = torch.ones(16, device="cuda:0")
    assert lib.rn_test_rcp_1to2(16, x.data_ptr(), x.data_ptr(), 3, None) != 0


def _sigmoid_inputs(dev):
    # about 86 million floats of each sign in [0, 110], every 13th bit pattern,
    # plus the ends: the whole normal range of the sigmoid, its subnormal tail
    # (z < -87.3) and the saturation to 1
    top = int(torch.tensor(110.0).view(torch.int32).item())
    pos = torch.arange(0, top + 1, 13, dtype=torch.int64, device=dev).to(torch.int32)
    z = pos.view(torch.float32)
    return torch.cat([z, -z])


def test_gate_sigmoid_error_bound(cuda_lib):
    # e^{-|z|} is CUDA's expf (within an ulp or two), 1 + e an IEEE add, its
    # reciprocal IEEE-exact (the test above) and e/(1+e) one IEEE multiply, so
    # s(z) lies within 8 ulp (2^-21 relative) of the exact sigmoid; subnormal
    # results (z < -87.3) within a few units of 2^-149 more.  Reference: the
    # fp64 sigmoid.
    lib = cuda_lib.load()
    dev = torch.device("cuda:0")
    z = _sigmoid_inputs(dev)
    out = torch.empty_like(z)
    st = torch.cuda.current_stream(dev).cuda_stream
    assert lib.rn_test_sigmoid(z.numel(), z.data_ptr(), out.data_ptr(), st) == 0
    torch.cuda.synchronize()
    ref = torch.sigmoid(z.double())
    lim = 2.0 ** -21 * ref + 4 * 2.0 ** -149
    err = (out.double() - ref).abs()
    bad = err > lim
    n_bad = int(bad.sum().item())
    if n_bad:
        i = int(torch.argmax((err / lim).masked_fill(~bad, 0)).item())
        raise AssertionError(f"{n_bad} of {z.numel()} sigmoids outside the bound; worst z="
                             f"{z[i].item()!r}: got {out[i].item()!r}, exact {ref[i].item()!r}")


def test_gate_sigmoid_special_values(cuda_lib):
    lib = cuda_lib.load()
    dev = torch.device("cuda:0")
    z = torch.tensor([float("inf"), float("-inf"), float("nan"), 0.0, -0.0, 200.0, -200.0],
                     device=dev)
    out = torch.empty_like(z)
    st = torch.cuda.current_stream(dev).cuda_stream
    assert lib.rn_test_sigmoid(z.numel(), z.data_ptr(), out.data_ptr(), st) == 0
    torch.cuda.synchronize()
    o = out.tolist()
    assert o[0] == 1.0 and o[1] == 0.0 and o[2] != o[2]
    assert o[3] == 0.5 and o[4] == 0.5           # 1 / (1 + 1), exactly
    assert o[5] == 1.0 and o[6] == 0.0           # e^-200 is below the smallest subnormal


def test_sigmoid_entry_point_rejects_bad_arguments(cuda_lib):
    lib = cuda_lib.load()
    assert lib.rn_test_sigmoid(-1, None, None, None) != 0
    assert lib.rn_test_sigmoid(16, None, None, None) != 0
