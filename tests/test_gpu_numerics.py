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
