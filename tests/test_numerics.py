"""The exponential the softmax kernels use: the special-function unit's
ex2.approx, run on the device through lg_exp2_device and compared with exact
2^x (relative error within 2^-21 over the range the softmax produces, exact
zero for -inf, the value masked entries carry). On the host: the call rejects
any other method.
"""

import pytest
import torch


def test_only_the_hardware_method_exists():
    import ctypes

    import attention_sink_long_b200 as lg

    L = lg.lib()
    for method in (1, 2, -1):
        assert L.lg_exp2_device(ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000), 16, method, None) == 1


@pytest.mark.gpu
def test_device_exponential_against_exact():
    import attention_sink_long_b200 as lg

    xs = torch.linspace(-126.0, 64.0, 2_000_003, dtype=torch.float32)
    xs = torch.cat([xs, torch.tensor([0.0, -0.5, 0.5, -1e-7, 1e-7, -8.0, 8.0])])
    x = xs.cuda()
    exact = torch.exp2(xs.double())
    y = torch.empty_like(x)
    lg.lg_exp2_device(x, y, 0)
    torch.cuda.synchronize()
    rel = (y.double().cpu() / exact - 1.0).abs()
    assert rel.max().item() < 2.0 ** -21, rel.max().item()
    z = torch.tensor([-float("inf"), -500.0], device="cuda")
    y = torch.empty_like(z)
    lg.lg_exp2_device(z, y, 0)
    torch.cuda.synchronize()
    assert torch.all(y == 0), y
