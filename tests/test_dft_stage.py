"""GPU checks of hyena_dft32_stage, the measurement of one radix-32 FFT
level on the FP32 pipes and on the tcgen05 tensor cores: both methods must
compute the scaled 32-point DFT (numpy's FFT on the same inputs), and four
applications must give the input back."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hy():
    from subquadratic_sequence_b200 import hyena
    assert torch.cuda.is_available()
    return hyena


def _x(count, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((count, 32)) + 1j * rng.standard_normal((count, 32))).astype(np.complex64)


@pytest.mark.parametrize("method", [0, 1])
@pytest.mark.parametrize("count", [1, 127, 128, 1000, 40000])
def test_one_application_is_the_scaled_dft(hy, method, count):
    x = _x(count, count + method)
    y = hy.hyena_dft32_stage(torch.from_numpy(x).cuda(), 1, method).cpu().numpy()
    ref = np.fft.fft(x.astype(np.complex128), axis=1) / np.sqrt(32.0)
    assert np.max(np.abs(y - ref)) <= 2e-6 * np.max(np.abs(ref))
    assert hy.LIB.hyena_device_fault_count() == 0


@pytest.mark.parametrize("method", [0, 1])
def test_four_applications_give_the_input_back(hy, method):
    x = _x(5000, 3)
    y = hy.hyena_dft32_stage(torch.from_numpy(x).cuda(), 8, method).cpu().numpy()
    assert np.max(np.abs(y - x)) <= 1e-5 * np.max(np.abs(x))


def test_methods_agree(hy):
    x = torch.from_numpy(_x(3000, 4)).cuda()
    a = hy.hyena_dft32_stage(x, 3, 0).cpu().numpy()
    b = hy.hyena_dft32_stage(x, 3, 1).cpu().numpy()
    assert np.max(np.abs(a - b)) <= 2e-6 * np.max(np.abs(a))
