"""The parity tests' output criterion, checked on the host (no GPU)."""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_out_close


def bf16(x):
    return torch.tensor(x, dtype=torch.float64).to(torch.bfloat16).double().numpy()


def test_correctly_rounded_large_outputs_pass():
    # |ref| = 4.23: the nearest bf16 value is 0.012 away, beyond the 1e-2 bound
    ref = np.array([-4.23072684079268, 3.1, 0.5])
    assert assert_out_close(bf16(ref), ref, torch.bfloat16) > 1e-2


def test_small_outputs_keep_the_absolute_bound():
    ref = np.array([1.0, 0.25])
    with pytest.raises(AssertionError):
        assert_out_close(ref + np.array([0.011, 0.0]), ref, torch.bfloat16)
    assert_out_close(ref + np.array([0.0099, 0.0]), ref, torch.bfloat16)
    with pytest.raises(AssertionError):
        assert_out_close(ref + np.array([0.0021, 0.0]), ref, torch.float16)


def test_large_outputs_allow_one_ulp_only():
    # ref lies between the bf16 values -4.25 and -4.21875 (spacing 2^-5): both
    # neighbours are within one ulp, the next one out (-4.1875) is not
    ref = np.array([-4.23072684079268])
    assert_out_close(np.array([-4.25]), ref, torch.bfloat16)
    assert_out_close(np.array([-4.21875]), ref, torch.bfloat16)
    with pytest.raises(AssertionError):
        assert_out_close(np.array([-4.1875]), ref, torch.bfloat16)
