"""The oracle against its pins (CPU only; see oracle_pins.py for what pins what)."""
import os, sys
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import pytest

import oracle
from oracle_pins import ALL_PINS
from oracle_pins_attention import ATTENTION_PINS
from oracle_pins_elementwise import ELEMENTWISE_PINS


@pytest.fixture(scope="module")
def orc():
    return oracle._oracle()


@pytest.mark.parametrize("pin", ALL_PINS + ATTENTION_PINS + ELEMENTWISE_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_argument_errors(orc):
    import numpy as np
    A = np.zeros((2, 3), np.uint16)
    B = np.zeros((3, 4), np.uint16)
    with pytest.raises(ValueError):
        orc.gemm(A, B, None, oracle.F16, oracle.EPI_BIAS_GELU)
    with pytest.raises(ValueError):
        orc.gemm(A, np.zeros((4, 3), np.uint16))
    with pytest.raises(ValueError):
        orc.gemm(A, B, rows=[2])
    with pytest.raises(ValueError):
        orc.gemm_points(A, B, None, oracle.F16, oracle.EPI_NONE, [0], [4])
    with pytest.raises(TypeError):
        orc.gemm(A.astype(np.float32), B)
