"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes runs out, records its site in the device error word and returns; the
host reads HALO_ERR_TIMEOUT with the site, the word is cleared, and the context
keeps working (a rotate+quantise right after matches the oracle)."""
import pytest
import torch

import hadamard_rotated_precision_halo_b200 as halo
import oracle
from hadamard_rotated_precision_halo_b200 import inputs
from tests._parity import check_codes, oracle_operand

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported():
    assert halo.halo_device_error() == (halo.HALO_OK, 0)  # clean start
    st = halo.lib().halo_selftest_wait_timeout(20_000_000, None)  # 20 ms bound
    assert st == halo.HALO_OK
    st, site = halo.halo_device_error()
    assert st == halo.HALO_ERR_TIMEOUT and site == 0xF01
    assert halo.halo_device_error() == (halo.HALO_OK, 0)  # read once, then cleared
    # the context is still usable
    x = inputs.activations(64, 256, seed=5, device="cpu")
    q, s = halo.halo_hadamard_quantize(x.to("cuda"), halo.HALO_AXIS_COLS, 128, halo.HALO_Q_INT8)
    torch.cuda.synchronize()
    codes, scales, t = oracle_operand(x, 1, 128, halo.HALO_Q_INT8)
    check_codes(q, s, codes, scales, t, halo.HALO_Q_INT8, blk=128, axis=1)
    assert halo.halo_device_error() == (halo.HALO_OK, 0)
