"""Failure detection without a GPU fault: a wait that nothing completes runs
out after a short bound, the kernel returns, the host reads SQ_ERR_TIMEOUT,
and the context stays usable for ordinary work afterwards."""
import numpy as np
import pytest
import torch

import oracle
import w8a8_post_quantization_channel_b200 as sq
from w8a8_post_quantization_channel_b200 import synth


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_device_stays_usable():
    assert sq.sq_check_device_error() == sq.SQ_OK  # nothing pending
    assert sq.sq_selftest_wait_timeout(100) == sq.SQ_OK  # launch accepted
    assert sq.sq_check_device_error() == sq.SQ_ERR_TIMEOUT
    assert sq.sq_check_device_error() == sq.SQ_OK  # the report clears it
    # ordinary work still runs and is still exact
    x = synth.activations(8, 256, synth.outliers(256, count=2, seed=1), seed=2)
    inv = torch.ones(256)
    xq, xs = sq.sq_quant_act(x.cuda(), inv.cuda())
    xq_ref, xs_ref = oracle.quant_act(x.numpy(), inv.numpy())
    np.testing.assert_array_equal(xq.cpu().numpy(), xq_ref)
    assert sq.sq_check_device_error() == sq.SQ_OK


def test_selftest_rejects_out_of_range_limits():
    # host-side checks only (no CUDA call is made): runs without a GPU
    f = sq.lib().sq_selftest_wait_timeout
    assert f(0, None) == sq.SQ_ERR_INVALID_ARG
    assert f(6000, None) == sq.SQ_ERR_INVALID_ARG
