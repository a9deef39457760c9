"""Failure detection without a GPU fault: a bounded wait that nothing
completes must give up, latch EAR_ERR_TIMEOUT in the device status word and
leave the context usable (the next calls run and report EAR_OK)."""
import numpy as np
import pytest

from clustered_block_sparse_b200 import inputs as gen


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_survives():
    import torch

    from clustered_block_sparse_b200 import _native as N
    from clustered_block_sparse_b200 import ear

    assert ear.ear_get_device_status() == N.EAR_OK  # also clears anything earlier
    ear.ear_selftest_wait_timeout()
    assert ear.ear_get_device_status() == N.EAR_ERR_TIMEOUT
    assert ear.ear_get_device_status() == N.EAR_OK  # read-and-clear

    # the context still runs the path: one small layer, status clean
    w = gen.TINY
    layer = gen.make_layer(w)
    q, k, v = (torch.from_numpy(a).cuda() for a in (layer.q, layer.k, layer.v))
    qi, ki = torch.from_numpy(layer.q_init).cuda(), torch.from_numpy(layer.k_init).cuda()
    res = ear.ear_layer(q, k, v, qi, ki, w.iters, w.density)
    torch.cuda.synchronize()
    assert ear.ear_get_device_status() == N.EAR_OK
    assert np.isfinite(res.o.float().cpu().numpy()).all()
