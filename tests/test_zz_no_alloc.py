"""ear_permute_static: the permutation for callers that cannot allocate device
memory (its scratch is a fixed array inside libear).  Called straight
through the C ABI and checked against ear_permute's results, on two calls in
a row with different shapes, so stale contents of the shared array would
show.  This file is named to be collected last."""
import ctypes

import numpy as np
import pytest
import torch

from clustered_block_sparse_b200 import _native as N
from clustered_block_sparse_b200 import ear
from clustered_block_sparse_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from clustered_block_sparse_b200 import build
    build.build()


def _static_via_abi(labels, c, x, want_mean):
    """Calls the C entry point directly with ctypes; outputs allocated here."""
    bh, n = labels.shape
    perm = torch.empty((bh, n), dtype=torch.int32, device="cuda")
    off = torch.empty((bh, c + 1), dtype=torch.int32, device="cuda")
    xp = torch.empty_like(x)
    mean = torch.empty((bh, c, x.shape[2]), dtype=torch.float32, device="cuda") if want_mean else None
    dt = N.EAR_BF16 if x.dtype == torch.bfloat16 else N.EAR_F32
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    status = N.lib().ear_permute_static(
        vp(labels), bh, n, c, vp(perm), vp(off), vp(x), vp(xp), dt, x.shape[2], vp(mean),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == N.EAR_OK, N.lib().ear_status_string(status)
    return perm, off, xp, mean


CASES = [  # (slices, tokens, clusters, dtype, d): the first is a Wan-sized key layer slice
    (8, 75600, 500, "bf16", 128),
    (3, 10001, 37, "f32", 64),
]


def test_static_permute_matches_workspace_permute_on_two_calls():
    rng = np.random.default_rng(2024)
    for bh, n, c, dtype, d in CASES:
        labels = rng.integers(0, c, (bh, n)).astype(np.int32)
        labels[labels == 3] = 4  # an empty cluster
        x_host = gen.round_to_dtype(rng.standard_normal((bh, n, d)), dtype)
        lab = torch.from_numpy(labels).cuda()
        x = torch.from_numpy(x_host).to("cuda", torch.bfloat16 if dtype == "bf16" else torch.float32)
        p_s, o_s, x_s, m_s = _static_via_abi(lab, c, x, True)
        p_w, o_w, x_w, m_w = ear.ear_permute(lab, c, x, seg_mean=True)
        torch.cuda.synchronize()
        assert torch.equal(p_s, p_w) and torch.equal(o_s, o_w) and torch.equal(x_s, x_w)
        ref = m_w.cpu().numpy()
        np.testing.assert_allclose(m_s.cpu().numpy(), ref, rtol=0,
                                   atol=1e-6 * max(np.abs(ref).max(), 1.0))
    assert ear.ear_get_device_status() == 0


def test_static_permute_rejects_a_problem_larger_than_its_array():
    # 65,535 slices x 65,536 clusters needs far more than the fixed array: refused on the host
    fake = ctypes.c_void_p(0x10000)
    status = N.lib().ear_permute_static(fake, 65535, 1 << 20, 65536, fake, fake, None, None, 0, 0,
                                        None, None)
    assert status == N.EAR_ERR_WORKSPACE
    need = N.workspace_bytes(N.EAR_OP_PERMUTE, 40, 75600, 0, 128, 500, 0)
    assert need <= N.PERMUTE_STATIC_MAX_BYTES


def test_static_permute_allocates_no_device_memory():
    """The entry point's defining property: with its outputs already allocated,
    a Wan-sized call (40 slices x 75,600 tokens in 500 clusters, which needs
    about 6 MB of scratch) leaves the device's free memory unchanged."""
    rng = np.random.default_rng(7)
    bh, n, c, d = 40, 75600, 500, 128
    lab = torch.from_numpy(rng.integers(0, c, (bh, n)).astype(np.int32)).cuda()
    x = torch.randn((bh, n, d), device="cuda").to(torch.bfloat16)
    _static_via_abi(lab, c, x, True)  # first call on this device: loads the module
    torch.cuda.synchronize()
    perm = torch.empty((bh, n), dtype=torch.int32, device="cuda")
    off = torch.empty((bh, c + 1), dtype=torch.int32, device="cuda")
    xp = torch.empty_like(x)
    mean = torch.empty((bh, c, d), dtype=torch.float32, device="cuda")
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        status = N.lib().ear_permute_static(
            vp(lab), bh, n, c, vp(perm), vp(off), vp(x), vp(xp), N.EAR_BF16, d, vp(mean),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert status == N.EAR_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    assert ear.ear_get_device_status() == 0
