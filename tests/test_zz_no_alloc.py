"""effort_gemv_static, the entry point whose scratch is the library's fixed
per-device array, against effort_gemv_ex on the same handle and inputs.

Both run the same kernel, so cutoff and |S| must agree bit for bit and out
within the parity tolerance of the other GPU tests.  Two static calls run
back to back (different vectors and efforts) to show that the words the call
clears at its start leave no state behind.  This file is collected last so
that it also runs after every other test in the same process; it passes
alone as well.
"""
import ctypes

import numpy as np
import pytest
import torch

from dynamic_approximate_gemv_b200 import inputs

REL_L2 = 1e-4
MAX_ABS = 1e-3


@pytest.fixture(scope="module")
def E():
    from dynamic_approximate_gemv_b200 import build
    build.build()
    import dynamic_approximate_gemv_b200 as E
    E.lib()
    return E


def test_static_entry_rejects_bad_arguments_without_a_device(E):
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: validation fails first
    L = E.lib()
    assert L.effort_gemv_static(None, fake, 0, ctypes.c_float(0.5), fake, None, None, None, None) == 1


def close(got, ref):
    got = got.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    nref = np.linalg.norm(ref)
    assert np.linalg.norm(got - ref) <= REL_L2 * nref
    assert np.max(np.abs(got - ref)) <= MAX_ABS * np.max(np.abs(ref))


def one_pair(pm, v, effort):
    dev = v.device
    c0 = torch.empty(1, device=dev, dtype=torch.float32)
    n0 = torch.full((1,), -1, device=dev, dtype=torch.int64)
    c1 = torch.empty(1, device=dev, dtype=torch.float32)
    n1 = torch.full((1,), -1, device=dev, dtype=torch.int64)
    st = torch.full((1,), -1, device=dev, dtype=torch.int32)
    ref = pm.gemv(v, effort, cutoff=c0, count=n0)
    got = pm.gemv_static(v, effort, cutoff=c1, count=n1, status=st)
    torch.cuda.synchronize()
    pm.check()
    assert int(st.item()) == 0
    assert c0.view(torch.int32).item() == c1.view(torch.int32).item()
    assert int(n0.item()) == int(n1.item()) > 0
    close(got, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("I,Od,keep", [(2048, 5000, 1.0), (4096, 14336, 1.0), (14336, 4096, 1.0)])
def test_static_matches_workspace_entry_two_calls(E, I, Od, keep):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    W = torch.from_numpy(inputs.weights(I, Od, 11)).cuda()
    pm = E.PreparedMatrix(W, keep)
    try:
        v1 = torch.from_numpy(inputs.vector(I, 12, "t3")).cuda()
        v2 = torch.from_numpy(inputs.vector(I, 13, "normal", np.float16)).cuda()
        one_pair(pm, v1, 0.25)
        one_pair(pm, v2, 0.1)
    finally:
        pm.close()


@pytest.mark.gpu
def test_static_reports_nonfinite_v(E):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    I, Od = 512, 768
    pm = E.PreparedMatrix(torch.from_numpy(inputs.weights(I, Od, 21)).cuda(), 1.0)
    try:
        v = torch.from_numpy(inputs.vector(I, 22)).cuda()
        v[7] = float("nan")
        st = torch.zeros(1, device="cuda", dtype=torch.int32)
        pm.gemv_static(v, 0.5, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) != 0
        v[7] = 1.0
        pm.gemv_static(v, 0.5, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
    finally:
        pm.close()


@pytest.mark.gpu
def test_static_calls_allocate_no_device_memory(E):
    """Many static calls change neither the device's free memory nor the
    memory the library holds (one warm-up call first: the first call on a
    device looks up the array's address)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    I, Od = 4096, 14336
    pm = E.PreparedMatrix(torch.from_numpy(inputs.weights(I, Od, 31)).cuda(), 1.0)
    try:
        v = torch.from_numpy(inputs.vector(I, 32, "t3")).cuda()
        out = torch.empty(Od, device="cuda")
        pm.gemv_static(v, 0.25, out=out)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        held0 = E.device_bytes_held()
        for k in range(50):
            pm.gemv_static(v, 0.05 + 0.01 * (k % 20), out=out)
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert free1 == free0
        assert E.device_bytes_held() == held0
    finally:
        pm.close()
