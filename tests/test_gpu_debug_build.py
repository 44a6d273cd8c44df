"""The bounds-checking build and the device error path.

libeffort_debug.so is the same library with every index a kernel takes from
data (rows, chunks, decoded columns) checked before use: a bad one sets a bit
of the handle's status word and the access is skipped, and effort_check then
returns EFFORT_ERR_DEVICE (5).  The test runs in a child process that loads
that build (EFFORT_DEBUG_LIB=1): a valid call matches the oracle, then one
gap byte of a stored chunk is changed so that a used slot decodes to a column
past its panel (at most 255 past, so the access would stay inside the block's
shared memory even unchecked) and the next call must report it.

The grid-wide waits have a time limit: a test hook makes the barrier count
unreachable, the call ends with the timeout bit set, effort_check reports
EFFORT_ERR_DEVICE and restarts the scratch, and the following call is right.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from dynamic_approximate_gemv_b200 import inputs
from oracle import effort_oracle as O

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import os, sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
import dynamic_approximate_gemv_b200 as E
from dynamic_approximate_gemv_b200 import build, inputs
from oracle import effort_oracle as O
build.build()
L = E.lib()
assert os.path.basename(L._name) == os.path.basename(E.LIB_DEBUG_PATH), L._name
I, Od, effort = 256, 2048, 0.25
Wn = inputs.weights(I, Od, 91)
v = inputs.vector(I, 92)
prep = O.Prepared(Wn.view(np.uint16), 1.0)
pm = E.PreparedMatrix(torch.from_numpy(Wn).cuda(), 1.0)
cut = torch.empty(1, device="cuda")
cnt = torch.zeros(1, device="cuda", dtype=torch.int64)
out = pm.gemv(torch.from_numpy(v).cuda(), effort, cutoff=cut, count=cnt)
pm.check()
ref = O.effort_gemv(prep, v, effort)
assert np.float32(cut.item()).view(np.uint32) == np.float32(ref.c).view(np.uint32)
assert int(cnt.item()) == ref.count
got = out.cpu().numpy().astype(np.float64)
assert np.linalg.norm(got - ref.out) <= 1e-4 * np.linalg.norm(ref.out)
# a row read as stored chunks whose first chunk is used whole
lay = pm.layout()
lists = lay["lists"].cpu().numpy()
gaps = lay["gaps"]
g_host = gaps.cpu().numpy().astype(np.int64)
v_host = lay["vals"].cpu().numpy()
target = None
for r in np.argsort(np.abs(v)):
    if not (100 <= ref.L[r] <= 600):
        continue
    c0 = int(lists[r, 0, 0])
    g = g_host[c0 * 64:(c0 + 1) * 64]
    cols = np.cumsum(g) - 1
    if cols[62] >= 1793 and g[63] > 0 and v_host[c0 * 64 + 63] != 0:
        target = (c0 * 64 + 63, int(g[63]))
        break
assert target is not None
gaps[target[0]] = 255  # slot 63 now decodes to cols[62] + 255 > 2047
pm.gemv(torch.from_numpy(v).cuda(), effort)
try:
    pm.check()
    raise SystemExit("the bad column was not reported")
except E.EffortError as e:
    assert e.status == 5, e.status
gaps[target[0]] = target[1]
pm.check()
print("DEBUG-BUILD-OK")
"""


@pytest.fixture(scope="module")
def E():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dynamic_approximate_gemv_b200 import build
    build.build()
    import dynamic_approximate_gemv_b200 as E
    E.lib()
    return E


def test_debug_build_reports_a_bad_column(E):
    env = dict(os.environ, EFFORT_DEBUG_LIB="1")
    res = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0 and "DEBUG-BUILD-OK" in res.stdout, res.stdout[-2000:] + res.stderr[-4000:]


def test_grid_wait_timeout_reports_device_error_and_recovers(E, monkeypatch):
    Wn = inputs.weights(512, 2048, 71)
    prep = O.Prepared(Wn.view(np.uint16), 1.0)
    pm = E.PreparedMatrix(torch.from_numpy(Wn).cuda(), 1.0)
    v = inputs.vector(512, 72)
    vt = torch.from_numpy(v).cuda()
    monkeypatch.setenv("EFFORT_TEST_UNREACHABLE_BARRIER", "1")
    pm.gemv(vt, 0.25)
    torch.cuda.synchronize()
    monkeypatch.delenv("EFFORT_TEST_UNREACHABLE_BARRIER")
    with pytest.raises(E.EffortError) as ei:
        pm.check()
    assert ei.value.status == 5
    cut = torch.empty(1, device="cuda")
    cnt = torch.zeros(1, device="cuda", dtype=torch.int64)
    out = pm.gemv(vt, 0.25, cutoff=cut, count=cnt)
    pm.check()
    ref = O.effort_gemv(prep, v, 0.25)
    assert np.float32(cut.item()).view(np.uint32) == np.float32(ref.c).view(np.uint32)
    assert int(cnt.item()) == ref.count
    got = out.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(got - ref.out) <= 1e-4 * np.linalg.norm(ref.out)
    pm.close()
