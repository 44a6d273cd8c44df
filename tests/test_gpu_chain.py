"""A decode chain through the library, checked matvec by matvec (teacher forced).

The stack follows the Mistral-7B layer pattern at a reduced width: per layer
q, k, v, o, w1, w3, w2 with every matvec input RMS-normalised, each output
feeding the next step.  Every matvec of two layers is compared with the oracle
on the GPU's own input to that step, under one effort for the whole stack and
under a schedule that changes the effort from matvec to matvec: the cutoff bit
for bit, the used count exactly, the output within the parity tolerance.
Selection exactness is thus defined at every step even though the chain's
inputs come from the GPU.
"""
import os
import sys

import numpy as np
import pytest
import torch

from dynamic_approximate_gemv_b200 import inputs
from oracle import effort_oracle as O

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REL_L2 = 1e-4
MAX_ABS = 1e-3


@pytest.fixture(scope="module")
def E():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dynamic_approximate_gemv_b200 import build
    build.build()
    import dynamic_approximate_gemv_b200 as E
    E.lib()
    return E


def f32bits(x):
    return int(np.array([x], np.float32).view(np.uint32)[0])


def checked_gemv(pm, prep, x, effort):
    cutoff = torch.empty(1, device="cuda", dtype=torch.float32)
    count = torch.full((1,), -1, device="cuda", dtype=torch.int64)
    out = pm.gemv(x, effort, cutoff=cutoff, count=count)
    torch.cuda.synchronize()
    ref = O.effort_gemv(prep, x.cpu().numpy(), effort)
    assert f32bits(cutoff.item()) == f32bits(ref.c)
    assert int(count.item()) == ref.count
    got = out.cpu().numpy().astype(np.float64)
    nref = np.linalg.norm(ref.out)
    assert np.linalg.norm(got - ref.out) <= REL_L2 * nref
    assert np.max(np.abs(got - ref.out)) <= MAX_ABS * np.max(np.abs(ref.out))
    return out


def run_chain(E, schedule):
    sys.path.insert(0, ROOT)
    import bench
    dims = (512, 128, 1792)  # d_model, kv width, ffn width (Mistral-7B pattern, scaled by 1/8)
    layers, keep = 2, 0.8
    mats, preps = [], []
    for l in range(layers):
        L, P = {}, {}
        for m, (name, a, b) in enumerate(bench.CHAIN_MATS):
            Wn = inputs.weights(dims[a], dims[b], 1000 * l + m)
            L[name] = E.PreparedMatrix(torch.from_numpy(Wn).cuda(), keep)
            P[name] = O.Prepared(Wn.view(np.uint16), keep)
        mats.append(L)
        preps.append(P)
    try:
        x = torch.from_numpy(inputs.vector(dims[0], 9)).cuda()
        for l, (L, P) in enumerate(zip(mats, preps)):
            e = {name: bench.effort_for(schedule, l, name) for name in L}
            xn = bench.rms_norm(x)
            q = checked_gemv(L["q"], P["q"], xn, e["q"])
            checked_gemv(L["k"], P["k"], xn, e["k"])
            checked_gemv(L["v"], P["v"], xn, e["v"])
            o = checked_gemv(L["o"], P["o"], bench.rms_norm(q), e["o"])
            h = bench.rms_norm(o)
            a = checked_gemv(L["w1"], P["w1"], h, e["w1"])
            b = checked_gemv(L["w3"], P["w3"], h, e["w3"])
            x = bench.rms_norm(checked_gemv(L["w2"], P["w2"], bench.rms_norm(a * b), e["w2"]))
        assert torch.isfinite(x).all()
    finally:
        for L in mats:
            for pm in L.values():
                pm.close()


def test_chain_two_layers_teacher_forced(E):
    run_chain(E, 0.25)


def test_chain_per_matrix_effort_schedule(E):
    """Effort set matvec by matvec (the pages' per-layer, per-matrix knob):
    each of the 14 matvecs takes the next effort of a cycle that includes the
    whole-matrix case, and each is checked against the oracle at its own
    effort."""
    sys.path.insert(0, ROOT)
    import bench
    cycle = (0.05, 0.15, 0.25, 0.5, 1.0)
    names = [n for n, _, _ in bench.CHAIN_MATS]
    run_chain(E, lambda layer, name: cycle[(7 * layer + names.index(name)) % len(cycle)])


def test_layer0_full_width_teacher_forced(E):
    """Layer 0 of the full-width decode stack (q, o 4096 x 4096; k, v
    4096 x 1024; w1, w3 4096 x 14336; w2 14336 x 4096; keep 0.8; effort
    0.25), every matvec checked against the oracle on the GPU's own input to
    that step."""
    sys.path.insert(0, ROOT)
    import bench
    dims, keep, effort = (4096, 1024, 14336), 0.8, 0.25
    mats = {}
    for m, (name, a, b) in enumerate(bench.CHAIN_MATS):
        mats[name] = E.PreparedMatrix(torch.from_numpy(inputs.weights(dims[a], dims[b], m)).cuda(), keep)

    def step(name, x):
        a, b = [(aa, bb) for n, aa, bb in bench.CHAIN_MATS if n == name][0]
        m = [k for k, (n, _, _) in enumerate(bench.CHAIN_MATS) if n == name][0]
        prep = O.Prepared(inputs.weights(dims[a], dims[b], m).view(np.uint16), keep)
        out = checked_gemv(mats[name], prep, x, effort)
        del prep
        return out

    try:
        xn = bench.rms_norm(torch.from_numpy(inputs.vector(dims[0], 9)).cuda())
        q = step("q", xn)
        step("k", xn)
        step("v", xn)
        o = step("o", bench.rms_norm(q))
        h = bench.rms_norm(o)
        a = step("w1", h)
        b = step("w3", h)
        y = step("w2", bench.rms_norm(a * b))
        assert torch.isfinite(y).all()
    finally:
        for pm in mats.values():
            pm.close()
