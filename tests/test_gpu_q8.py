"""GPU parity for Q8 matrices (int8 q, binary16 row scales): the CUDA path
through the C ABI against the Q8 oracle, under the same contract as the fp16
parity tests (c bit for bit, |S| and every L_i exact, out within relative
L2 1e-4 and max abs 1e-3 ||out||_inf), plus the stored layout against the
oracle's sort."""
import numpy as np
import pytest
import torch

from dynamic_approximate_gemv_b200 import inputs
from oracle import effort_oracle as F
from oracle import effort_q8_oracle as Q
from tests.test_gpu_parity import E, assert_out_close, f32bits, run_gpu  # noqa: F401 (E is a fixture)

pytestmark = pytest.mark.gpu


def make_q8(E, I, Od, seed, keep=1.0, no_zero=False):
    q, s = inputs.q8_weights(I, Od, seed)
    if no_zero:
        q = np.where(q == 0, np.int8(1), q).astype(np.int8)
    prep = Q.PreparedQ8(q, s.view(np.uint16), keep)
    pm = E.PreparedMatrix.from_q8(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), keep)
    return q, s, prep, pm


def check_call(E, prep, pm, v_np, effort):
    c, count, rowlen, out = run_gpu(E, pm, torch.from_numpy(v_np).cuda(), effort)
    ref = Q.effort_gemv(prep, v_np, effort)
    assert f32bits(c) == f32bits(ref.c), (c, float(ref.c))
    assert count == ref.count
    assert np.array_equal(rowlen, ref.L)
    assert_out_close(out, ref.out)
    return ref


def mag16(qrow, szero):
    """binary16 bits of |q| (0 on a zero-scale row)."""
    m = np.abs(qrow.astype(np.int64)).astype(np.float16).view(np.uint16).astype(np.int64)
    return np.zeros_like(m) if szero else m


@pytest.mark.parametrize("I,Od,keep", [(40, 300, 1.0), (33, 513, 0.75), (24, 5000, 0.8)])
def test_q8_layout_matches_oracle_order(E, I, Od, keep):
    q, s, prep, pm = make_q8(E, I, Od, 7 + I, keep, no_zero=True)
    L = {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for k, v in pm.layout().items()}
    assert L["weight_kind"] == 1
    assert np.array_equal(L["scales"].view(np.uint16), s.view(np.uint16))
    n, P, PW, cs = prep.n, L["n_panels"], L["panel_width"], L["chunk_slots"]
    seen = np.zeros(L["total_chunks"], dtype=bool)
    for i in range(I):
        order = prep.W_idx[i, :n]
        mag = mag16(q[i], False)
        for p in range(P):
            first, S, tail, kept = (int(x) for x in L["lists"][i, p])
            cols = order[order // PW == p]
            assert kept == cols.size
            nstore = (3 * kept + 7) // 8
            assert tail == (mag[cols[nstore]] if kept > nstore else 0)
            got = []
            for k in range(S):
                c = first + k
                assert not seen[c]
                seen[c] = True
                v = L["vals"][c * cs:(c + 1) * cs].astype(np.int64)
                g = L["gaps"][c * cs:(c + 1) * cs].astype(np.int64)
                ccols = -1 + np.cumsum(g)
                ent = [t for t in range(cs) if v[t] != 0]  # no stored q is 0 here
                assert all(g[t] == 255 for t in range(cs) if v[t] == 0 and t < ent[-1])  # fillers
                assert all(g[t] == 0 for t in range(ent[-1] + 1, cs))                    # pads
                assert np.all(np.diff(ccols[ent]) > 0)
                chunk_cols = ccols[ent] + p * PW
                assert np.array_equal(v[ent], q[i, chunk_cols].astype(np.int64))
                run = cols[len(got):len(got) + len(ent)]
                assert np.array_equal(np.sort(run), chunk_cols)
                assert int(L["head"][c]) & 0xFFFF == mag[run[0]]
                got.extend(run.tolist())
            assert len(got) == nstore
        ranks, weights = F.probe_layout(n)
        exp_probes = np.where(weights > 0, mag[order][np.maximum(ranks, 0)], 0)
        assert np.array_equal(L["probes"][i].view(np.uint16), exp_probes)
        dense = np.zeros(L["dense_stride"], np.int8)
        dense[order] = q[i, order]
        assert np.array_equal(L["wdense"][i], dense)
    assert seen.all()
    pm.close()


@pytest.mark.parametrize("effort", [0.25, 0.6, 1.0])
def test_q8_512_square(E, effort):
    q, s, prep, pm = make_q8(E, 512, 512, 0)
    check_call(E, prep, pm, inputs.vector(512, 0), effort)
    pm.close()


@pytest.mark.parametrize("I,Od,dist,effort,keep", [
    (4096, 4096, "normal", 0.25, 1.0), (4096, 14336, "t3", 0.25, 1.0), (777, 3000, "t3", 0.15, 0.75),
    (300, 2049, "normal", 0.4, 0.5)])
def test_q8_shapes(E, I, Od, dist, effort, keep):
    q, s, prep, pm = make_q8(E, I, Od, 3, keep)
    check_call(E, prep, pm, inputs.vector(I, 4, dist), effort)
    d, sp = pm.last_call_bytes()
    assert d % 256 == 0 and sp % 128 == 0  # int8 stripes, 2-byte slots
    pm.close()


def test_q8_zero_and_negative_scales(E):
    I, Od = 300, 2000
    q, s = inputs.q8_weights(I, Od, 12)
    s = s.copy()
    s[[3, 50, 51]] = np.float16(0.0)
    s[[4, 7, 100]] = -s[[4, 7, 100]]
    prep = Q.PreparedQ8(q, s.view(np.uint16), 1.0)
    pm = E.PreparedMatrix.from_q8(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), 1.0)
    v = inputs.vector(I, 13, "t3")
    for effort in (0.3, 1.0):
        ref = check_call(E, prep, pm, v, effort)
        assert not ref.mask[3].any() or effort == 1.0
    pm.close()


def test_q8_tiny_effort_and_repeat(E):
    q, s, prep, pm = make_q8(E, 256, 1024, 21)
    v = inputs.vector(256, 22)
    check_call(E, prep, pm, v, 1.0 / (256 * 1024))  # K = 1
    r1 = run_gpu(E, pm, torch.from_numpy(v).cuda(), 0.3)
    r2 = run_gpu(E, pm, torch.from_numpy(v).cuda(), 0.3)
    assert r1[0] == r2[0] and r1[1] == r2[1] and np.array_equal(r1[2], r2[2])
    pm.close()


def test_q8_batched_union_pair(E):
    """Two selecting pairs on one Q8 matrix share a grid (union read)."""
    I, Od = 2048, 4096
    q, s, prep, pm = make_q8(E, I, Od, 31)
    V = np.stack([inputs.vector(I, 32, "t3"), inputs.vector(I, 33)])
    hidx, vidx, eff = [0, 0], [0, 1], [0.25, 0.12]
    ws = E.Workspace(I, Od, max_pairs=2)
    cut = torch.empty(2, device="cuda")
    cnt = torch.zeros(2, device="cuda", dtype=torch.int64)
    OUT = E.gemv_batched(ws, [pm], hidx, vidx, torch.from_numpy(V).cuda(), eff, cutoffs=cut, counts=cnt)
    torch.cuda.synchronize()
    ws.check()
    for p in range(2):
        ref = Q.effort_gemv(prep, V[vidx[p]], eff[p])
        assert f32bits(cut[p].item()) == f32bits(ref.c)
        assert int(cnt[p].item()) == ref.count
        assert_out_close(OUT[p].cpu().numpy(), ref.out)
    ws.close()
    pm.close()


def test_q8_nonfinite_scale_is_rejected(E):
    q, s = inputs.q8_weights(8, 64, 41)
    s = s.copy()
    s[2] = np.float16(np.inf)
    with pytest.raises(E.EffortError) as ei:
        E.PreparedMatrix.from_q8(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), 1.0)
    assert ei.value.status == 4  # EFFORT_ERR_NONFINITE
