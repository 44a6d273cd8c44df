"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Contract per call, on seeded synthetic inputs:
  * the cutoff c equals the oracle's bit for bit;
  * the used set for that c matches exactly: |S| and every row's used length
    L_i equal the oracle's (used sets are leading parts of each row's sorted
    order, and the kernel's predicate is the oracle's, so equal per-row counts
    with no double visits mean equal sets; one-hot vectors check single rows
    product by product);
  * out agrees with the oracle's float64 sum over the same set to relative
    L2 <= 1e-4 and max abs error <= 1e-3 * ||out||_inf.
The cutoff, |S| and the L_i are also identical from call to call.  out is
accumulated with reductions whose order varies, so repeated calls agree to
rounding (checked at relative L2 1e-5), not bit for bit.
"""
import numpy as np
import pytest
import torch

from dynamic_approximate_gemv_b200 import inputs
from oracle import effort_oracle as O

pytestmark = pytest.mark.gpu

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


def assert_out_close(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    nref = np.linalg.norm(ref)
    inf = np.max(np.abs(ref)) if ref.size else 0.0
    if nref == 0.0:
        assert np.max(np.abs(got)) == 0.0
        return
    assert np.linalg.norm(got - ref) <= REL_L2 * nref, np.linalg.norm(got - ref) / nref
    assert np.max(np.abs(got - ref)) <= MAX_ABS * inf


def run_gpu(E, pm, v, effort):
    I = pm.in_dim
    dev = torch.device("cuda")
    cutoff = torch.empty(1, device=dev, dtype=torch.float32)
    count = torch.full((1,), -1, device=dev, dtype=torch.int64)
    rowlen = torch.full((I,), -7, device=dev, dtype=torch.int32)
    out = pm.gemv(v, effort, cutoff=cutoff, count=count, rowlen=rowlen)
    torch.cuda.synchronize()
    pm.check()
    return float(cutoff.item()), int(count.item()), rowlen.cpu().numpy().astype(np.int64), out.cpu().numpy()


def check_call(E, prep, pm, v_np, effort):
    v = torch.from_numpy(v_np).cuda()
    c, count, rowlen, out = run_gpu(E, pm, v, effort)
    ref = O.effort_gemv(prep, v_np, effort)
    assert f32bits(c) == f32bits(ref.c), (c, float(ref.c))
    assert count == ref.count
    assert np.array_equal(rowlen, ref.L)
    assert_out_close(out, ref.out)
    return ref


def make(E, I, Od, seed, keep=1.0):
    Wn = inputs.weights(I, Od, seed)
    prep = O.Prepared(Wn.view(np.uint16), keep)
    pm = E.PreparedMatrix(torch.from_numpy(Wn).cuda(), keep)
    return Wn, prep, pm


# ------------------------------------------------------------------ format
def decode_chunk(vals, gaps, c, cs):
    """(column, value bits, kind) of the slots of chunk c; kind is 'entry',
    'filler' (value +0, gap 255) or 'pad' (value +0, gap 0, after the entries)."""
    v = vals[c * cs:(c + 1) * cs].view(np.uint16).astype(np.int64)
    g = gaps[c * cs:(c + 1) * cs].astype(np.int64)
    cols = -1 + np.cumsum(g)
    kinds = []
    for s_ in range(cs):
        if v[s_] != 0:
            kinds.append("entry")
        elif g[s_] == 255:
            kinds.append("filler")
        else:
            kinds.append("pad")
    return cols, v, kinds


def check_layout(prep, pm):
    L = {k: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for k, v in pm.layout().items()}
    I, Od, n = prep.in_dim, prep.out_dim, prep.n
    P, PW, cs = L["n_panels"], L["panel_width"], L["chunk_slots"]
    assert L["n_kept"] == n and P == (Od + PW - 1) // PW
    Wb = prep.W_bits
    seen = np.zeros(L["total_chunks"], dtype=bool)
    for i in range(I):
        order = prep.W_idx[i, :n]
        mag = (Wb[i] & 0x7FFF).astype(np.int64)
        for p in range(P):
            first, S, tail, kept = (int(x) for x in L["lists"][i, p])
            cols = order[order // PW == p]              # the list: panel p's kept entries in row order
            assert kept == cols.size
            nstore = (3 * kept + 7) // 8
            assert tail == (mag[cols[nstore]] if kept > nstore else 0)
            got = []
            for k in range(S):
                c = first + k
                assert not seen[c]
                seen[c] = True
                ccols, cv, kinds = decode_chunk(L["vals"], L["gaps"], c, cs)
                ent = [s_ for s_ in range(cs) if kinds[s_] == "entry"]
                # slots in column order, pads only after the last entry, fillers before an entry
                assert np.all(np.diff(ccols[ent]) > 0)
                last = ent[-1]
                assert all(kd == "pad" for kd in kinds[last + 1:])
                assert all(kd != "pad" for kd in kinds[:last])
                assert ccols[0] >= 0 and ccols[last] < min(PW, Od - p * PW)
                chunk_cols = ccols[ent] + p * PW
                assert np.array_equal(cv[ent], Wb[i, chunk_cols])
                # a chunk is a run of consecutive ranks: its entries are the next ones of the list
                run = cols[len(got):len(got) + len(ent)]
                assert np.array_equal(np.sort(run), chunk_cols)
                assert int(L["head"][c]) & 0xFFFF == mag[run[0]]
                if k < S - 1:
                    assert kinds.count("pad") == 0  # the greedy cut fills every chunk but the last
                got.extend(run.tolist())
            assert len(got) == nstore
        ranks, weights = O.probe_layout(n)
        srt = mag[order]
        exp_probes = np.where(weights > 0, srt[np.maximum(ranks, 0)], 0)
        assert np.array_equal(L["probes"][i].view(np.uint16), exp_probes)
        dense = np.zeros(L["dense_stride"], np.uint16)
        dense[order] = Wb[i, order]
        assert np.array_equal(L["wdense"][i].view(np.uint16), dense)
    assert seen.all()


@pytest.mark.parametrize("I,Od,keep", [(40, 300, 1.0), (33, 513, 0.75), (7, 9, 1.0), (24, 5000, 0.8),
                                       (6, 14336, 1.0)])
def test_layout_matches_oracle_order(E, I, Od, keep):
    _, prep, pm = make(E, I, Od, 101, keep)
    check_layout(prep, pm)


def test_layout_fillers_bridge_wide_gaps(E):
    """Rows whose consecutive ranks sit far apart in column: |w_ij| falls with
    j mod 300, so a chunk's run of ranks takes a few residues from every
    300-column stretch and its sorted columns jump by about 290, which filler
    slots bridge."""
    I, Od = 4, 4096
    j = np.arange(Od)
    sign = np.where(inputs.weights(I, Od, 5) < 0, -1.0, 1.0)
    Wn = (sign * (1.0 - (j % 300) / 1000.0)[None, :]).astype(np.float16)
    prep = O.Prepared(Wn.view(np.uint16), 1.0)
    pm = E.PreparedMatrix(torch.from_numpy(Wn).cuda(), 1.0)
    check_layout(prep, pm)
    g = pm.layout()["gaps"].cpu().numpy()
    assert np.any(g == 255)


def test_storage_within_1_6x_of_fp16(E):
    """The stored format (chunks, dense copy, tables) stays within 1.6x the
    fp16 bytes of W at keep 1."""
    _, prep, pm = make(E, 1024, 14336, 3)
    info = pm.info()
    assert info["device_bytes"] <= 1.6 * 2 * 1024 * 14336


# ------------------------------------------------------------------ parity
@pytest.mark.parametrize("effort", [0.25, 0.15, 0.4, 0.5, 1.0, 0.05])
def test_512_square(E, effort):
    _, prep, pm = make(E, 512, 512, 0)
    v = inputs.vector(512, 1)
    check_call(E, prep, pm, v, effort)


@pytest.mark.parametrize("I,Od,keep,dist,effort", [
    (100, 300, 1.0, "normal", 0.25),   # ragged last tile
    (33, 513, 0.75, "t3", 0.3),        # one-column last tile, keep < 1
    (1, 1, 1.0, "normal", 1.0),
    (1, 1, 1.0, "normal", 0.5),
    (5, 7, 1.0, "t3", 0.4),
    (2000, 700, 0.6, "t3", 0.2),
    (777, 2049, 1.0, "normal", 0.12),
    (64, 32768, 1.0, "normal", 0.25),  # widest supported row
])
def test_ragged_and_edge_shapes(E, I, Od, keep, dist, effort):
    _, prep, pm = make(E, I, Od, 7, keep)
    check_call(E, prep, pm, inputs.vector(I, 8, dist), effort)


def test_tiny_effort_selects_nothing(E):
    _, prep, pm = make(E, 64, 64, 3)
    ref = check_call(E, prep, pm, inputs.vector(64, 4), 1e-6)
    assert ref.count == 0 and np.isinf(ref.c)


def test_zero_and_repeated_vector_entries(E):
    _, prep, pm = make(E, 300, 600, 5)
    v = inputs.vector(300, 6)
    v[::4] = 0.0
    v[1::7] = v[1]
    for e in (0.1, 0.3, 0.9):
        check_call(E, prep, pm, v, e)


def test_all_zero_vector(E):
    _, prep, pm = make(E, 50, 300, 9)
    ref = check_call(E, prep, pm, np.zeros(50, np.float32), 0.3)
    assert float(ref.c) == 0.0  # chart is all zero: every kept product (all zero) is used


def test_fp16_vector(E):
    _, prep, pm = make(E, 512, 768, 11)
    v = inputs.vector(512, 12, dtype=np.float16)
    check_call(E, prep, pm, v, 0.25)


@pytest.mark.parametrize("dtype", [np.float32, np.float16])
def test_host_buffers_match_device_call(E, dtype):
    """effort_gemv_host (host v copied in, out copied back) matches the
    oracle within the contract, for pinned and pageable buffers."""
    _, prep, pm = make(E, 1000, 1300, 21, keep=0.9)
    v_np = inputs.vector(1000, 22, "t3", dtype=dtype)
    v_host = torch.from_numpy(v_np).pin_memory()
    out_host = torch.full((1300,), float("nan"), dtype=torch.float32).pin_memory()
    pm.gemv_host(v_host, 0.3, out_host)
    torch.cuda.synchronize()
    ref = O.effort_gemv(prep, v_np, 0.3).out
    assert_out_close(out_host.numpy(), ref)
    # pageable host memory: the same copies, staged by CUDA
    out2 = torch.zeros(1300, dtype=torch.float32)
    pm.gemv_host(torch.from_numpy(v_np), 0.3, out2)
    torch.cuda.synchronize()
    assert_out_close(out2.numpy(), ref)
    # an effort that targets no product: out is all zeros
    pm.gemv_host(v_host, 1e-9, out_host)
    torch.cuda.synchronize()
    assert not out_host.any()
    # new contents written into the same pinned buffers between calls are
    # seen, call after call
    for seed in (23, 24, 25):
        w_np = inputs.vector(1000, seed, "normal", dtype=dtype)
        v_host.copy_(torch.from_numpy(w_np))
        pm.gemv_host(v_host, 0.3, out_host)
        torch.cuda.synchronize()
        assert_out_close(out_host.numpy(), O.effort_gemv(prep, w_np, 0.3).out)


def test_one_hot_rows_product_by_product(E):
    """A single nonzero v_i: out_j is the one product v_i w_ij exactly where
    (i, j) is used and 0 elsewhere (the used columns match the oracle's
    one by one; each product is exact up to the accumulator's fixed-point
    rounding, far below 1e-6 of it)."""
    Wn, prep, pm = make(E, 64, 700, 13)
    for i in (0, 17, 63):
        v = np.zeros(64, np.float32)
        v[i] = -1.7
        ref = O.effort_gemv(prep, v, 0.004)
        out = pm.gemv(torch.from_numpy(v).cuda(), 0.004).cpu().numpy()
        w = Wn[i].astype(np.float32)
        exp = np.where(ref.mask[i], (np.float32(-1.7) * w).astype(np.float32), 0.0)
        assert np.array_equal(out != 0, ref.mask[i] & (w != 0))
        np.testing.assert_allclose(out, exp, rtol=1e-6, atol=0)


def close_run_to_run(a, b, rel=1e-5):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    assert np.linalg.norm(a - b) <= rel * np.linalg.norm(b)


def test_repeat_calls_agree(E):
    """c, |S| and every L_i are identical over 100 calls; out to rounding."""
    _, prep, pm = make(E, 1024, 1536, 14)
    v = torch.from_numpy(inputs.vector(1024, 15, "t3")).cuda()
    c0, n0, L0, o0 = run_gpu(E, pm, v, 0.25)
    for _ in range(100):
        c1, n1, L1, o1 = run_gpu(E, pm, v, 0.25)
        assert f32bits(c1) == f32bits(c0) and n1 == n0 and np.array_equal(L1, L0)
        close_run_to_run(torch.from_numpy(o1), torch.from_numpy(o0))


def test_back_to_back_calls_on_one_handle(E):
    """Calls queued back to back on one handle and stream, with no host sync:
    each call's blocks start as the previous call's blocks leave and reuse its
    scratch.  Every output must match the same call made alone (to rounding)."""
    _, prep, pm = make(E, 2048, 3072, 31)
    vs = [torch.from_numpy(inputs.vector(2048, 40 + k, "t3" if k % 2 else "normal")).cuda() for k in range(4)]
    efforts = [0.25, 0.1, 0.5, 0.25, 1.0, 0.05, 0.3, 0.25]
    alone = []
    for k, e in enumerate(efforts):
        alone.append(pm.gemv(vs[k % 4], e).clone())
        torch.cuda.synchronize()
    outs = [torch.empty(3072, device="cuda") for _ in efforts]
    for rep in range(3):
        for k, e in enumerate(efforts):
            pm.gemv(vs[k % 4], e, out=outs[k])
        torch.cuda.synchronize()
        for k in range(len(efforts)):
            close_run_to_run(outs[k], alone[k])
    ref = O.effort_gemv(prep, vs[1].cpu().numpy(), efforts[1])
    assert_out_close(alone[1].cpu().numpy(), ref.out)


def test_effort_sweep_4096_square(E):
    _, prep, pm = make(E, 4096, 4096, 2)
    v = inputs.vector(4096, 3, dtype=np.float16)
    refs = [check_call(E, prep, pm, v, e) for e in (1.0, 0.5, 0.4, 0.25, 0.15)]
    counts = [r.count for r in refs]
    assert counts == sorted(counts, reverse=True)


@pytest.mark.parametrize("I,Od,keep", [(4096, 14336, 1.0), (14336, 4096, 1.0), (4096, 14336, 0.75),
                                       (14336, 4096, 0.75)])
def test_ffn_shapes_full_size(E, I, Od, keep):
    """The FFN workload at full size: both shapes, keep 1 and 0.75, efforts
    0.25 and 0.15, v Student-t(3) / sqrt(3)."""
    _, prep, pm = make(E, I, Od, 4, keep)
    for k, effort in enumerate((0.25, 0.15)):
        check_call(E, prep, pm, inputs.vector(I, 7 + k, "t3"), effort)
    pm.close()


def test_handles_of_different_geometries_interleave(E):
    """Each geometry needs its own amount of shared memory per block; a
    matrix prepared after another one with a smaller need must not leave the
    first one unable to launch."""
    Wb, prep_b, pm_b = make(E, 14336, 1024, 81)   # the larger per-block need
    Ws, prep_s, pm_s = make(E, 512, 1024, 82)     # prepared afterwards
    for pm, prep, I in ((pm_b, prep_b, 14336), (pm_s, prep_s, 512), (pm_b, prep_b, 14336)):
        check_call(E, prep, pm, inputs.vector(I, 83, "t3"), 0.25)
    pm_b.close()
    pm_s.close()


def test_tie_heavy_input_takes_the_many_candidates_path(E):
    """Constant |v| and W drawn from eight magnitudes give the chart eight
    distinct values, so the crossing bin holds one value shared by about
    8192 chart entries: more candidates than one block resolves, which sends
    the cutoff through its two extra grid-wide histogram passes.  All ties at
    c are used (|S| differs from K by the probes' estimate, as always)."""
    rng = np.random.default_rng(77)
    mags = np.array([0.001, 0.002, 0.004, 0.008, 0.016, 0.03, 0.05, 0.07], np.float16)
    I = Od = 4096
    Wn = (mags[rng.integers(0, 8, size=(I, Od))] * rng.choice(np.array([-1, 1], np.float16), size=(I, Od)))
    Wn = Wn.astype(np.float16)
    v = (rng.choice(np.array([-0.5, 0.5]), size=I)).astype(np.float32)
    prep = O.Prepared(Wn.view(np.uint16), 1.0)
    pm = E.PreparedMatrix(torch.from_numpy(Wn).cuda(), 1.0)
    for effort in (0.25, 0.5, 0.15):
        check_call(E, prep, pm, v, effort)
    pm.close()


def test_nonfinite_inputs_are_reported(E):
    Wn = inputs.weights(16, 32, 1)
    Wn[3, 5] = np.float16(np.inf)
    with pytest.raises(E.EffortError) as ei:
        E.PreparedMatrix(torch.from_numpy(Wn).cuda())
    assert ei.value.status == 4
    _, prep, pm = make(E, 16, 32, 2)
    v = inputs.vector(16, 3)
    v[2] = np.nan
    pm.gemv(torch.from_numpy(v).cuda(), 0.5)
    with pytest.raises(E.EffortError) as ei:
        pm.check()
    assert ei.value.status == 4
    pm.check()  # the flag is cleared


def test_argument_errors(E):
    _, _, pm = make(E, 16, 32, 2)
    v = torch.zeros(16, device="cuda")
    for bad in (0.0, 1.5, float("nan"), -1.0):
        with pytest.raises(E.EffortError):
            pm.gemv(v, bad)


# ------------------------------------------------------------------ batched / MoE
def test_batched_pairs_match_single_calls(E):
    I, Od = 512, 1024
    mats, preps = [], []
    for x in range(3):
        Wn = inputs.weights(I, Od, 100 + x)
        preps.append(O.Prepared(Wn.view(np.uint16), 1.0))
        mats.append(E.PreparedMatrix(torch.from_numpy(Wn).cuda()))
    V = np.stack([inputs.vector(I, 200 + k) for k in range(4)])
    hidx = [0, 2, 1, 2, 0, 1, 2]
    vidx = [0, 0, 1, 1, 2, 3, 3]
    eff = [0.5, 0.25, 0.12, 0.25, 1.0, 0.4, 0.05]
    ws = E.Workspace(I, Od, max_pairs=len(hidx))
    Vt = torch.from_numpy(V).cuda()
    cut = torch.empty(len(hidx), device="cuda")
    cnt = torch.zeros(len(hidx), device="cuda", dtype=torch.int64)
    OUT = E.gemv_batched(ws, mats, hidx, vidx, Vt, eff, cutoffs=cut, counts=cnt)
    torch.cuda.synchronize()
    for p in range(len(hidx)):
        ref = O.effort_gemv(preps[hidx[p]], V[vidx[p]], eff[p])
        assert f32bits(cut[p].item()) == f32bits(ref.c)
        assert int(cnt[p].item()) == ref.count
        assert_out_close(OUT[p].cpu().numpy(), ref.out)


def test_batched_more_pairs_than_one_launch(E):
    I, Od = 256, 512
    Wn = inputs.weights(I, Od, 300)
    prep = O.Prepared(Wn.view(np.uint16), 1.0)
    m = E.PreparedMatrix(torch.from_numpy(Wn).cuda())
    n = 37
    V = np.stack([inputs.vector(I, 400 + k) for k in range(n)])
    ws = E.Workspace(I, Od, max_pairs=n)
    OUT = E.gemv_batched(ws, [m], [0] * n, list(range(n)), torch.from_numpy(V).cuda(), [0.25] * n)
    for p in (0, 15, 16, 36):
        assert_out_close(OUT[p].cpu().numpy(), O.effort_gemv(prep, V[p], 0.25).out)


def test_batched_union_of_two_vectors_tie_heavy(E):
    """Two selecting pairs on one matrix run as one grid that reads the union
    of their prefixes once.  With a tie-heavy matrix (eight magnitudes) and
    constant |v| each vector's crossing bin holds more candidates than one
    block resolves, so both cutoffs take the grid-wide histogram passes
    inside the shared grid; a third pair on the same matrix runs alone."""
    rng = np.random.default_rng(91)
    mags = np.array([0.001, 0.002, 0.004, 0.008, 0.016, 0.03, 0.05, 0.07], np.float16)
    I, Od = 4096, 2048
    Wn = (mags[rng.integers(0, 8, size=(I, Od))] * rng.choice(np.array([-1, 1], np.float16), size=(I, Od)))
    Wn = Wn.astype(np.float16)
    prep = O.Prepared(Wn.view(np.uint16), 1.0)
    pm = E.PreparedMatrix(torch.from_numpy(Wn).cuda(), 1.0)
    V = np.stack([rng.choice(np.array([-0.5, 0.5]), size=I).astype(np.float32) for _ in range(2)]
                 + [inputs.vector(I, 92)])
    hidx, vidx, eff = [0, 0, 0], [0, 1, 2], [0.25, 0.4, 0.3]
    ws = E.Workspace(I, Od, max_pairs=3)
    cut = torch.empty(3, device="cuda")
    cnt = torch.zeros(3, device="cuda", dtype=torch.int64)
    OUT = E.gemv_batched(ws, [pm], hidx, vidx, torch.from_numpy(V).cuda(), eff, cutoffs=cut, counts=cnt)
    torch.cuda.synchronize()
    for p in range(3):
        ref = O.effort_gemv(prep, V[vidx[p]], eff[p])
        assert f32bits(cut[p].item()) == f32bits(ref.c)
        assert int(cnt[p].item()) == ref.count
        assert_out_close(OUT[p].cpu().numpy(), ref.out)
    ws.close()
    pm.close()


def test_batched_nonfinite_vector_is_reported(E):
    """A non-finite entry in one pair's v of a batched call (here inside a
    two-pair grid) is reported by the workspace's check, which then clears."""
    Wn, prep, pm = make(E, 256, 1024, 98)
    V = np.stack([inputs.vector(256, 99), inputs.vector(256, 100)])
    V[1, 17] = np.inf
    ws = E.Workspace(256, 1024, max_pairs=2)
    E.gemv_batched(ws, [pm], [0, 0], [0, 1], torch.from_numpy(V).cuda(), [0.25, 0.25])
    with pytest.raises(E.EffortError) as ei:
        ws.check()
    assert ei.value.status == 4
    ws.check()
    V[1, 17] = 0.5
    OUT = E.gemv_batched(ws, [pm], [0, 0], [0, 1], torch.from_numpy(V).cuda(), [0.25, 0.25])
    ws.check()
    for k in range(2):
        assert_out_close(OUT[k].cpu().numpy(), O.effort_gemv(prep, V[k], 0.25).out)
    ws.close()
    pm.close()


def test_batched_union_reads_fewer_bytes_than_separate_calls(E):
    """A two-pair grid on one matrix reads each unit once, as far as the
    lower threshold needs: its bytes are at least those of either pair alone
    and at most their sum."""
    Wn, prep, pm = make(E, 2048, 6000, 95)
    V = np.stack([inputs.vector(2048, 96, "t3"), inputs.vector(2048, 97, "t3")])
    Vt = torch.from_numpy(V).cuda()
    ws = E.Workspace(2048, 6000, max_pairs=2)
    E.gemv_batched(ws, [pm], [0, 0], [0, 1], Vt, [0.25, 0.15])
    union = sum(ws.last_call_bytes())
    alone = []
    for k, e in enumerate((0.25, 0.15)):
        pm.gemv(Vt[k], e)
        alone.append(sum(pm.last_call_bytes()))
    assert max(alone) <= union <= sum(alone)
    assert union < sum(alone)
    ws.close()
    pm.close()


def test_batched_moe_full_size_sampled_pairs(E):
    """The batched / MoE workload at full size: 8 experts of 4096 x 14336,
    16 vectors N(0,1) routed top-2 by a seeded N(0,1)/64 gate (ties to the
    lower expert), one cutoff per pair, all 32 pairs in one batched call per
    effort.  The oracle checks three pairs on the most used expert per effort
    (its preparation and the full-size oracle calls are the expensive part on
    the host)."""
    I, Od, n_exp, nv = 4096, 14336, 8, 16
    mats, Wns = [], []
    for x in range(n_exp):
        Wn = inputs.weights(I, Od, 100 + x)
        Wns.append(Wn)
        mats.append(E.PreparedMatrix(torch.from_numpy(Wn).cuda()))
    V = np.stack([inputs.vector(I, 200 + 16 + k) for k in range(nv)])
    gate = inputs.gate(n_exp, I, 300)
    order = np.argsort(-(gate.astype(np.float64) @ V.astype(np.float64).T), axis=0, kind="stable")
    hidx = [int(order[r, k]) for k in range(nv) for r in range(2)]
    vidx = [k for k in range(nv) for _ in range(2)]
    used = sorted(set(hidx), key=lambda x: (-hidx.count(x), x))[:1]
    preps = {x: O.Prepared(Wns[x].view(np.uint16), 1.0) for x in used}
    del Wns
    ws = E.Workspace(I, Od, max_pairs=len(hidx))
    Vt = torch.from_numpy(V).cuda()
    cut = torch.empty(len(hidx), device="cuda")
    cnt = torch.zeros(len(hidx), device="cuda", dtype=torch.int64)
    checked = 0
    for effort in (0.5, 0.25, 0.12):
        OUT = E.gemv_batched(ws, mats, hidx, vidx, Vt, [effort] * len(hidx), cutoffs=cut, counts=cnt)
        torch.cuda.synchronize()
        on_expert = [p for p in range(len(hidx)) if hidx[p] in preps]
        for p in on_expert[:3]:
            ref = O.effort_gemv(preps[hidx[p]], V[vidx[p]], effort)
            assert f32bits(cut[p].item()) == f32bits(ref.c)
            assert int(cnt[p].item()) == ref.count
            assert_out_close(OUT[p].cpu().numpy(), ref.out)
            checked += 1
    assert checked == 9
    ws.close()
    for m in mats:
        m.close()


# ------------------------------------------------------------------ dense baseline
@pytest.mark.parametrize("I,Od", [(512, 512), (100, 296), (4096, 4096)])
def test_dense_gemv(E, I, Od):
    Wn = inputs.weights(I, Od, 21)
    v = inputs.vector(I, 22)
    ws = E.Workspace(I, Od)
    out = E.dense_gemv(ws, torch.from_numpy(Wn).cuda(), torch.from_numpy(v).cuda()).cpu().numpy()
    assert_out_close(out, O.dense_gemv(Wn.view(np.uint16), v))
