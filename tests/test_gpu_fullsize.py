"""GPU parity at the benchmark's full sizes, in the launch configuration the
benchmark times (its own workload classes, CUDA-graph capture and replay,
programmatically dependent launches), on sampled outputs the CPU oracle
computes one unit or one row at a time.

Workloads: the Llama-3.1-8B-shaped decode layer (8 sequences, 32 query heads
over 8 KV heads, 8192 cached tokens, k in {128, 96, 64, 32}), the
131072-token single-sequence decode, the 4096-token prompt in 512-token chunks
(k = 96 and the dense k = d comparator) and the truncated-cache decode with
H2O eviction (32 sequences, m = 96, k = 64, budget 2048 = 256 recent + heavy
hitters).  Every input comes from the seeded generators; P is the oracle's
SVD basis rounded to f32, given to both sides.
"""
import numpy as np
import pytest
import torch

import bench
import synth
from oracle import aqua_oracle as O
import sparse_dimension_attention_b200 as aq
from aqua_testlib import calib_P, check_selection, rel_err_rows, tdev

pytestmark = pytest.mark.gpu

TOL_BF16_OUT = 2e-3   # bf16 output vs the oracle output rounded to bf16
K_STEPS, W_STEPS = 4, 3


def _decode_unit_ref(inp, P64, b, g, G, s, k):
    """Oracle output of step s for the G query heads of KV head g of sequence b:
    the history plus the first s + 1 appended tokens (keys drawn as one stream)."""
    k_all = np.concatenate([inp["k_hist"][b, :, g], inp["k_new"][:s + 1, b, g]], axis=0)     # [T, d]
    v_all = np.concatenate([inp["v_hist"][b, :, g], inp["v_new"][:s + 1, b, g]], axis=0)
    T = k_all.shape[0]
    Kt = O.build_key_cache(k_all[:, None], P64[g:g + 1], "bf16")[:, 0]                       # [T, d]
    ref = O.decode(inp["q"][s, b:b + 1, g * G:(g + 1) * G], P64[g:g + 1], Kt[None, None],
                   v_all[None, None].astype(np.float64), [T], k, out_dtype="bf16")
    return ref["out"][0]


@pytest.fixture(scope="module")
def llama_decode():
    wl = bench.WORKLOADS["llama3.1-8b-decode"]
    P64, P32 = calib_P(wl["Hkv"])
    db = bench.DecodeBench(wl, K_STEPS, W_STEPS, P=tdev(P32))
    inp = synth.decode_inputs(wl["B"], wl["Hq"], wl["Hkv"], wl["T"] - 1, bf16=True, steps=db.n_in)
    yield wl, db, inp, P64
    del db
    torch.cuda.empty_cache()


@pytest.mark.parametrize("k", [96, 128, 64, 32])
def test_llama_decode_graph_sampled_units(llama_decode, k):
    """K decode steps (fused append) captured in one CUDA graph and replayed, as
    the benchmark times them; the last step's output of sampled (sequence, KV
    head) units against the oracle, every length advanced by K."""
    wl, db, inp, P64 = llama_decode
    G = wl["Hq"] // wl["Hkv"]
    db.timed(K_STEPS, W_STEPS, k, world=1, clocks=False, graph=True)
    torch.cuda.synchronize()
    assert aq.aqua_status(db.cache.desc) == aq.AQUA_OK
    assert (db.cache.len.cpu().numpy() == db.T0 + K_STEPS).all()
    out = db.out.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(out).all()
    for b, g in [(0, 0), (3, 5), (7, 7), (5, 2)]:
        ref = _decode_unit_ref(inp, P64, b, g, G, K_STEPS - 1, k)
        err = rel_err_rows(out[b, g * G:(g + 1) * G], ref)
        assert np.max(err) <= TOL_BF16_OUT, (b, g, np.max(err))


def test_long_context_decode_graph_sampled_units():
    """131072-token decode through the benchmark's graph path (split-K over many
    CTAs per unit), sampled KV heads against the oracle."""
    wl = bench.WORKLOADS["long-context-decode"]
    P64, P32 = calib_P(wl["Hkv"])
    K, W = 2, 3
    db = bench.DecodeBench(wl, K, W, P=tdev(P32))
    db.timed(K, W, wl["k"], world=1, clocks=False, graph=True)
    torch.cuda.synchronize()
    assert aq.aqua_status(db.cache.desc) == aq.AQUA_OK
    out = db.out.float().cpu().numpy().astype(np.float64)
    del db
    torch.cuda.empty_cache()
    inp = synth.decode_inputs(wl["B"], wl["Hq"], wl["Hkv"], wl["T"] - 1, bf16=True, steps=max(K, W, 1) + 1)
    G = wl["Hq"] // wl["Hkv"]
    for g in (1, 6):
        ref = _decode_unit_ref(inp, P64, 0, g, G, K - 1, wl["k"])
        err = rel_err_rows(out[0, g * G:(g + 1) * G], ref)
        assert np.max(err) <= TOL_BF16_OUT, (g, np.max(err))


@pytest.fixture(scope="module")
def prompt():
    wl = bench.PREFILL
    P64, P32 = calib_P(wl["Hkv"])
    pb = bench.PrefillBench(wl, tdev(P32))
    inp = synth.prefill_inputs(wl["L_total"], wl["Hq"], wl["Hkv"], bf16=True, B=wl["B"])
    Kt = O.build_key_cache(inp["k"][0], P64, "bf16").transpose(1, 0, 2)        # [Hkv, L, d]
    V = inp["v"][0].transpose(1, 0, 2).astype(np.float64)
    yield wl, pb, inp, P64, Kt, V
    del pb
    torch.cuda.empty_cache()


@pytest.mark.parametrize("k", [96, 128])
def test_prompt_graph_last_chunk_sampled_rows(prompt, k):
    """The whole prompt pass (8 appends + 8 attention calls) captured in one
    CUDA graph and replayed; rows of the last chunk (attending up to 4096
    tokens) against the oracle, every query head."""
    wl, pb, inp, P64, Kt, V = prompt
    pb.timed_graph(1, W_STEPS, k)
    torch.cuda.synchronize()
    assert aq.aqua_status(pb.cache.desc) == aq.AQUA_OK
    assert int(pb.cache.len[0].item()) == wl["L_total"]
    C = wl["chunk"]
    pos0 = wl["L_total"] - C
    out = pb.out.float().cpu().numpy().astype(np.float64)[0]                    # [C, Hq, d]
    assert np.isfinite(out).all()
    for i in (0, 1, 31, 32, 127, 128, 300, C - 1):
        p = pos0 + i
        ref, _ = O.prefill(inp["q"][0, p:p + 1], p, P64, Kt, V, k, out_dtype="bf16")
        err = rel_err_rows(out[i], ref[0])
        assert np.max(err) <= TOL_BF16_OUT, (i, np.max(err))
    # the last chunk once more, eagerly, exporting its selection and q~: the
    # output is bit-identical to the graph's, and every (row, head) selection
    # is exactly the oracle's on the kernel's own q~ (and on the f64 q~ away
    # from near ties)
    Hq, G = wl["Hq"], wl["Hq"] // wl["Hkv"]
    o2 = torch.empty_like(pb.out)
    sel = torch.full((1, C, Hq, k), -1, dtype=torch.int32, device="cuda")
    qp = torch.empty((1, C, Hq, 128), dtype=torch.float32, device="cuda")
    aq.aqua_prefill_attn(pb.cache.desc, pb.q[:, pos0:pos0 + C], pos0, C, pb.P, Hq, k, o2, pb.ws, sel_out=sel,
                         qproj_out=qp)
    torch.cuda.synchronize()
    assert torch.equal(o2, pb.out)
    qt64 = np.einsum("lhi,hij->lhj", inp["q"][0, pos0:pos0 + C].astype(np.float64), P64[np.arange(Hq) // G])
    ref_sel = np.stack([[O.select_dims(qt64[i, h], k) for h in range(Hq)] for i in range(C)])
    near = check_selection(sel.cpu().numpy()[0], qp.cpu().numpy()[0], ref_sel, qt64, k)
    # (row, head) pairs whose f64 k-th/(k+1)-th magnitude gap is within 1e-5 of
    # the largest magnitude are skipped by the protocol (the kernel selects on
    # f32 q~ computed in another summation order); at k = 96 of 128 the gaps
    # near the cut are small and about 0.4% of the pairs fall there.  This
    # bound only rejects a degenerate q~; the exact check above is the parity.
    assert near <= C * Hq // 20, near


def _h2o_oracle_state(inp, P64, b, Hkv, n0, m):
    return [O.H2OSeq(pos=list(range(n0)), score=[0.0] * n0,
                     kt=list(O.build_key_cache(inp["k_hist"][b, :, g][:, None], P64[g][None], "bf16", m)[:, 0]),
                     v=list(inp["v_hist"][b, :, g].astype(np.float64)))
            for g in range(Hkv)]


def _h2o_oracle_step(seq, q_b, kn_b, vn_b, t_abs, P64, wl, got_ev_b):
    """One oracle step of one sequence (accumulate, then evict by the oracle's
    rule).  Where the oracle's victim and the library's differ, the two
    candidates' f64 cumulative scores must be a near tie (several victims are
    then correct); the oracle then follows the library's choice so that the
    states stay comparable.  Returns the step's output."""
    o, _ = O.h2o_decode_step(seq, q_b, kn_b, vn_b, t_abs, P64, wl["k"], 10 ** 9, wl["recent"], "bf16", wl["m"])
    for g, s in enumerate(seq):
        if len(s.pos) <= wl["budget"]:
            assert got_ev_b[g] == -1
            continue
        vi = O.h2o_choose_victim(s.score, s.pos, t_abs, wl["recent"])
        gi = s.pos.index(int(got_ev_b[g]))
        if gi != vi:
            assert s.pos[gi] <= t_abs - wl["recent"], "library evicted a token of the recent window"
            gap = abs(s.score[gi] - s.score[vi])
            assert gap <= 1e-4 * abs(s.score[vi]) + 1e-12, (g, s.pos[gi], s.pos[vi], gap)
        for lst in (s.pos, s.score, s.kt, s.v):
            del lst[gi]
    return o


def test_h2o_full_size_eager_vs_oracle_and_graph_bitwise():
    """Truncated cache + H2O at the benchmark's size.  (1) Steps issued one by
    one through the benchmark's step (decode with fused append, scores and lse
    out, then the H2O update): outputs and evictions of sampled sequences
    against the oracle.  (2) The same steps captured in a CUDA graph and
    replayed from the same cache state give bit-identical outputs, evictions
    and cache contents."""
    wl = bench.H2O_WL
    B, Hq, Hkv, n0, m = wl["B"], wl["Hq"], wl["Hkv"], wl["budget"], wl["m"]
    P64, P32 = calib_P(Hkv)
    hb = bench.H2OBench(wl, tdev(P32))
    inp = synth.decode_inputs(B, Hq, Hkv, n0, bf16=True, steps=hb.n_in)
    sampled = (0, 21)
    seqs = {b: _h2o_oracle_state(inp, P64, b, Hkv, n0, m) for b in sampled}

    def eager_steps(n):
        for _ in range(n):
            i, t_abs = hb.n_steps % hb.n_in, n0 + hb.n_steps
            hb.step()
            torch.cuda.synchronize()
            out = hb.out.float().cpu().numpy().astype(np.float64)
            ev = hb.ev.cpu().numpy()
            for b in sampled:
                o = _h2o_oracle_step(seqs[b], inp["q"][i, b], inp["k_new"][i, b], inp["v_new"][i, b],
                                     t_abs, P64, wl, ev[b])
                err = rel_err_rows(out[b], O.round_bf16(o))
                assert np.max(err) <= TOL_BF16_OUT, (hb.n_steps, b, np.max(err))

    eager_steps(6)
    # (2) graph vs eager from the same state
    snap = hb.cache.snapshot()
    n_at = hb.n_steps
    N = 16
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(N):
            hb.step()
    torch.cuda.synchronize()
    hb.cache.restore(snap)
    g.replay()
    torch.cuda.synchronize()
    out_graph = hb.out.clone()
    ev_graph = hb.ev.clone()
    state_graph = hb.cache.snapshot()
    del g
    hb.cache.restore(snap)
    hb.n_steps = n_at
    eager_steps(N)
    assert torch.equal(out_graph, hb.out)
    assert torch.equal(ev_graph, hb.ev)
    state_eager = hb.cache.snapshot()
    for name in ("k_proj", "v", "len", "n_abs", "pos", "score"):
        assert torch.equal(state_graph[name], state_eager[name]), name
    assert (hb.cache.len.cpu().numpy() == n0).all()
    assert aq.aqua_status(hb.cache.desc) == aq.AQUA_OK
    # retained positions of the sampled sequences agree with the oracle's as sets
    n = int(hb.cache.len[0].item())
    pos = hb.cache.pos.cpu().numpy()
    for b in sampled:
        for gg in range(Hkv):
            assert sorted(pos[b, gg, :n].tolist()) == sorted(seqs[b][gg].pos)
