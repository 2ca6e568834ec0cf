"""GPU parity of the offline calibration and of H2O eviction on a truncated
AQUA cache, against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import synth
from oracle import aqua_oracle as O
import sparse_dimension_attention_b200 as aq
from aqua_testlib import calib_P, fill_cache, rel_err_rows, tdev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [16384, 1000, 129])
def test_calibration_matches_svd(n):
    X = synth.calibration_matrix(n_q=n // 2, n_k=n - n // 2)
    P_ref, s_ref = O.calibrate(X)
    Xd = tdev(X)
    P = torch.empty((128, 128), dtype=torch.float32, device="cuda")
    s = torch.empty((128,), dtype=torch.float32, device="cuda")
    ws = torch.empty(aq.aqua_calibrate_workspace_size(n, 128), dtype=torch.uint8, device="cuda")
    aq.aqua_calibrate(Xd, P, s, ws)
    torch.cuda.synchronize()
    Pg = P.cpu().numpy().astype(np.float64)
    sg = s.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(sg, s_ref, rtol=1e-5)
    np.testing.assert_allclose(Pg.T @ Pg, np.eye(128), atol=1e-5)
    sign = np.sign(np.sum(Pg * P_ref, axis=0))
    np.testing.assert_allclose(Pg * sign[None, :], P_ref, atol=2e-5)
    # sign convention: each column's largest-magnitude entry is positive
    idx = np.argmax(np.abs(Pg), axis=0)
    assert np.all(Pg[idx, np.arange(128)] > 0)


def _h2o_setup(B, Hq, Hkv, T0, m, budget, dtype=torch.bfloat16):
    P64, P32 = calib_P(Hkv)
    Tcap = (budget + 1 + 15) // 16 * 16
    cache = aq.AquaCache(B, Hkv, Tcap, d_store=m, h2o=True, dtype=dtype)
    return P64, P32, cache


def test_h2o_decision_is_bit_exact():
    """Given the GPU's own f32 cumulative scores, the victim equals the oracle's rule."""
    B, Hq, Hkv, T0, m, k, budget, recent = 2, 8, 2, 80, 96, 64, 80, 16
    P64, P32, cache = _h2o_setup(B, Hq, Hkv, T0, m, budget)
    inp = synth.decode_inputs(B, Hq, Hkv, T0, bf16=True, steps=6)
    Pt = fill_cache(cache, inp["k_hist"], inp["v_hist"], P32)
    sc = torch.zeros((B, Hq, cache.Tcap), dtype=torch.float32, device="cuda")
    lse = torch.zeros((B, Hq), dtype=torch.float32, device="cuda")
    out = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(aq.aqua_decode_workspace_size(cache.desc, Hq), dtype=torch.uint8, device="cuda")
    ev = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
    inf_lse = torch.full((B, Hq), float("inf"), device="cuda")
    for s in range(6):
        aq.aqua_project_keys(cache.desc, tdev(inp["k_new"][s][:, None], torch.bfloat16),
                             tdev(inp["v_new"][s][:, None], torch.bfloat16), Pt, 1)
        aq.aqua_decode_attn(cache.desc, tdev(inp["q"][s], torch.bfloat16), Pt, Hq, k, out, ws, scores_out=sc,
                            lse_out=lse)
        aq.aqua_h2o_update(cache.desc, sc, lse, Hq, 10 ** 9, recent, ev)      # accumulate only
        torch.cuda.synchronize()
        assert (ev.cpu().numpy() == -1).all()
        n = int(cache.len[0].item())
        score = cache.score.cpu().numpy()[:, :, :n].astype(np.float64)
        pos = cache.pos.cpu().numpy()[:, :, :n]
        newest = int(cache.n_abs[0].item()) - 1
        aq.aqua_h2o_update(cache.desc, sc, inf_lse, Hq, budget, recent, ev)  # evict only
        torch.cuda.synchronize()
        got = ev.cpu().numpy()
        for b in range(B):
            for g in range(Hkv):
                vi = O.h2o_choose_victim(score[b, g], pos[b, g], newest, recent)
                assert got[b, g] == (pos[b, g][vi] if n > budget and vi >= 0 else -1)
        assert int(cache.len[0].item()) == min(n, budget)


@pytest.mark.parametrize("fused,G,kv", [(False, 4, "bf16"), (True, 4, "bf16"), (True, 2, "bf16"), (True, 1, "bf16"),
                                         (True, 4, "f32")])
def test_h2o_steps_match_oracle(fused, G, kv):
    """Truncated cache (m = 96), k = 64 within it, budget 64 = 16 recent + 48 heavy, 40 steps;
    the step's key/value appended by aqua_project_keys or by the decode call
    itself; G query heads per KV head (the update sums the group's heads);
    bf16 or f32 cache."""
    B, Hkv, T0, m, k, budget, recent, steps = 2, 2, 64, 96, 64, 64, 16, 40
    Hq = G * Hkv
    dt = torch.bfloat16 if kv == "bf16" else torch.float32
    P64, P32, cache = _h2o_setup(B, Hq, Hkv, T0, m, budget, dtype=dt)
    inp = synth.decode_inputs(B, Hq, Hkv, T0, bf16=(kv == "bf16"), steps=steps)
    Pt = fill_cache(cache, inp["k_hist"], inp["v_hist"], P32)
    # oracle state after the same warm-up
    seqs = [[O.H2OSeq(pos=list(range(T0)), score=[0.0] * T0,
                      kt=list(O.build_key_cache(inp["k_hist"][b, :, g][:, None], P64[g][None], kv, m)[:, 0]),
                      v=list(inp["v_hist"][b, :, g].astype(np.float64)))
             for g in range(Hkv)] for b in range(B)]
    sc = torch.zeros((B, Hq, cache.Tcap), dtype=torch.float32, device="cuda")
    lse = torch.zeros((B, Hq), dtype=torch.float32, device="cuda")
    out = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(aq.aqua_decode_workspace_size(cache.desc, Hq), dtype=torch.uint8, device="cuda")
    ev = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
    for s in range(steps):
        kn, vn = tdev(inp["k_new"][s], dt), tdev(inp["v_new"][s], dt)
        if fused:
            aq.aqua_decode_attn(cache.desc, tdev(inp["q"][s], dt), Pt, Hq, k, out, ws, scores_out=sc,
                                lse_out=lse, k_new=kn, v_new=vn)
        else:
            aq.aqua_project_keys(cache.desc, kn[:, None], vn[:, None], Pt, 1)
            aq.aqua_decode_attn(cache.desc, tdev(inp["q"][s], dt), Pt, Hq, k, out, ws, scores_out=sc,
                                lse_out=lse)
        aq.aqua_h2o_update(cache.desc, sc, lse, Hq, budget, recent, ev)
        torch.cuda.synchronize()
        got_out = out.float().cpu().numpy().astype(np.float64)
        got_ev = ev.cpu().numpy()
        for b in range(B):
            o_ref, ev_ref = O.h2o_decode_step(seqs[b], inp["q"][s, b], inp["k_new"][s, b], inp["v_new"][s, b],
                                              T0 + s, P64, k, budget, recent, kv, m)
            assert list(got_ev[b]) == ev_ref, f"step {s} seq {b}: {list(got_ev[b])} vs {ev_ref}"
            err = rel_err_rows(got_out[b], O.round_bf16(o_ref))
            assert np.max(err) <= 2e-3, (s, b, np.max(err))
        # retained positions agree as sets
        n = int(cache.len[0].item())
        assert n == min(T0 + s + 1, budget)
        pos = cache.pos.cpu().numpy()
        for b in range(B):
            for g in range(Hkv):
                assert sorted(pos[b, g, :n].tolist()) == sorted(seqs[b][g].pos)
    assert aq.aqua_status(cache.desc) == aq.AQUA_OK
