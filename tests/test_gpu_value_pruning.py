"""GPU parity of AQUA-Memory value pruning (projected values, the first dv
dimensions stored, outputs brought back by P's first dv columns) against the
CPU oracle, through the C ABI: the stored values, decode at several widths,
group sizes, cache types and lengths (split-K included), the two-phase and
no-workspace entry points, and H2O eviction on a cache whose keys and values
are both pruned."""
import numpy as np
import pytest
import torch

import synth
from oracle import aqua_oracle as O
import sparse_dimension_attention_b200 as aq
from aqua_testlib import calib_P, check_selection, fill_cache, oracle_cache, rel_err_rows, tdev, torch_dtype

pytestmark = pytest.mark.gpu

TOL_BF16_OUT = 2e-3   # bf16 output vs the oracle output rounded to bf16
TOL_F32_OUT = 1e-5    # f32 output, f32 cache


def _inputs(B, Hq, Hkv, T, kv, steps=1):
    inp = synth.decode_inputs(B, Hq, Hkv, T, bf16=(kv == "bf16"), steps=steps)
    k_all = np.concatenate([inp["k_hist"], inp["k_new"].transpose(1, 0, 2, 3)], axis=1)   # [B, T+s, Hkv, d]
    v_all = np.concatenate([inp["v_hist"], inp["v_new"].transpose(1, 0, 2, 3)], axis=1)
    return inp, k_all, v_all


@pytest.mark.parametrize("kv", ["bf16", "f32"])
def test_projected_value_storage(kv):
    """Stored V^ is the cache-type rounding of (v P)[:dv]: for bf16 it equals the
    oracle's RNE except where the exact value lies within the f32 projection's
    rounding-error bound of a bf16 midpoint; for f32 it is within that bound of
    the exact product.  The fused append (decode call) stores the same bits as
    aqua_project_keys."""
    B, Hq, Hkv, T, dv = 2, 8, 2, 150, 96
    P64, P32 = calib_P(Hkv)
    inp, k_all, v_all = _inputs(B, Hq, Hkv, T, kv, steps=1)
    dt = torch_dtype(kv)
    a = aq.AquaCache(B, Hkv, 160, dtype=dt, dv_store=dv)
    b = aq.AquaCache(B, Hkv, 160, dtype=dt, dv_store=dv)
    Pt = fill_cache(a, k_all, v_all, P32, chunk=64)                       # history + the new token
    fill_cache(b, inp["k_hist"], inp["v_hist"], P32, chunk=64)            # history, then the fused append
    ws = torch.zeros(aq.aqua_decode_workspace_size(b.desc, Hq), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, Hq, 128), dtype=dt, device="cuda")
    aq.aqua_decode_attn(b.desc, tdev(inp["q"][0], dt), Pt, Hq, 64, out, ws, k_new=tdev(inp["k_new"][0], dt),
                        v_new=tdev(inp["v_new"][0], dt))
    torch.cuda.synchronize()
    assert torch.equal(a.v, b.v) and torch.equal(a.k_proj, b.k_proj) and torch.equal(a.len, b.len)
    assert a.v.shape[-1] == dv
    got = a.v.float().cpu().numpy()[:, :, :T + 1].transpose(0, 2, 1, 3).astype(np.float64)   # [B, T+1, Hkv, dv]
    vv = v_all.astype(np.float64)
    exact = np.einsum("btgi,gij->btgj", vv, P64)[..., :dv]
    bound = 128 * 2.0 ** -24 * np.einsum("btgi,gij->btgj", np.abs(vv), np.abs(P64))[..., :dv]
    if kv == "f32":
        assert np.all(np.abs(got - exact) <= bound)
        return
    ref = O.build_value_cache(v_all, P64, "bf16", dv)
    diff = got != ref
    if diff.any():
        g, r, e, bd = got[diff], ref[diff], exact[diff], bound[diff]
        assert np.all(O.round_bf16(g) == g)
        assert np.all(np.abs(e - (g + r) / 2) <= bd)                   # a midpoint within f32 error
    assert diff.mean() < 2e-3


@pytest.mark.parametrize("kv,dv,G,d_store,k,out", [
    ("bf16", 96, 4, 96, 64, "bf16"),      # keys and values both pruned to 96 dims
    ("bf16", 64, 2, 128, 96, "bf16"),     # values only: one 64-dim V half
    ("bf16", 128, 1, 128, 48, "bf16"),    # projected, not pruned
    ("bf16", 32, 4, 128, 96, "f32"),
    ("f32", 96, 4, 128, 96, "f32"),
    ("f32", 48, 2, 96, 32, "f32"),
])
def test_decode_projected_values(kv, dv, G, d_store, k, out):
    B, Hkv, T = 3, 2, 600
    Hq = G * Hkv
    P64, P32 = calib_P(Hkv)
    inp, k_all, v_all = _inputs(B, Hq, Hkv, T, kv)
    cache = aq.AquaCache(B, Hkv, 608, d_store=d_store, dtype=torch_dtype(kv), dv_store=dv)
    Pt = fill_cache(cache, k_all, v_all, P32)
    lens = [T + 1, 37, 0]                                          # ragged, one empty sequence
    cache.len.copy_(torch.tensor(lens, dtype=torch.int32))
    q = inp["q"][0]
    od = torch_dtype(out)
    o = torch.full((B, Hq, 128), 5.0, dtype=od, device="cuda")
    sel = torch.empty((B, Hq, k), dtype=torch.int32, device="cuda")
    qp = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    ws = torch.zeros(aq.aqua_decode_workspace_size(cache.desc, Hq), dtype=torch.uint8, device="cuda")
    aq.aqua_decode_attn(cache.desc, tdev(q, torch_dtype(kv)), Pt, Hq, k, o, ws, sel_out=sel, qproj_out=qp,
                        lse_out=lse)
    torch.cuda.synchronize()
    assert aq.aqua_status(cache.desc) == aq.AQUA_OK
    Kt = oracle_cache(k_all, P64, kv, d_store)
    Vh = O.build_value_cache(v_all, P64, kv, dv).transpose(0, 2, 1, 3)
    ref = O.decode(q, P64, Kt, Vh, lens, k, m=d_store, out_dtype=out, v_projected=True)
    got = o.float().cpu().numpy().astype(np.float64)
    live = [i for i, L in enumerate(lens) if L > 0]
    tol = TOL_BF16_OUT if out == "bf16" else (TOL_F32_OUT if kv == "f32" else 1e-4)
    assert np.max(rel_err_rows(got[live], ref["out"][live])) <= tol
    assert np.all(got[2] == 0.0) and np.all(np.isneginf(lse.cpu().numpy()[2]))
    np.testing.assert_allclose(lse.cpu().numpy()[live], ref["lse"][live], rtol=1e-5, atol=1e-5)
    check_selection(sel.cpu().numpy(), qp.cpu().numpy(), ref["sel"], ref["qt"], k, d_store)


def test_long_context_projected_values_split_k():
    """One sequence of 40000 tokens over 8 KV heads: every unit is split over
    many CTAs, so the pre-projection outputs are merged from partials before
    the back-projection."""
    B, Hq, Hkv, T, k, dv = 1, 32, 8, 39999, 96, 96
    P64, P32 = calib_P(Hkv)
    inp, k_all, v_all = _inputs(B, Hq, Hkv, T, "bf16")
    cache = aq.AquaCache(B, Hkv, T + 1, dv_store=dv)
    Pt = fill_cache(cache, k_all, v_all, P32, chunk=8192)
    o = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    ws = torch.zeros(aq.aqua_decode_workspace_size(cache.desc, Hq), dtype=torch.uint8, device="cuda")
    aq.aqua_decode_attn(cache.desc, tdev(inp["q"][0], torch.bfloat16), Pt, Hq, k, o, ws)
    torch.cuda.synchronize()
    got = o.cpu().numpy().astype(np.float64)
    for g in (0, 3, 7):
        Kt = O.build_key_cache(k_all[:, :, g:g + 1], P64[g:g + 1], "bf16").transpose(0, 2, 1, 3)
        Vh = O.build_value_cache(v_all[:, :, g:g + 1], P64[g:g + 1], "bf16", dv).transpose(0, 2, 1, 3)
        ref = O.decode(inp["q"][0][:, g * 4:(g + 1) * 4], P64[g:g + 1], Kt, Vh, [T + 1], k, v_projected=True)
        assert np.max(rel_err_rows(got[:, g * 4:(g + 1) * 4], ref["out"])) <= 1e-4


def test_projected_values_two_phase_and_no_workspace_entry_points():
    """aqua_decode_select + aqua_decode_attend (given P) and aqua_decode_attn_static
    give the bits of aqua_decode_attn on a cache with projected values."""
    B, Hq, Hkv, T, k, dv = 2, 16, 4, 900, 64, 80
    P64, P32 = calib_P(Hkv)
    inp, _, _ = _inputs(B, Hq, Hkv, T, "bf16", steps=2)
    caches = [aq.AquaCache(B, Hkv, 912, dv_store=dv) for _ in range(3)]
    for c in caches:
        Pt = fill_cache(c, inp["k_hist"], inp["v_hist"], P32)
    outs = []
    for mode, c in enumerate(caches):
        ws = torch.zeros(aq.aqua_decode_workspace_size(c.desc, Hq), dtype=torch.uint8, device="cuda")
        r = []
        for s in range(2):
            q = tdev(inp["q"][s], torch.bfloat16)
            kn, vn = tdev(inp["k_new"][s], torch.bfloat16), tdev(inp["v_new"][s], torch.bfloat16)
            o = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
            if mode == 0:
                aq.aqua_decode_attn(c.desc, q, Pt, Hq, k, o, ws, k_new=kn, v_new=vn)
            elif mode == 1:
                aq.aqua_decode_select(c.desc, q, Pt, Hq, k, ws, k_new=kn, v_new=vn)
                aq.aqua_decode_attend(c.desc, Hq, o, ws, appended=True, P=Pt)
            else:
                aq.aqua_decode_attn_static(c.desc, q, Pt, Hq, k, o, k_new=kn, v_new=vn)
            r.append(o.clone())
        torch.cuda.synchronize()
        outs.append(r)
    for mode in (1, 2):
        for s in range(2):
            assert torch.equal(outs[0][s], outs[mode][s]), (mode, s)
        assert torch.equal(caches[0].v, caches[mode].v) and torch.equal(caches[0].len, caches[mode].len)


def test_h2o_with_pruned_keys_and_values():
    """AQUA-Memory on both keys (m = 96) and values (dv = 96), k = 64, H2O budget
    64 = 16 recent + 48 heavy, 30 steps with the fused append: evictions and
    outputs against the oracle (pruned values; the H2O rule is unchanged)."""
    B, Hq, Hkv, T0, m, dv, k, budget, recent, steps = 2, 8, 2, 64, 96, 96, 64, 64, 16, 30
    P64, P32 = calib_P(Hkv)
    cache = aq.AquaCache(B, Hkv, (budget + 1 + 15) // 16 * 16, d_store=m, h2o=True, dv_store=dv)
    inp = synth.decode_inputs(B, Hq, Hkv, T0, bf16=True, steps=steps)
    Pt = fill_cache(cache, inp["k_hist"], inp["v_hist"], P32)
    seqs = [[O.H2OSeq(pos=list(range(T0)), score=[0.0] * T0,
                      kt=list(O.build_key_cache(inp["k_hist"][b, :, g][:, None], P64[g][None], "bf16", m)[:, 0]),
                      v=list(O.build_value_cache(inp["v_hist"][b, :, g][:, None], P64[g][None], "bf16", dv)[:, 0]))
             for g in range(Hkv)] for b in range(B)]
    sc = torch.zeros((B, Hq, cache.Tcap), dtype=torch.float32, device="cuda")
    lse = torch.zeros((B, Hq), dtype=torch.float32, device="cuda")
    out = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(aq.aqua_decode_workspace_size(cache.desc, Hq), dtype=torch.uint8, device="cuda")
    ev = torch.empty((B, Hkv), dtype=torch.int32, device="cuda")
    for s in range(steps):
        kn, vn = tdev(inp["k_new"][s], torch.bfloat16), tdev(inp["v_new"][s], torch.bfloat16)
        aq.aqua_decode_attn(cache.desc, tdev(inp["q"][s], torch.bfloat16), Pt, Hq, k, out, ws, scores_out=sc,
                            lse_out=lse, k_new=kn, v_new=vn)
        aq.aqua_h2o_update(cache.desc, sc, lse, Hq, budget, recent, ev)
        torch.cuda.synchronize()
        got_out = out.float().cpu().numpy().astype(np.float64)
        got_ev = ev.cpu().numpy()
        for b in range(B):
            o_ref, ev_ref = O.h2o_decode_step(seqs[b], inp["q"][s, b], inp["k_new"][s, b], inp["v_new"][s, b],
                                              T0 + s, P64, k, budget, recent, "bf16", m, m_v=dv)
            assert list(got_ev[b]) == ev_ref, f"step {s} seq {b}: {list(got_ev[b])} vs {ev_ref}"
            assert np.max(rel_err_rows(got_out[b], O.round_bf16(o_ref))) <= TOL_BF16_OUT, (s, b)
    n = int(cache.len[0].item())
    pos = cache.pos.cpu().numpy()
    vcache = cache.v.float().cpu().numpy()
    for b in range(B):
        for g in range(Hkv):
            assert sorted(pos[b, g, :n].tolist()) == sorted(seqs[b][g].pos)
            # the retained value rows are the oracle's pruned rows, slot by slot
            order = {p_: i for i, p_ in enumerate(seqs[b][g].pos)}
            for slot in range(0, n, 7):
                ref_row = seqs[b][g].v[order[int(pos[b, g, slot])]]
                assert np.max(np.abs(vcache[b, g, slot] - ref_row)) <= 2.0 ** -7 * np.max(np.abs(ref_row))
    assert aq.aqua_status(cache.desc) == aq.AQUA_OK
