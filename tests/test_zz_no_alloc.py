"""aqua_decode_attn_static: the decode step for callers that cannot give the
library device scratch memory (their device memory belongs to another
allocator, or their interface has no place for a workspace).  It uses a
scratch array built into the library instead of allocating.  Checked against
aqua_decode_attn (which takes a caller workspace) on two calls in a row, with
the tolerance of the decode parity tests.  Collected last on purpose, so a
failure here cannot hide the other tests' results."""
import numpy as np
import pytest
import torch

import synth
import sparse_dimension_attention_b200 as aq
from aqua_testlib import calib_P, fill_cache, rel_err_rows, tdev

pytestmark = pytest.mark.gpu

TOL_BF16_OUT = 2e-3


def test_static_scratch_matches_workspace_entry_point():
    B, Hq, Hkv, T, k = 4, 32, 8, 2000, 96
    P64, P32 = calib_P(Hkv)
    inp = synth.decode_inputs(B, Hq, Hkv, T, bf16=True, steps=2)
    with_ws = aq.AquaCache(B, Hkv, T + 16)
    static = aq.AquaCache(B, Hkv, T + 16)
    for c in (with_ws, static):
        Pt = fill_cache(c, inp["k_hist"], inp["v_hist"], P32)
    ws = torch.zeros(aq.aqua_decode_workspace_size(with_ws.desc, Hq), dtype=torch.uint8, device="cuda")
    for s in range(2):                                   # two calls in a row
        q = tdev(inp["q"][s], torch.bfloat16)
        kn, vn = tdev(inp["k_new"][s], torch.bfloat16), tdev(inp["v_new"][s], torch.bfloat16)
        out_ws = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
        out_st = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
        lse_ws = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        lse_st = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        aq.aqua_decode_attn(with_ws.desc, q, Pt, Hq, k, out_ws, ws, k_new=kn, v_new=vn, lse_out=lse_ws)
        aq.aqua_decode_attn_static(static.desc, q, Pt, Hq, k, out_st, k_new=kn, v_new=vn, lse_out=lse_st)
        torch.cuda.synchronize()
        a = out_st.float().cpu().numpy().astype(np.float64)
        b = out_ws.float().cpu().numpy().astype(np.float64)
        assert np.max(rel_err_rows(a, b)) <= TOL_BF16_OUT
        np.testing.assert_allclose(lse_st.cpu().numpy(), lse_ws.cpu().numpy(), rtol=1e-6, atol=1e-6)
    assert torch.equal(with_ws.len, static.len) and static.max_len == with_ws.max_len == T + 2
    assert aq.aqua_status(static.desc) == aq.AQUA_OK


def test_static_scratch_rejects_shapes_beyond_its_size():
    big = aq.AquaCache(512, 8, 16)              # 4096 units: more scratch than the built-in 8 MiB
    q = torch.zeros((512, 32, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    P = torch.zeros((8, 128, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(aq.AquaError) as err:
        aq.aqua_decode_attn_static(big.desc, q, P, 32, 96, out)
    assert err.value.code == aq.abi.AQUA_ERR_WORKSPACE
