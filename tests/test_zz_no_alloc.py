"""aqua_decode_attn_static: the decode step for callers that cannot give the
library device scratch memory (their device memory belongs to another
allocator they may not bypass, or their interface has no place for a
workspace).  It uses a scratch array built into the library instead of
allocating.  The two entry points run the same kernels on the same inputs, so
their outputs, log-sum-exps and caches must be bit-identical, on two calls in
a row and across calls that alternate shapes, cache types and group sizes
(state left in the shared array by a larger call must not leak into the next
one).  One call is also checked against the oracle.  Collected last on
purpose, so a failure here cannot hide the other tests' results."""
import numpy as np
import pytest
import torch

import synth
from oracle import aqua_oracle as O
import sparse_dimension_attention_b200 as aq
from aqua_testlib import calib_P, fill_cache, oracle_cache, rel_err_rows, tdev, torch_dtype

pytestmark = pytest.mark.gpu

TOL_BF16_OUT = 2e-3


def _pair(B, Hq, Hkv, T, kv):
    """Two identical caches filled with the same history, and the step inputs."""
    P64, P32 = calib_P(Hkv)
    inp = synth.decode_inputs(B, Hq, Hkv, T, bf16=(kv == "bf16"), steps=2)
    caches = [aq.AquaCache(B, Hkv, T + 16, dtype=torch_dtype(kv)) for _ in range(2)]
    for c in caches:
        Pt = fill_cache(c, inp["k_hist"], inp["v_hist"], P32)
    return caches, inp, Pt, P64


def _step_both(caches, inp, Pt, s, Hq, k, kv, out_dtype):
    """Step s through aqua_decode_attn (caches[0]) and aqua_decode_attn_static (caches[1])."""
    dt = torch_dtype(kv)
    B = inp["q"].shape[1]
    q = tdev(inp["q"][s], dt)
    kn, vn = tdev(inp["k_new"][s], dt), tdev(inp["v_new"][s], dt)
    res = []
    for mode, c in enumerate(caches):
        out = torch.empty((B, Hq, 128), dtype=out_dtype, device="cuda")
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        sel = torch.empty((B, Hq, k), dtype=torch.int32, device="cuda")
        if mode == 0:
            ws = torch.zeros(aq.aqua_decode_workspace_size(c.desc, Hq), dtype=torch.uint8, device="cuda")
            aq.aqua_decode_attn(c.desc, q, Pt, Hq, k, out, ws, k_new=kn, v_new=vn, lse_out=lse, sel_out=sel)
        else:
            aq.aqua_decode_attn_static(c.desc, q, Pt, Hq, k, out, k_new=kn, v_new=vn, lse_out=lse, sel_out=sel)
        res.append((out, lse, sel))
    torch.cuda.synchronize()
    for a, b in zip(res[0], res[1]):
        assert torch.equal(a, b)
    for name in ("k_proj", "v", "len", "n_abs"):
        assert torch.equal(getattr(caches[0], name), getattr(caches[1], name)), name
    assert caches[0].max_len == caches[1].max_len
    return res[1]


def test_static_scratch_matches_workspace_entry_point():
    """Two calls in a row at the Llama head layout (32 query heads over 8 KV
    heads), bit-identical to the workspace entry point; the second call's
    output also against the oracle."""
    B, Hq, Hkv, T, k = 4, 32, 8, 2000, 96
    caches, inp, Pt, P64 = _pair(B, Hq, Hkv, T, "bf16")
    for s in range(2):
        out, lse, sel = _step_both(caches, inp, Pt, s, Hq, k, "bf16", torch.bfloat16)
    assert caches[1].max_len == T + 2 and (caches[1].len.cpu().numpy() == T + 2).all()
    k_all = np.concatenate([inp["k_hist"], inp["k_new"].transpose(1, 0, 2, 3)], axis=1)
    v_all = np.concatenate([inp["v_hist"], inp["v_new"].transpose(1, 0, 2, 3)], axis=1)
    ref = O.decode(inp["q"][1], P64, oracle_cache(k_all, P64, "bf16"), v_all.transpose(0, 2, 1, 3),
                   [T + 2] * B, k, out_dtype="bf16")
    assert np.max(rel_err_rows(out.float().cpu().numpy().astype(np.float64), ref["out"])) <= TOL_BF16_OUT
    assert aq.aqua_status(caches[1].desc) == aq.AQUA_OK


def test_static_scratch_alternating_shapes():
    """A large bf16 call (many units, split-K partials all over the array),
    then a small f32 call with one query head per KV head, then the large
    shape again: every call bit-identical to the workspace entry point."""
    big = _pair(32, 32, 8, 1500, "bf16")
    small = _pair(1, 2, 2, 300, "f32")
    _step_both(*big[:3], 0, 32, 64, "bf16", torch.bfloat16)
    _step_both(*small[:3], 0, 2, 96, "f32", torch.float32)
    _step_both(*big[:3], 1, 32, 64, "bf16", torch.float32)
    _step_both(*small[:3], 1, 2, 17, "f32", torch.float32)
    for c in (big[0][1], small[0][1]):
        assert aq.aqua_status(c.desc) == aq.AQUA_OK
        assert int(c.ctrl[1:].abs().sum().item()) == 0          # tickets back at zero


def test_static_scratch_rejects_shapes_beyond_its_size():
    big = aq.AquaCache(512, 8, 16)              # 4096 units: more scratch than the built-in 8 MiB
    q = torch.zeros((512, 32, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    P = torch.zeros((8, 128, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(aq.AquaError) as err:
        aq.aqua_decode_attn_static(big.desc, q, P, 32, 96, out)
    assert err.value.code == aq.abi.AQUA_ERR_WORKSPACE
