"""Guard words and the device time-out path on the GPU.

Every buffer the library writes (outputs, workspace, cache arrays) sits between
two 1 KB regions filled with a canary byte; after appends, decode steps with
the fused append, H2O updates and a prefill chunk, every canary must be
intact.  The time-out path: a wait on a barrier that nothing completes runs
out, the status word reports AQUA_ERR_TIMEOUT, and the context keeps working."""
import numpy as np
import pytest
import torch

import synth
import sparse_dimension_attention_b200 as aq
from sparse_dimension_attention_b200 import abi
from aqua_testlib import calib_P, tdev

pytestmark = pytest.mark.gpu

GUARD = 1024           # bytes on each side
CANARY = 0xA5


class Guarded:
    """Device buffers carved out of byte tensors with canary regions around them."""

    def __init__(self):
        self.raw = []

    def __call__(self, shape, dtype, zero=True):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        raw = torch.full((n + 2 * GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        inner = raw[GUARD:GUARD + n].view(dtype).view(shape)
        if zero:
            inner.zero_()
        self.raw.append(raw)
        return inner

    def check(self):
        torch.cuda.synchronize()
        for i, raw in enumerate(self.raw):
            head, tail = raw[:GUARD], raw[-GUARD:]
            assert bool((head == CANARY).all()) and bool((tail == CANARY).all()), f"guard {i} overwritten"


def _guarded_cache(gb, B, Hkv, Tcap, d_store=128, h2o=False):
    kp = gb((B, Hkv, d_store, Tcap), torch.bfloat16)
    v = gb((B, Hkv, Tcap, 128), torch.bfloat16)
    ln = gb((B,), torch.int32)
    na = gb((B,), torch.int32)
    ctrl = gb((abi.AQUA_CTRL_WORDS,), torch.int32)
    pos = gb((B, Hkv, Tcap), torch.int32) if h2o else None
    sc = gb((B, Hkv, Tcap), torch.float32) if h2o else None
    desc = abi.aqua_cache(kp.data_ptr(), v.data_ptr(), ln.data_ptr(), na.data_ptr(),
                          pos.data_ptr() if h2o else None, sc.data_ptr() if h2o else None, ctrl.data_ptr(),
                          B, Hkv, 128, d_store, Tcap, 0, abi.AQUA_BF16)
    return desc, (kp, v, ln, na, ctrl, pos, sc)


def test_guard_words_intact_decode_h2o():
    B, Hq, Hkv, T0, k, budget, steps = 3, 16, 4, 200, 64, 160, 6
    P64, P32 = calib_P(Hkv)
    gb = Guarded()
    desc, bufs = _guarded_cache(gb, B, Hkv, 256, d_store=96, h2o=True)
    Pt = tdev(P32)
    inp = synth.decode_inputs(B, Hq, Hkv, T0, bf16=True, steps=steps)
    aq.aqua_project_keys(desc, tdev(inp["k_hist"], torch.bfloat16), tdev(inp["v_hist"], torch.bfloat16), Pt, T0)
    out = gb((B, Hq, 128), torch.bfloat16)
    sel = gb((B, Hq, k), torch.int32)
    qp = gb((B, Hq, 128), torch.float32)
    sco = gb((B, Hq, 256), torch.float32)
    lse = gb((B, Hq), torch.float32)
    ev = gb((B, Hkv), torch.int32)
    ws = gb((aq.aqua_decode_workspace_size(desc, Hq),), torch.uint8)
    for s in range(steps):
        aq.aqua_decode_attn(desc, tdev(inp["q"][s], torch.bfloat16), Pt, Hq, k, out, ws,
                            k_new=tdev(inp["k_new"][s], torch.bfloat16), v_new=tdev(inp["v_new"][s], torch.bfloat16),
                            sel_out=sel, qproj_out=qp, scores_out=sco, lse_out=lse)
        aq.aqua_h2o_update(desc, sco, lse, Hq, budget, 32, ev)
    gb.check()
    assert aq.aqua_status(desc) == aq.AQUA_OK
    assert bool(torch.isfinite(out.float()).all())
    assert int(bufs[2][0].item()) == T0                          # one append and one eviction per step


def test_guard_words_intact_prefill():
    B, Hq, Hkv, L = 2, 8, 2, 150
    P64, P32 = calib_P(Hkv)
    gb = Guarded()
    desc, bufs = _guarded_cache(gb, B, Hkv, 160)
    Pt = tdev(P32)
    inp = synth.prefill_inputs(L, Hq, Hkv, bf16=True, B=B)
    aq.aqua_project_keys(desc, tdev(inp["k"], torch.bfloat16), tdev(inp["v"], torch.bfloat16), Pt, L)
    out = gb((B, L, Hq, 128), torch.float32)
    sel = gb((B, L, Hq, 96), torch.int32)
    ws = gb((aq.aqua_prefill_workspace_size(desc, Hq, L),), torch.uint8)
    aq.aqua_prefill_attn(desc, tdev(inp["q"], torch.bfloat16), 0, L, Pt, Hq, 96, out, ws, sel_out=sel)
    gb.check()
    assert aq.aqua_status(desc) == aq.AQUA_OK
    assert bool(torch.isfinite(out).all())


def test_device_wait_times_out_and_context_survives():
    """A bounded wait on a barrier nothing completes reports AQUA_ERR_TIMEOUT;
    afterwards a normal decode step runs and matches a fresh run."""
    Hkv = 1
    P64, P32 = calib_P(Hkv)
    cache = aq.AquaCache(1, Hkv, 64)
    aq.aqua_selftest_wait_timeout(cache.desc, 20_000_000)            # 20 ms
    assert aq.aqua_status(cache.desc) == abi.AQUA_ERR_TIMEOUT
    assert aq.aqua_status(cache.desc) == aq.AQUA_OK                  # the status word was read and cleared
    inp = synth.decode_inputs(1, 4, Hkv, 40, bf16=True, steps=1)
    Pt = tdev(P32)
    aq.aqua_project_keys(cache.desc, tdev(inp["k_hist"], torch.bfloat16), tdev(inp["v_hist"], torch.bfloat16), Pt, 40)
    outs = []
    for _ in range(2):
        out = torch.empty((1, 4, 128), dtype=torch.float32, device="cuda")
        ws = torch.zeros(aq.aqua_decode_workspace_size(cache.desc, 4), dtype=torch.uint8, device="cuda")
        aq.aqua_decode_attn(cache.desc, tdev(inp["q"][0], torch.bfloat16), Pt, 4, 64, out, ws)
        outs.append(out.cpu())
    assert aq.aqua_status(cache.desc) == aq.AQUA_OK
    assert torch.equal(outs[0], outs[1]) and bool(torch.isfinite(outs[0]).all())
