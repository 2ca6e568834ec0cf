"""Helpers for the GPU parity tests: build caches through the C ABI, run the
library, run the oracle on the same seeded inputs, compare."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import aqua_oracle as O
import sparse_dimension_attention_b200 as aq

_P_CACHE = {}


def calib_P(Hkv: int = 1, n_q: int = 8192, n_k: int = 8192) -> tuple[np.ndarray, np.ndarray]:
    """P from the oracle's SVD of the synthetic calibration matrix, rounded to f32
    (both sides use exactly these numbers).  Returns (P64 [Hkv,d,d], P32)."""
    key = (n_q, n_k)
    if key not in _P_CACHE:
        P, _ = O.calibrate(synth.calibration_matrix(n_q=n_q, n_k=n_k))
        _P_CACHE[key] = P.astype(np.float32)
    P32 = np.ascontiguousarray(np.broadcast_to(_P_CACHE[key], (Hkv, 128, 128)))
    return P32.astype(np.float64), P32


def tdev(x: np.ndarray, dtype=torch.float32) -> torch.Tensor:
    return torch.from_numpy(np.array(x, order="C", copy=True)).to(dtype).cuda()


def torch_dtype(kv: str):
    return torch.bfloat16 if kv == "bf16" else torch.float32


def fill_cache(cache: aq.AquaCache, k_tok: np.ndarray, v_tok: np.ndarray, P32: np.ndarray, chunk: int | None = None):
    """Append tokens k_tok, v_tok [B, L, Hkv, d] through aqua_project_keys."""
    Pt = tdev(P32)
    L = k_tok.shape[1]
    chunk = chunk or L
    for s in range(0, L, chunk):
        e = min(L, s + chunk)
        kt = tdev(k_tok[:, s:e], cache.dtype)
        vt = tdev(v_tok[:, s:e], cache.dtype)
        aq.aqua_project_keys(cache.desc, kt, vt, Pt, e - s)
    torch.cuda.synchronize()
    return Pt


def run_decode(cache: aq.AquaCache, q: np.ndarray, Pt: torch.Tensor, k: int, out_dtype=torch.bfloat16,
               scores: bool = False):
    B, Hq, d = q.shape
    qt = tdev(q, cache.dtype)
    out = torch.empty((B, Hq, d), dtype=out_dtype, device="cuda")
    sel = torch.full((B, Hq, k), -1, dtype=torch.int32, device="cuda")
    qproj = torch.empty((B, Hq, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    sc = torch.zeros((B, Hq, cache.Tcap), dtype=torch.float32, device="cuda") if scores else None
    ws = torch.zeros(aq.aqua_decode_workspace_size(cache.desc, Hq), dtype=torch.uint8, device="cuda")
    aq.aqua_decode_attn(cache.desc, qt, Pt, Hq, k, out, ws, sel_out=sel, qproj_out=qproj, lse_out=lse,
                        scores_out=sc)
    torch.cuda.synchronize()
    res = {"out": out.float().cpu().numpy().astype(np.float64), "sel": sel.cpu().numpy(),
           "qt": qproj.cpu().numpy(), "lse": lse.cpu().numpy()}
    if scores:
        res["scores"] = sc.cpu().numpy()
    return res


def oracle_cache(k_tok: np.ndarray, P64: np.ndarray, kv: str, m: int | None = None) -> np.ndarray:
    """K~ [B, Hkv, T, m] (token-major) from the oracle."""
    return O.build_key_cache(k_tok, P64, kv, m).transpose(0, 2, 1, 3)


def rel_err_rows(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Relative L2 error per row (last axis)."""
    num = np.linalg.norm(a - b, axis=-1)
    den = np.linalg.norm(b, axis=-1)
    return num / np.maximum(den, 1e-30)


def check_selection(sel_gpu: np.ndarray, qt_gpu: np.ndarray, sel_ref: np.ndarray, qt_ref: np.ndarray, k: int,
                    m: int | None = None) -> int:
    """Exact-set parity.  (1) The oracle's selection on the GPU's own f32 q~ must
    equal the GPU's sets exactly.  (2) Against the f64 q~, every head whose gap
    between the k-th and (k+1)-th magnitude exceeds 1e-5 * max|q~| must match.
    Returns the number of near-tie heads skipped in (2)."""
    flat_sel = sel_gpu.reshape(-1, k)
    flat_qt = qt_gpu.reshape(-1, qt_gpu.shape[-1]).astype(np.float64)
    for i in range(flat_sel.shape[0]):
        np.testing.assert_array_equal(flat_sel[i], O.select_dims(flat_qt[i], k, m), err_msg=f"head {i}")
    near = 0
    fr = sel_ref.reshape(-1, k)
    fq = qt_ref.reshape(-1, qt_ref.shape[-1])
    for i in range(fr.shape[0]):
        mm = fq.shape[-1] if m is None else m
        mag = np.sort(np.abs(fq[i, :mm]))[::-1]
        gap = mag[k - 1] - (mag[k] if k < mm else -np.inf)
        if gap <= 1e-5 * mag[0]:
            near += 1
            continue
        np.testing.assert_array_equal(flat_sel[i], fr[i], err_msg=f"head {i}")
    return near
