"""Magnitude selection versus slicing off the first dimensions, on the synthetic workload.

TEST INFRASTRUCTURE (CPU only): computes, with the oracle's functions, the two
retention losses (query energy outside the kept dimensions; relative error of
the attention output against standard attention) of AQUA's magnitude
selection and of keeping the first k projected dimensions, for several k.
The edgentiq blog ("Validation and Generalizability") reports that magnitude
selection roughly halves the information retention loss of slicing on
Llama-3.1-8B; these inputs are synthetic (the anisotropic query/key law of the
benchmark, P from the SVD of its calibration matrix), so the numbers describe
this law, not a language model.

    python oracle/retention_diagnostic.py [--T 4096] [--kv-heads 4] [--group 4] [--json out.json]
"""
from __future__ import annotations

import argparse
import json
import os
import sys


_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if _ROOT not in sys.path:
    sys.path.insert(0, _ROOT)

import synth  # noqa: E402
from oracle import aqua_oracle as O  # noqa: E402


def run(T: int = 4096, kv_heads: int = 4, group: int = 4, ks=(112, 96, 64, 32)) -> dict:
    P, _ = O.calibrate(synth.calibration_matrix())
    inp = synth.decode_inputs(1, kv_heads * group, kv_heads, T, bf16=False, steps=1)
    q = inp["q"][0, 0]                                       # [Hq, d]
    rows = []
    for k in ks:
        acc = {"magnitude": {"energy": 0.0, "output": 0.0}, "slicing": {"energy": 0.0, "output": 0.0}}
        for g in range(kv_heads):
            r = O.retention_losses(q[g * group:(g + 1) * group], P, inp["k_hist"][0, :, g], inp["v_hist"][0, :, g], k)
            for name in acc:
                for m in acc[name]:
                    acc[name][m] += r[name][m] / kv_heads
        rows.append({"k": k, **{f"{n}_{m}": acc[n][m] for n in acc for m in acc[n]},
                     "output_loss_ratio_slicing_over_magnitude": acc["slicing"]["output"] / acc["magnitude"]["output"],
                     "energy_loss_ratio_slicing_over_magnitude": acc["slicing"]["energy"] / acc["magnitude"]["energy"]})
    return {"T": T, "query_heads": kv_heads * group, "kv_heads": kv_heads, "rows": rows}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--T", type=int, default=4096)
    ap.add_argument("--kv-heads", type=int, default=4)
    ap.add_argument("--group", type=int, default=4)
    ap.add_argument("--json", default=None)
    a = ap.parse_args()
    res = run(a.T, a.kv_heads, a.group)
    print(f"T={res['T']}, {res['query_heads']} query heads over {res['kv_heads']} KV heads (synthetic law)")
    print(f"{'k':>4} | {'energy loss: magnitude':>22} {'slicing':>9} {'ratio':>6} | "
          f"{'output loss: magnitude':>22} {'slicing':>9} {'ratio':>6}")
    for r in res["rows"]:
        print(f"{r['k']:>4} | {r['magnitude_energy']:>22.3e} {r['slicing_energy']:>9.3e} "
              f"{r['energy_loss_ratio_slicing_over_magnitude']:>6.2f} | {r['magnitude_output']:>22.3e} "
              f"{r['slicing_output']:>9.3e} {r['output_loss_ratio_slicing_over_magnitude']:>6.2f}")
    if a.json:
        with open(a.json, "w") as f:
            json.dump(res, f, indent=1)


if __name__ == "__main__":
    main()
