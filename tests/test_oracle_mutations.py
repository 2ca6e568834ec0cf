"""The oracle's pins catch plausible mistakes.  Each case plants one mistake
in one oracle function (a dropped or wrong scale, a transposed operand, a
wrong sign, tie or index rule, a wrong head mapping, an off-by-one in the
visible tokens, a missing rounding, a wrong truncation side, a wrong H2O
rule), by rewriting a single expression of that function's source in a copy.
The copy replaces the function for the duration of the case. Every pin in
test_oracle_pins.py then runs, and at least one of them must fail.  CPU only;
the product is not involved.
"""
import inspect

import pytest

from oracle import aqua_oracle as O
import test_oracle_pins as PINS

# (oracle function, expression in its source, planted replacement, what the mistake is)
MUTANTS = [
    ("default_scale", "return 1.0 / np.sqrt(d)", "return 1.0", "scale dropped"),
    ("default_scale", "return 1.0 / np.sqrt(d)", "return 1.0 / d", "1/d instead of 1/sqrt(d)"),
    ("project", "@ np.asarray(P, dtype=np.float64)", "@ np.asarray(P, dtype=np.float64).T",
     "transposed projection"),
    ("select_dims", "mag = np.abs(qt[:m])", "mag = qt[:m]", "signed value instead of magnitude"),
    ("select_dims", "mag = np.abs(qt[:m])", "mag = -np.abs(qt[:m])", "smallest magnitudes"),
    ("select_dims", "np.lexsort((np.arange(m), -mag))", "np.lexsort((-np.arange(m), -mag))",
     "ties to the higher index"),
    ("select_dims", "mag = np.abs(qt[:m])", "mag = np.abs(qt[:m]); m = d; mag = np.abs(qt)",
     "truncation ignored in the selection"),
    ("select_dims", "return np.sort(order[:k])", "return order[:k]", "indices not in ascending order"),
    ("sparse_scores", "[:, S] @ np.asarray(qt, dtype=np.float64)[S]", "@ np.asarray(qt, dtype=np.float64)",
     "scores over every dimension"),
    ("softmax", "return e / z, float(mx + np.log(z))", "return e / z, float(np.log(z))",
     "log-sum-exp without the max"),
    ("decode", "g = h // G", "g = h % Hkv", "query head to KV head mapping"),
    ("decode", "V[b, g, :T], scale, m)", "V[b, g, :T] @ P[g], scale, m)", "projected values"),
    ("decode", "T = int(lens[b])", "T = int(lens[b]) - 1", "newest token not visible"),
    ("prefill", "T = pos0 + i + 1", "T = pos0 + i", "causal mask excludes the row's own token"),
    ("build_key_cache", "return store(kt[..., :m], kv_dtype)", "return kt[..., :m]",
     "cache storage rounding dropped"),
    ("build_key_cache", "return store(kt[..., :m], kv_dtype)", "return store(kt[..., d - m:], kv_dtype)",
     "trailing dimensions kept"),
    ("round_bf16", "np.round(np.ldexp(xv, -q))", "np.trunc(np.ldexp(xv, -q))", "bf16 rounding toward zero"),
    ("calibrate", "return vt.T.copy(), sigma", "return vt[::-1].T.copy(), sigma[::-1]",
     "ascending singular values"),
    ("calibrate", "X = np.asarray(X, dtype=np.float64)",
     "X = np.asarray(X, dtype=np.float64); X = X - X.mean(axis=0)", "centred (PCA instead of SVD)"),
    ("h2o_choose_victim", "score[i] == score[best] and pos[i] < pos[best]",
     "score[i] == score[best] and pos[i] > pos[best]", "H2O ties to the newest"),
    ("h2o_choose_victim", "if pos[i] > t_newest - recent:", "if pos[i] > t_newest - recent + 1:",
     "recent window one token short"),
    ("h2o_choose_victim", "if pos[i] > t_newest - recent:", "if pos[i] >= t_newest - recent:",
     "recent window one token long"),
    ("h2o_decode_step", "acc += p", "acc = p", "score of the last head only"),
    ("h2o_decode_step", "s.score[i] += acc[i]", "s.score[i] = acc[i]", "score not cumulative"),
    ("build_value_cache", "return store(vt[..., :m_v], kv_dtype)",
     "return store(vt[..., v.shape[-1] - m_v:], kv_dtype)", "trailing value dimensions kept"),
    ("build_value_cache", 'np.einsum("...gi,gij->...gj", v, P)', 'np.einsum("...gi,gji->...gj", v, P)',
     "values projected by the transpose of P"),
    ("build_value_cache", "return store(vt[..., :m_v], kv_dtype)", "return store(v[..., :m_v], kv_dtype)",
     "values pruned without the projection"),
    ("unproject_values", "[:, :m_v].T", "[:m_v, :]", "back-projection by rows of P instead of columns"),
    ("decode", "o = unproject_values(o, P[g])", "o = unproject_values(o, P[0])",
     "back-projection with another KV head's P"),
    ("h2o_decode_step", "unproject_values(o, P[g])", "unproject_values(o, P[0])",
     "H2O back-projection with another KV head's P"),
    ("query_energy_loss", "np.sum(qt[np.asarray(S)] ** 2)", "np.sum(np.abs(qt[np.asarray(S)]))",
     "retention measured on magnitudes instead of energy"),
    ("attention_output_loss", "np.linalg.norm(o_S - o) / np.linalg.norm(o)",
     "np.linalg.norm(o_S - o) / np.linalg.norm(o_S)", "output loss normalised by the approximate output"),
    ("select_first_dims", "return np.arange(k)", "return np.arange(d - k, d)", "slicing the last dimensions"),
    ("retention_losses", "select_dims(qt, k)", "select_dims(q[h], k)", "selection on the unprojected query"),
    ("breakeven_length", "d * d * (1.0 + 1.0 / G)", "d * d * 1.0", "break-even without the key projection share"),
    ("breakeven_length", "d * d * (1.0 + 1.0 / G)", "d * k * (1.0 + 1.0 / G)",
     "break-even with d k instead of d^2 projection work"),
    ("breakeven_length", "d * d * (1.0 + 1.0 / G)", "d * d * (1.0 + G)", "break-even with G key projections"),
]


def _mutant(fn_name: str, old: str, new: str):
    src = inspect.getsource(getattr(O, fn_name))
    assert src.count(old) == 1, f"{fn_name}: expression to mutate not found once"
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), f"<mutant of {fn_name}>", "exec"), ns)
    return ns[fn_name]


def _pins():
    calls = []
    for name, fn in vars(PINS).items():
        if not name.startswith("test_") or not callable(fn):
            continue
        if name == "test_select_dims_brute_force_tiny":
            calls += [(name, fn, {"seed": s}) for s in range(40)]
        elif name == "test_magnitude_selection_minimises_the_energy_loss":
            calls += [(name, fn, {"seed": s}) for s in range(6)]
        else:
            calls.append((name, fn, {}))
    return calls


def _failing_pins():
    failed = []
    for name, fn, kw in _pins():
        if name in failed:
            continue
        try:
            fn(**kw)
        except Exception:                      # an assertion, or an error the mistake provokes
            failed.append(name)
    return failed


def test_pins_pass_on_the_unmodified_oracle():
    assert _failing_pins() == []


@pytest.mark.parametrize("fn_name,old,new,what", MUTANTS, ids=[m[3] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(monkeypatch, fn_name, old, new, what):
    monkeypatch.setattr(O, fn_name, _mutant(fn_name, old, new))
    failed = _failing_pins()
    assert failed, f"no pin catches: {what}"
