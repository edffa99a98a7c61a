"""Plants plausible mistakes in copies of the oracle (on the CPU) and checks that the pins
catch every one: a pin suite that a dropped term, a flipped sign, a transposed operand or a
reversed tie-break slips through would not pin anything."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

from oracle import build as oracle_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, text in oracle.cpp, replacement, which occurrence to replace [0-based])
MUTANTS = [
    ("silu_sign", "g / (1.0 + exp(-g))", "g / (1.0 + exp(g))", 0),
    ("silu_dropped", "return g / (1.0 + exp(-g));", "return g;", 0),
    ("keep_count_no_guard", "floor(s * (double)I + 1e-9)", "floor(s * (double)I)", 0),
    ("keep_count_off_by_one", "(long)I - (long)floor", "(long)I - 1 - (long)floor", 0),
    ("neuron_tie_reversed", "return p < q;", "return p > q;", 0),
    ("keeps_lowest", "return score[p] > score[q];", "return score[p] < score[q];", 0),
    ("down_transposed", "(size_t)h * I + n", "(size_t)n * H + h", 0),
    ("threshold_not_strict", "score[n] > sel.threshold", "score[n] >= sel.threshold", 0),
    ("softmax_denominator", "z += exp(logits[idx[i]] - m);", "z += exp(logits[idx[i]]);", 0),
    ("shared_dropped", "j < k ? w[(size_t)t * k + j] : 1.0", "j < k ? w[(size_t)t * k + j] : 0.0", 0),
    ("expert_tie_reversed", "return p < q;", "return p > q;", 1),
    ("up_dropped", "double coef = a[n] * u;", "double coef = a[n];", 0),
    ("gate_without_x", "load(wg, elt, (size_t)n * H + h) * xd[h]", "load(wg, elt, (size_t)n * H + h)", 0),
    ("signed_score", "score[n] = fabs(a[n]);", "score[n] = a[n];", 0),
    ("sigmoid_sign", "1.0 / (1.0 + exp(-logits[idx[i]]))", "1.0 / (1.0 + exp(logits[idx[i]]))", 0),
    ("calibration_index", "scores[(size_t)(m - 1)]", "scores[(size_t)m]", 0),
    ("softmax_all_as_topk", "if (L.route == 1) {\n    for (int e = 0; e < E; ++e) z +=",
     "if (L.route == 99) {\n    for (int e = 0; e < E; ++e) z +=", 0),
    ("weight_not_applied", "o[h] += wj * yj[h];", "o[h] += yj[h];", 0),
    ("score_from_gate", "score[n] = fabs(a[n]);", "score[n] = fabs(g[n]);", 0),
    ("calibration_score_from_gate", "scores[(size_t)job * In + n] = fabs(a[n]);",
     "scores[(size_t)job * In + n] = fabs(g[n]);", 0),
    ("router_transposed", "load(L.router, L.elt, (size_t)e * H + h)",
     "load(L.router, L.elt, (size_t)h * E + e)", 0),
    ("calibration_ceil", "(long long)floor(s * (double)N)", "(long long)ceil(s * (double)N)", 0),
    ("shared_uses_routed_sparsity", "      sel = shared;", "      sel = routed;", 0),
    ("h_from_g_not_silu", "keep, a.data(), &y", "keep, g.data(), &y", 0),
    ("roster_bias_on_weights", "route_weights(*L, lg.data(), idx + (size_t)t * k",
     "route_weights(*L, sel.data(), idx + (size_t)t * k", 0),
    ("roster_tie_reversed", "return p < q;", "return p > q;", 2),
    ("roster_no_exploration", "else if (distinct < m)", "else if (distinct < 0)", 0),
    ("roster_barrier_sign", "b[e] = member[e] ? delta : -delta;",
     "b[e] = member[e] ? -delta : delta;", 0),
    ("roster_pin_ignored", "if (pinned[t]) b[e]", "if (pinned[t] && 0) b[e]", 0),
    ("roster_update_ignored", "counts[(size_t)t * E + e] += 1;", "counts[(size_t)t * E + e] += 0;", 0),
]


def _replace_nth(text, old, new, n):
    start = -1
    for _ in range(n + 1):
        start = text.find(old, start + 1)
        assert start >= 0, f"mutation anchor not found: {old!r} #{n}"
    return text[:start] + new + text[start + len(old):]


def _run_pins(paths):
    proc = subprocess.run([sys.executable, "-m", "tests.oracle_pins", *paths], cwd=ROOT,
                          capture_output=True, text=True, timeout=900)
    res = {}
    for line in proc.stdout.splitlines():
        if line.startswith("FAILED_PINS "):
            path, failed = line[len("FAILED_PINS "):].split("=", 1)
            res[path] = [p for p in failed.split(",") if p]
    return res


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    d = tmp_path_factory.mktemp("mutants")
    src = open(oracle_build.SRC).read()

    def make(m):
        name, old, new, nth = m
        mutated = _replace_nth(src, old, new, nth)
        assert mutated != src
        cpp = d / f"{name}.cpp"
        cpp.write_text(mutated)
        so = str(d / f"lib{name}.so")
        oracle_build.compile_oracle(str(cpp), so, extra=("-O1",))
        return name, so

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        sos = dict(ex.map(make, MUTANTS))
    res = _run_pins(list(sos.values()))
    out = {}
    for name, so in sos.items():
        if so not in res:  # the batch run died on an earlier mutant: run this one alone
            alone = _run_pins([so])
            out[name] = alone.get(so, ["crashed"])
        else:
            out[name] = res[so]
    return out


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, mutant_results):
    assert mutant_results[name], f"mutant {name} passed every pin"
