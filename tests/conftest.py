import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Totals of the parity comparisons of the session, with the two kinds of exemption apart:
    inside the 1e-6 band around a cut (allowed) and outside it but inside the fp32 bound
    (listed one by one; a test fails on them unless it names an allowance)."""
    from tests import parity
    recs = parity.RECORDS
    if not recs:
        return
    tr = terminalreporter
    tr.section("parity exemptions")
    tot = lambda f: sum(f(r) for r in recs)
    tr.write_line(
        f"comparisons={len(recs)} tokens_routed={tot(lambda r: r.tokens_routed)} "
        f"pairs_selected={tot(lambda r: r.pairs)} tokens_output={tot(lambda r: r.tokens_output)}")
    tr.write_line(
        f"within 1e-6 of the cut: routing experts={tot(lambda r: r.route_band)} "
        f"selection pairs={tot(lambda r: r.sel_band_pairs)} "
        f"neurons={tot(lambda r: r.sel_band_neurons)}")
    tr.write_line(
        f"outside 1e-6, inside the fp32 bound only: routing={tot(lambda r: len(r.route_fp32_only))} "
        f"selection={tot(lambda r: len(r.sel_fp32_only))}")
    for r in recs:
        if r.fp32_only or r.route_band or r.sel_band_pairs:
            tr.write_line(f"  {r.name}: {r}")
    tr.write_line(f"max scaled output error={max(r.max_err for r in recs):.3e}")
