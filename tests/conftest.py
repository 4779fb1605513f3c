import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Boundary swaps of every GPU parity case run in this session: kernel
    index sets that differ from the oracle's only at the K-th boundary, where
    the two oracle scores lie within 1e-4 relative (counted, not hidden)."""
    mod = sys.modules.get("tests._parity")
    rows = getattr(mod, "RESULTS", None) if mod else None
    rows = [r for r in (rows or []) if "block_swaps" in r]
    if not rows:
        return
    tr = terminalreporter
    tr.write_sep("-", "boundary swaps vs the oracle (blocks/tokens: separate calls | select_step; groups)")
    parts = [f"{r['case']} {r['block_swaps']}/{r['token_swaps']}|{r.get('step_block_swaps', '-')}/"
             f"{r.get('step_token_swaps', '-')};{r['groups']}" for r in rows]
    line = ""
    for p in parts:
        if len(line) + len(p) > 150:
            tr.write_line(line.rstrip(", "))
            line = ""
        line += p + ", "
    if line:
        tr.write_line(line.rstrip(", "))
    tot = [sum(r.get(k, 0) for r in rows) for k in ("block_swaps", "token_swaps", "step_block_swaps", "step_token_swaps")]
    tr.write_line(f"total over {len(rows)} cases: blocks {tot[0]}, tokens {tot[1]} (separate calls); "
                  f"blocks {tot[2]}, tokens {tot[3]} (select_step)")
