import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """List every parity comparison: raw max |out - ref| / RMS next to the error
    beyond the output's own rounding (the figure the bf16 bar applies to)."""
    try:
        from gpu_helpers import RECORDS
    except ImportError:
        return
    if not RECORDS:
        return
    tr = terminalreporter
    tr.section("parity errors (max |out - ref| / RMS(ref))")
    tr.write_line(f"{'test':<78} {'label':<16} {'dtype':<5} {'raw':>10} {'beyond rounding':>16} {'rows':>9}")
    for test, label, dtype, raw, err, rows in RECORDS:
        tr.write_line(f"{test[-78:]:<78} {label[:16]:<16} {dtype:<5} {raw:10.3e} {err:16.3e} {rows:9d}")
    path = os.environ.get("SPCONV_PARITY_LOG")
    if path:
        import json
        with open(path, "w") as f:
            json.dump([dict(zip(("test", "label", "dtype", "raw", "beyond_rounding", "rows"), r)) for r in RECORDS], f,
                      indent=1)
