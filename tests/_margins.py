"""Measured parity margins of the GPU tests, printed at the end of the run.

Every element-wise comparison against the oracle records its worst errors
here, so that a passing run still shows how far each case sits from the
tolerances (O max-abs 2e-2, O mean-abs 2e-3, lse max-abs 1e-3).
"""

RECORDS = []


def record(what, o_max, o_mean, lse_max):
    RECORDS.append((str(what), float(o_max), float(o_mean), float(lse_max)))


def summary_lines():
    if not RECORDS:
        return []
    out = [f"{'case':<64} {'O max-abs':>10} {'O mean-abs':>11} {'lse max-abs':>12}"]
    for what, a, b, c in RECORDS:
        out.append(f"{what[:64]:<64} {a:10.3e} {b:11.3e} {c:12.3e}")
    worst = max(RECORDS, key=lambda r: r[1] / 2e-2)
    out.append(f"largest O max-abs relative to its bound: {worst[1]:.3e} of 2e-2 ({worst[0]})")
    return out
