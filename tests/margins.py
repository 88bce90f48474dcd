"""Parity margins recorded by the GPU tests, printed at the end of the session.

Each GPU comparison against the oracle appends (what, output max-abs, output relative L2, state
relative L2) here; the conftest hook writes one line per comparison to stderr after the run, so a
quiet run (``pytest -q``) still shows how far inside the tolerances every case landed.
"""
MARGINS = []
NOTES = []


def note(line):
    """A free-form margin line (for checks that are not an output / state comparison)."""
    NOTES.append(str(line))


def record(what, o_max_abs, o_rel_l2, s_rel_l2=None):
    MARGINS.append((str(what), float(o_max_abs), float(o_rel_l2),
                    None if s_rel_l2 is None else float(s_rel_l2)))


def summary_lines():
    lines = [f"  {n}" for n in NOTES]
    if lines:
        lines.insert(0, "other margins:")
    if not MARGINS:
        return lines
    lines += ["parity margins against the fp64 oracle (tolerances: o max-abs 3e-2, o rel-L2 1e-2, "
             "state rel-L2 1e-2):"]
    for what, ma, rl, rs in MARGINS:
        st = "-" if rs is None else f"{rs:.2e}"
        lines.append(f"  {what}: o max-abs {ma:.2e}  o rel-L2 {rl:.2e}  state rel-L2 {st}")
    worst = max(MARGINS, key=lambda m: max(m[1] / 3e-2, m[2] / 1e-2, (m[3] or 0.0) / 1e-2))
    lines.append(f"  worst relative to its tolerance: {worst[0]}")
    return lines
