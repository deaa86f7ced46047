"""The per-CTA report of the timeline tool, on synthetic marks (no GPU): a planted phase shift
and planted phase durations must come out as planted."""
import numpy as np

from bit_dequant_expert_gemv_b200.timeline import timeline as T

# event ids of the engine's marks that the per-CTA view reads, with planted times (ns after the
# CTA's unit start): x ready, router done, x digits, shared g/u done, top-K start, logits
# stored, top-K done, expert 0 and 3 gate/up, shared down, last down segments, outputs
PLANT = [(24, 0), (25, 2500), (26, 3900), (27, 6600), (3, 6700), (70, 2400), (4, 10500),
         (30, 11500), (38, 13500), (33, 19700), (41, 21600), (28, 22000), (29, 24800),
         (56, 31000), (57, 33000), (62, 33700)]
PERIOD = 33000


def synthetic(late, shift_ns):
    buf = np.zeros((T.ALL_CTAS, T.UNITS, T.EVENTS), dtype=np.uint64)
    for c in range(T.ALL_CTAS):
        shift = shift_ns if c in late else 10 * (c % 7)
        for u in range(T.UNITS):
            t0 = 10**9 + u * PERIOD + shift
            for ev, dt in PLANT:
                buf[c, u, ev] = t0 + dt
    return buf


def test_report_finds_the_planted_shift_and_durations(capsys):
    T.report_all_ctas(synthetic({90, 91}, 2400), T.ALL_CTAS)
    out = capsys.readouterr().out
    latest = out.split("latest:")[1].split("\n")[0]
    assert latest.split()[:2] == ["CTA", "90"] or latest.split()[:2] == ["CTA", "91"]
    assert "+2.3" in latest.split("CTA")[1] or "+2.4" in latest.split("CTA")[1]
    rows = {line.split()[0]: line.split()[-3:] for line in out.splitlines()
            if line.startswith("  ") and line.split()[0] in ("router", "top-K", "outputs")}
    assert rows["router"] == ["2.50", "2.50", "2.50"]
    assert rows["top-K"] == ["3.80", "3.80", "3.80"]
    assert rows["outputs"] == ["0.70", "0.70", "0.70"]
    period = [line for line in out.splitlines() if "unit period" in line][0].split()[-3:]
    assert period == ["33.00", "33.00", "33.00"]
    # the last logits (the late CTAs': shift 2.4 + 2.4 us) against the median CTA's top-K
    # start (6.7 us plus its small shift of 0.03 us)
    gap = float(out.split("top-K start: median")[1].split()[0])
    assert abs(gap - (2.4 + 2.4 - 6.7 - 0.03)) < 0.02
