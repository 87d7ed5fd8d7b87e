"""The per-CTA timeline summary (trace_report) on a hand-made trace."""
import numpy as np

from mxfp4_latent_moe_router_b200 import trace_report as tr

NAMES = ["dense_front", "expert_gate_up", "expert_down", "latent_tail", "fused_block"]


def _trace():
    t = np.zeros((5, 4, 24), np.uint64)
    base = 1_000_000
    # front: CTAs 0..3 start at base + 100c ns, end at base + 10 us + c us
    for c in range(4):
        t[0, c, tr.START] = base + 100 * c
        t[0, c, tr.END] = base + 10_000 + 1_000 * c
        t[0, c, tr.FIRST_STAGE] = base + 2_000
        t[0, c, tr.PIECES] = c
        t[0, c, tr.CONS_COMP] = 1_965 * 3  # 3 us at 1.965 GHz
        t[0, c, tr.SM] = c
        t[0, c, tr.LOGITS_PUBLISHED] = base + 4_000 + 100 * c if c < 3 else 0
    # the routing CTA (the last): stamps
    t[0, 3, tr.ROUTE_START] = base + 5_000
    t[0, 3, tr.ROUTE_SELECTED] = base + 7_000
    t[0, 3, tr.ROUTE_SCANNED] = base + 7_500
    t[0, 3, tr.ROUTE_END] = base + 8_000
    # expert gate/up: two CTAs
    for c in range(2):
        t[1, c, tr.START] = base + 13_000
        t[1, c, tr.END] = base + 20_000
        t[1, c, tr.FIRST_STAGE] = base + 15_000
        t[1, c, tr.SM] = c
    return t


def test_summary_times_and_counts():
    rows = tr.summarize(_trace(), NAMES)
    assert [r["kernel"] for r in rows] == ["dense_front", "expert_gate_up"]
    front, egu = rows
    assert front["ctas"] == 4 and egu["ctas"] == 2
    assert front["start_us"] == (0.0, 0.3)
    assert front["end_us"] == (10.0, 11.5, 13.0)
    assert front["pieces"] == (0, 3)
    assert abs(front["consumer_us"]["compute"] - 3.0) < 1e-9
    assert front["distinct_sms"] == 4
    r = front["routing_us"]
    assert (r["logits_published_last"], r["start"], r["selected"], r["tables_built"], r["published"]) == \
        (4.2, 5.0, 7.0, 7.5, 8.0)
    assert "routing_us" not in egu
    assert egu["first_stage_median_us"] == 15.0 and egu["life_us"] == (7.0, 7.0)
    text = tr.format_summary(rows)
    assert "dense_front" in text and "routing" in text


def test_empty_trace():
    assert tr.summarize(np.zeros((5, 2, 24), np.uint64), NAMES) == []
