"""Per-CTA timeline of one forward, summarised per kernel.

A plan created with the environment variable MOE_TRACE set records, for every
CTA of every launch slot, start and end times, pieces, finalisations, the
consumer and producer cycle split and the routing CTA's phase stamps
(``moe_debug_trace``; the slot layout is documented in include/moe.h).  This
module turns that array into one summary per kernel.

    MOE_TRACE=1 python -m mxfp4_latent_moe_router_b200.trace_report --workload b64

By default the forward is timed on its own (no other work on the GPU), after
three warm-up forwards, so the figures describe a single step, not a steady
stream.  With --steady the traced forward is the last of a CUDA graph of ten
back to back, so its first kernel overlaps the previous forward's last one as
in the benchmark (times are still relative to its own first CTA start).
"""
from __future__ import annotations

import argparse
import os

import numpy as np

# slot indices within a CTA's 24 values
START, END, PIECES, FINALIZES, ROUTE_START, ROUTE_END, FIRST_STAGE, FIN_NS = 0, 1, 2, 3, 4, 5, 6, 7
CONS_WAIT, CONS_COMP, CONS_END, PROD_WAIT, PROD_ISSUE, PROD_STAGES, SM = 8, 9, 10, 11, 12, 13, 14
ROUTE_CLEARED, ROUTE_SELECTED, ROUTE_SCANNED, LOGITS_PUBLISHED = 16, 17, 18, 19
ROUTE_FIRST_GROUP, ROUTE_STAGED, ROUTE_FIRST_TOKEN = 20, 21, 22
# expert kernels (slots the front kernel's routing uses): producer cycles in
# stage set-up (header, weight tile copies) and in the activation copies; the
# tensor-core MMA warp's waiting and issuing cycles
PROD_BEGIN, PROD_ACT, MMA_WAIT, MMA_ISSUE = 20, 21, 22, 23
EXPERT_KERNELS = ("expert_gate_up", "expert_down")


def summarize(trace: np.ndarray, names, clock_ghz: float = 1.965) -> list[dict]:
    """trace: uint64 [slots][num_sms][24] from ``moe_debug_trace``.  Times are
    returned in µs after the first CTA start of the forward; cycle counts are
    converted at clock_ghz."""
    t = trace.astype(np.int64)
    starts = t[:, :, START]
    if not (starts > 0).any():
        return []
    t0 = starts[starts > 0].min()
    us = lambda ns: (ns - t0) / 1e3  # noqa: E731
    out = []
    for k, name in enumerate(names):
        rows = t[k]
        used = rows[:, START] > 0
        if not used.any():
            continue
        r = rows[used]
        life = (r[:, END] - r[:, START]) / 1e3
        cyc = lambda col: float(np.median(r[:, col])) / (clock_ghz * 1e3)  # noqa: E731
        s = {
            "kernel": name,
            "ctas": int(used.sum()),
            "start_us": (float(us(r[:, START].min())), float(us(r[:, START].max()))),
            "first_stage_median_us": float(np.median(us(r[:, FIRST_STAGE]))),
            "end_us": (float(us(r[:, END].min())), float(np.median(us(r[:, END]))),
                       float(us(r[:, END].max()))),
            "life_us": (float(np.median(life)), float(life.max())),
            "pieces": (int(r[:, PIECES].min()), int(r[:, PIECES].max())),
            "finalize_us_max": float(r[:, FIN_NS].max() / 1e3),
            "consumer_us": {"wait": cyc(CONS_WAIT), "compute": cyc(CONS_COMP), "close": cyc(CONS_END)},
            "producer_us": {"wait": cyc(PROD_WAIT), "issue": cyc(PROD_ISSUE)},
            "stages_median": float(np.median(r[:, PROD_STAGES])),
            **({"producer_split_us": {"begin": cyc(PROD_BEGIN), "act": cyc(PROD_ACT)},
                "mma_warp_us": {"wait": cyc(MMA_WAIT), "issue": cyc(MMA_ISSUE)}}
               if name in EXPERT_KERNELS else {}),
            "distinct_sms": int(len(set(r[:, SM].tolist()))),
        }
        route = np.where(rows[:, ROUTE_START] > 0)[0]
        if len(route):
            c = rows[route[0]]
            pub = rows[:, LOGITS_PUBLISHED]
            st = lambda i: float(us(c[i])) if c[i] > 0 else None  # noqa: E731
            s["routing_us"] = {
                "logits_published_last": float(us(pub[pub > 0].max())) if (pub > 0).any() else None,
                "cleared": st(ROUTE_CLEARED), "staged_or_slices": st(ROUTE_STAGED),
                "first_token_or_merge": st(ROUTE_FIRST_TOKEN), "first_group": st(ROUTE_FIRST_GROUP),
                "start": float(us(c[ROUTE_START])),
                "selected": float(us(c[ROUTE_SELECTED])),
                "tables_built": float(us(c[ROUTE_SCANNED])),
                "published": float(us(c[ROUTE_END])),
            }
        out.append(s)
    return out


def format_summary(rows: list[dict]) -> str:
    lines = []
    for s in rows:
        lines.append(
            "%-15s ctas=%d start %.1f..%.1f  first stage %.1f  end %.1f / %.1f / %.1f (min/med/max)"
            "  pieces %d..%d  stages %.0f" % (
                s["kernel"], s["ctas"], *s["start_us"], s["first_stage_median_us"], *s["end_us"],
                *s["pieces"], s["stages_median"]))
        lines.append("    consumer wait %.1f compute %.1f close %.1f | producer wait %.1f issue %.1f (µs, median CTA)"
                     % (s["consumer_us"]["wait"], s["consumer_us"]["compute"], s["consumer_us"]["close"],
                        s["producer_us"]["wait"], s["producer_us"]["issue"]))
        if "producer_split_us" in s:
            lines.append("    producer set-up %.1f activations %.1f | MMA warp wait %.1f issue %.1f (µs, median CTA)"
                         % (s["producer_split_us"]["begin"], s["producer_split_us"]["act"],
                            s["mma_warp_us"]["wait"], s["mma_warp_us"]["issue"]))
        if "routing_us" in s:
            r = s["routing_us"]
            f = lambda v: "-" if v is None else "%.1f" % v  # noqa: E731
            lines.append("    routing: logits %s, start %.1f, cleared %s, slices/staged %s, merge/first token %s, "
                         "first group %s, selected %.1f, tables %.1f, published %.1f"
                         % (f(r["logits_published_last"]), r["start"], f(r["cleared"]),
                            f(r["staged_or_slices"]), f(r["first_token_or_merge"]), f(r["first_group"]),
                            r["selected"], r["tables_built"], r["published"]))
    return "\n".join(lines)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--workload", default="b1")
    ap.add_argument("--steady", action="store_true",
                    help="trace the last of ten forwards replayed back to back from a CUDA graph")
    args = ap.parse_args(argv)
    if not os.environ.get("MOE_TRACE"):
        raise SystemExit("set MOE_TRACE=1: the plan keeps the timeline only then")
    import torch

    import mxfp4_latent_moe_router_b200 as moe
    from mxfp4_latent_moe_router_b200 import synth

    shape = synth.SHAPES[args.workload]
    w = synth.make_weights(shape)
    plan = moe.MoePlan(moe.config_from_shape(shape))
    try:
        plan.load(moe.weights_to_device(w))
        del w
        x = torch.from_numpy(synth.make_x(shape).view(np.int16)).cuda()
        out = torch.empty_like(x)
        for _ in range(3):
            plan.forward(x, out)
        torch.cuda.synchronize()
        if args.steady:
            s = torch.cuda.Stream()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    for _ in range(10):
                        plan.forward(x, out, stream=s)
                g.replay()
                g.replay()
            s.synchronize()
            del g
        else:
            plan.forward(x, out)
        torch.cuda.synchronize()
        info = plan.info()
        tr = moe.moe_debug_trace(plan.handle, info.num_sms)
        print(format_summary(summarize(tr, moe.KERNEL_NAMES)))
    finally:
        plan.close()
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
