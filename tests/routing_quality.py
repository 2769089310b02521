"""Approximation quality of page routing: per query head vs per KV group.

Reported, not gated: the pages give no quality figure for the routing.  For
each seeded synthetic workload (shrunk so that the fp64 oracle runs in
seconds) and each routing ("head", "group_sum", "group_max"), the oracle's
decode step is compared with

  * the same step with every page selected (the error of the routing alone),
  * dense attention of each query head over all raw values, projected by its
    rows of W_O (the routing plus the rank-r Value latent),

and the dense softmax mass (raw keys, all tokens) that falls on the pages a
head attends to is averaged over heads, as are the pages read per KV group.

    python -m tests.routing_quality [--seqs N] [--out FILE]
"""
from __future__ import annotations

import argparse
import json
import math
import time

import numpy as np

from long_context_decode_basiskv_b200.workloads import WORKLOADS, make_case, shrink
from oracle import basiskv_oracle as O
from tests.harness import OracleCase, to64

ROUTINGS = ["head", "group_sum", "group_max"]

CASES = {
    "llama3_8b_32k": shrink(WORKLOADS["llama3_8b_32k"], batch=2, name="llama3_8b_32k"),
    "single_seq_131k@32k": shrink(WORKLOADS["single_seq_131k"], context=32768, name="single_seq_131k@32k"),
    "llama3_70b_64k@32k": shrink(WORKLOADS["llama3_70b_64k"], batch=1, context=32768, name="llama3_70b_64k@32k"),
    "ragged_serving": shrink(WORKLOADS["ragged_serving"], batch=2, name="ragged_serving"),
}


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _dense(q, K, V, W_O, group):
    """sum_h softmax(q_h K_g^T / sqrt d) V_g W_O,h over every token, and the softmax rows."""
    Hq, d = q.shape
    y = np.zeros(W_O.shape[1])
    probs = []
    for h in range(Hq):
        g = h // group
        s = K[:, g] @ q[h] / math.sqrt(d)
        w = np.exp(s - s.max())
        w /= w.sum()
        probs.append(w)
        y += (w @ V[:, g]) @ W_O[h * d:(h + 1) * d]
    return y, probs


def measure(wl, seqs: int):
    case = make_case(wl, "cpu")
    oc = OracleCase(case)
    W_O = to64(case.W_O)
    group = wl.num_q_heads // wl.num_kv_heads
    rows = {r: {"y_rel_vs_all_pages": [], "y_rel_vs_dense": [], "mass_on_selected": [],
                "pages_per_group": []} for r in ROUTINGS}
    for b in range(min(seqs, wl.batch)):
        K, V = to64(case.keys[b]), to64(case.values[b])
        L = K.shape[0]
        q = to64(case.q[b])
        cache = O.prefill(K[:-1], V[:-1], oc.A, oc.P, oc.E, wl.page_size, oc.storage, capacity=L)
        cache.length = L - 1
        full = O.decode_step(cache, K[-1], V[-1], q, oc.A, oc.P, oc.E, oc.G, 1 << 30)
        y_dense, probs = _dense(q, K, V, W_O, group)
        for routing in ROUTINGS:
            cache.length = L - 1
            out = O.decode_step(cache, K[-1], V[-1], q, oc.A, oc.P, oc.E, oc.G, wl.top_k, routing=routing)
            r = rows[routing]
            r["y_rel_vs_all_pages"].append(_rel(out["y"], full["y"]))
            r["y_rel_vs_dense"].append(_rel(out["y"], y_dense))
            for h in range(wl.num_q_heads):
                tok = np.concatenate([np.arange(p * wl.page_size, min(L, (p + 1) * wl.page_size))
                                      for p in out["sel"][h]])
                r["mass_on_selected"].append(float(probs[h][tok].sum()))
            for g in range(wl.num_kv_heads):
                r["pages_per_group"].append(len(set().union(*[set(out["sel"][h].tolist())
                                                               for h in range(g * group, (g + 1) * group)])))
        rows["all_pages_vs_dense"] = rows.get("all_pages_vs_dense", []) + [_rel(full["y"], y_dense)]
    summary = {}
    for routing in ROUTINGS:
        summary[routing] = {k: round(float(np.mean(v)), 5) for k, v in rows[routing].items()}
    summary["all_pages_y_rel_vs_dense"] = round(float(np.mean(rows["all_pages_vs_dense"])), 5)
    return summary


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--seqs", type=int, default=1, help="sequences per workload")
    ap.add_argument("--out", default=None)
    ap.add_argument("--cases", nargs="*", default=sorted(CASES))
    args = ap.parse_args()
    report = {}
    for name in args.cases:
        t0 = time.time()
        report[name] = measure(CASES[name], args.seqs)
        report[name]["seconds"] = round(time.time() - t0, 1)
        print(name, json.dumps(report[name]), flush=True)
    if args.out:
        with open(args.out, "w") as f:
            json.dump(report, f, indent=1)


if __name__ == "__main__":
    main()
