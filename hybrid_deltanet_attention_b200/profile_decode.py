"""Small decode driver for profilers and the per-barrier phase trace.

    python -m hybrid_deltanet_attention_b200.profile_decode [--model 0.8b|tiny] [--prompt 8] [--steps 4] [--trace]

Loads the seeded synthetic model, feeds a short prompt (one decode launch per
token) and runs `--steps` decode launches. With --trace it prints, for the last
launch, CTA 0's time between consecutive grid-barrier exits (the phase times) and
its wait inside each barrier, in microseconds.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--model", default="0.8b")
    ap.add_argument("--prompt", type=int, default=8)
    ap.add_argument("--steps", type=int, default=4)
    ap.add_argument("--trace", action="store_true")
    ap.add_argument("--mhz", type=float, default=1965.0, help="SM clock used to convert trace cycles to us")
    ap.add_argument("--device-weights", action="store_true",
                    help="4-bit models: generate the blocks on the device (timing only, see synth.device_q4_weights)")
    args = ap.parse_args()

    import numpy as np
    import torch
    import synth
    import hybrid_deltanet_attention_b200 as hda

    cfg = synth.CONFIGS[args.model]
    dev = torch.device("cuda", 0)
    weights = (synth.device_q4_weights(cfg, dev, cfg.seed) if args.device_weights
               else hda.weights_to_device(synth.make_weights(cfg), dev))
    m = hda.Model(cfg, weights, max_ctx=args.prompt + args.steps + 8)
    del weights
    tok = torch.empty(args.steps + 1, dtype=torch.int32, device=dev)
    m.prefill(torch.from_numpy(synth.make_prompt(cfg, args.prompt)).to(dev), next_token=tok[0:1])
    q4 = cfg.weight_format == synth.W_Q4K
    nbar = sum((5 if q4 else 3) if k == "D" else (6 if q4 else 4) for k in cfg.pattern)
    G = int(m.sizes.grid_ctas)
    buf = torch.zeros(16384 + 2 * (nbar + 1) * G, dtype=torch.int64, device=dev) if args.trace else None
    for i in range(args.steps):
        if buf is not None and i == args.steps - 1:
            m.phase_trace(buf)
        m.decode(tok[i:i + 1], tok[i + 1:i + 2])
    m.phase_trace(None)
    err = m.sync()
    if err:
        raise SystemExit(f"device error word 0x{err:x}")
    if buf is not None:
        raw = buf.cpu().numpy()
        t = raw[:16384].astype("float64") * (1000.0 / args.mhz)      # cycles -> ns
        exits = [t[0]] + [t[2 * k] for k in range(1, nbar + 1)]
        arrivals = [t[2 * k - 1] for k in range(1, nbar + 1)]
        end = t[2 * nbar + 1]
        phases = [(exits[k + 1] - exits[k]) / 1e3 for k in range(nbar)] + [(end - exits[nbar]) / 1e3]
        waits = [(exits[k] - arrivals[k - 1]) / 1e3 for k in range(1, nbar + 1)]
        names = []
        for li, kind in enumerate(cfg.pattern):
            if q4:
                names += [f"L{li}.in", f"L{li}.dn", f"L{li}.out", f"L{li}.gateup", f"L{li}.down"] if kind == "D" else \
                         [f"L{li}.in", f"L{li}.attn", f"L{li}.attn_out", f"L{li}.out", f"L{li}.gateup", f"L{li}.down"]
            else:
                names += [f"L{li}.in", f"L{li}.dn+out", f"L{li}.mlp"] if kind == "D" else \
                         [f"L{li}.in", f"L{li}.attn", f"L{li}.attn_out", f"L{li}.mlp"]
        names.append("lm_head")
        rows = [{"phase": n, "us": round(p, 2), "barrier_wait_us": round(w, 2) if i < len(waits) else None}
                for i, (n, p, w) in enumerate(zip(names, phases, waits + [0.0]))]
        total = (end - t[0]) / 1e3
        chunks = []
        for n in range((len(t) - 512) // 4):
            iss, arr, acq, done = t[512 + 4 * n], t[513 + 4 * n], t[514 + 4 * n], t[515 + 4 * n]
            if iss == 0 and acq == 0:
                break
            chunks.append([round((x - t[0]) / 1e3, 3) for x in (iss, arr, acq, done)])
        # all CTAs (global timer, ns): per phase kind, the work (median arrival - median
        # exit of the previous barrier), the skew (last arrival - median arrival) and the
        # propagation (median exit - last arrival)
        grid = raw[16384:16384 + 2 * (nbar + 1) * G].astype("float64").reshape(nbar + 1, G, 2)
        kinds = {}
        for k in range(1, nbar + 1):
            a, e = grid[k, :, 0], grid[k, :, 1]
            work = (np.median(a) - np.median(grid[k - 1, :, 1])) / 1e3 if k > 1 else None
            kind = names[k - 1].split(".")[-1]
            d = kinds.setdefault(kind, {"n": 0, "work_us": 0.0, "skew_us": 0.0, "prop_us": 0.0})
            d["n"] += 1
            d["work_us"] += (work or 0.0)
            d["skew_us"] += (a.max() - np.median(a)) / 1e3
            d["prop_us"] += (np.median(e) - a.max()) / 1e3
        for d in kinds.values():
            for key in ("work_us", "skew_us", "prop_us"):
                d[key] = round(d[key] / d["n"], 3)
        print(json.dumps({"total_us": round(total, 1), "phases": rows, "exits_us": [round((e - t[0]) / 1e3, 2) for e in exits],
                          "chunks_issue_wait_have_done_us": chunks, "grid_barriers": kinds}))
    print(f"ok: {m.launches} launches")


if __name__ == "__main__":
    main()
