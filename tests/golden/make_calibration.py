"""Write tests/golden/top_p_calibrated.json: per-head top-p for the ~90%-sparsity workloads.

The workloads "wan1.3b", "wan14b" and "hunyuan" fix a target fraction of
skipped key blocks (after the text-keep and frame-0 overrides) rather than a
top-p value.  For every head this script bisects p on the oracle's own
selection (CPU oracle only: pool -> P' -> top-p -> overrides) until the
head's block density is as close as it gets to 1 - target.  The resulting fp32
values are then fed unchanged to both the oracle and the CUDA path.

Run:  python tests/golden/make_calibration.py [workload ...]
"""
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from block_sparse_attention_45_b200 import synth  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "top_p_calibrated.json")


def density(ora, L1, probs_h, flags, p):
    m, _ = ora.topp(L1, probs_h, np.float32(p))
    m = ora.overrides(L1, flags, m)
    return float(m.mean())


def calibrate(name, ora):
    w = synth.WORKLOADS[name]
    target = 1.0 - w.target_skip
    L = w.layout()
    ps, dens = [], []
    t0 = time.time()
    for h in range(w.heads):
        x = synth.generate(w, ("q", "k"), heads=[h])
        L1 = dict(L, heads=1)
        qc = ora.pool(L1, x["q"], w.q_block)
        kc = ora.pool(L1, x["k"], w.k_block)
        P = ora.scores(L1, qc, kc)
        lo, hi = 0.0, 1.0
        dlo = density(ora, L1, P, w.flags, lo)
        if dlo >= target:
            best = lo
        else:
            for _ in range(30):
                mid = float(np.float32((lo + hi) / 2))
                if mid in (lo, hi):
                    break
                if density(ora, L1, P, w.flags, mid) < target:
                    lo = mid
                else:
                    hi = mid
            dl, dh = density(ora, L1, P, w.flags, lo), density(ora, L1, P, w.flags, hi)
            best = lo if abs(dl - target) <= abs(dh - target) else hi
        ps.append(float(np.float32(best)))
        dens.append(density(ora, L1, P, w.flags, best))
        print("%s head %d: p=%.6f density=%.4f (%.0fs)" % (name, h, ps[-1], dens[-1], time.time() - t0),
              flush=True)
    return dict(top_p=ps, density=dens, target_skip=w.target_skip,
                mean_density=float(np.mean(dens)))


def main(names):
    ora = oracle.default()
    data = json.load(open(OUT)) if os.path.exists(OUT) else {}
    data["_source"] = ("Per-head top-p calibrated on the CPU oracle's selection (pool, P', "
                       "per-row top-p, text keep, frame-0 override) so that each head skips "
                       "target_skip of its key blocks; written by tests/golden/make_calibration.py.")
    for n in names:
        data[n] = calibrate(n, ora)
        with open(OUT, "w") as f:
            json.dump(data, f, indent=1)


if __name__ == "__main__":
    main(sys.argv[1:] or ["wan1.3b", "wan14b", "hunyuan"])
