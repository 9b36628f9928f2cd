"""Writes vmajor_tau.json: the V-Major threshold tau of each workload and
target active fraction, computed by the oracle from the seeded inputs.

Reading (the CoCoDiff article gives no threshold value, only that it is
tuned per denoising stage): tau sits at the midpoint of the widest gap between
consecutive sorted per-token L1 values within 1% of the target rank, so that
the mask does not depend on the precision or order of the fp32 sum.

Run from the repository root: python tests/golden/make_vmajor_tau.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def main():
    out = {"_source": __doc__.strip().splitlines()[0], "workloads": {}}
    for w in synth.WORKLOADS:
        if not w.vmajor_f:
            continue
        n = w.B * w.T * w.S
        cur, prev = synth.vmajor_pair(w, n, w.C)
        l1 = oracle.l1_change(cur, prev)
        entry = {}
        for f in w.vmajor_f:
            tau, margin, frac = oracle.tau_for_fraction(l1, f)
            entry[str(f)] = {"tau": tau, "margin": margin, "active_fraction": frac,
                             "n_active": int(round(frac * n))}
        out["workloads"][w.name] = entry
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "vmajor_tau.json")
    with open(path, "w") as fh:
        json.dump(out, fh, indent=1)
    print(path)


if __name__ == "__main__":
    main()
