"""Write tiny_oracle_digest.txt: SHA-256 digests of the oracle's results on
the tiny workload (16 tokens, d_model = d_ff = 256, 8 experts, top-4, seed 0).

Calls only the CPU oracle and the seeded input generator.  The digest guards
the oracle against unintended changes; it is regenerated only by a commit
whose message names the page passage (or its reading) that justifies the
change in the oracle's arithmetic.
"""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synthetic as syn  # noqa: E402


def main():
    wl = syn.WORKLOADS["tiny"]
    x = syn.activations(wl)
    lg = syn.logits(wl)
    gq, gs = oracle.quantize_experts(syn.w_gate_up(wl))
    dq, ds = oracle.quantize_experts(syn.w_down(wl))
    idx, _ = oracle.route(lg, wl.k)
    out = oracle.layer_forward(x, lg, wl.k, gq, gs, dq, ds)
    rows = [
        ("w_gu_codes", gq), ("w_gu_scales", gs), ("w_dn_codes", dq), ("w_dn_scales", ds),
        ("topk_idx", idx), ("out", out),
    ]
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_digest.txt")
    with open(path, "w") as f:
        f.write("# oracle results on the tiny workload (T=16, D=F=256, E=8, k=4, seed 0)\n")
        f.write("# written by tests/golden/make_golden.py\n")
        for name, arr in rows:
            f.write(f"{name} {hashlib.sha256(arr.tobytes()).hexdigest()}\n")


if __name__ == "__main__":
    main()
