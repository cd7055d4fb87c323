"""Writes tests/golden/traces.txt from the CPU oracle (and nothing else).

Single-element trajectories with lr=1e-3, beta=(0.9, 0.999), eps=1e-8 from
zero state, recorded as the fp32 bit pattern of the parameter after each
step.  They are regression fixtures of the oracle's documented operation
order; the first seven rows also agree bit for bit with a hand computation
in that order made before the oracle was written, and the p0=0 case at step
1 is fixed independently by the step-one closed form (-lr exactly).

Run:  python -m tests.golden.make_golden
"""
import os

import numpy as np

CASES = {
    # name: (algo, p0, grads, wd, beta3, alpha)
    "adam_g0.5": ("adam", 1.0, [0.5, 0.5, 0.5], 0.0, 0.0, 0.0),
    "adamw_wd0.01_g0.5": ("adam", 1.0, [0.5, 0.5], 0.01, 0.0, 0.0),
    "ademamix_b3_0.9999_a5_g0.5": ("ademamix", 1.0, [0.5, 0.5], 0.0, 0.9999, 5.0),
    "adam_p0_g+1-1": ("adam", 0.0, [1.0, -1.0], 0.0, 0.0, 0.0),
}


def run_trace(case):
    import oracle
    algo, p0, grads, wd, b3, alpha = CASES[case]
    p = np.array([p0], np.float32)
    s1 = np.zeros(2 if algo == "ademamix" else 1, np.float32)
    s2 = np.zeros(1, np.float32)
    out = []
    for t, g in enumerate(grads, 1):
        oracle.step_f32(p, np.array([g], np.float32), s1, s2, dtype="f32",
                        algo=algo, step=t, lr=1e-3, beta1=0.9, beta2=0.999,
                        eps=1e-8, beta3=b3, alpha=alpha, weight_decay=wd)
        out.append("0x%08x" % int(p.view(np.uint32)[0]))
    return out


def main():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "traces.txt")
    with open(path, "w") as f:
        f.write("# case step param_bits -- written by tests/golden/make_golden.py\n")
        for case in CASES:
            for t, h in enumerate(run_trace(case), 1):
                f.write(f"{case} {t} {h}\n")


if __name__ == "__main__":
    main()
