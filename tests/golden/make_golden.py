"""Write tests/golden/tiny_f32_L256.json from the CPU oracle alone.

The pages print no worked numeric example of the layer, so the only stored
values are the oracle's own, on the seeded tiny fp32 workload (batch 1,
L=256, 2 heads, P=N=16, checkpoint stride 64).  They guard the oracle
against unintended drift; its correctness rests on the pins in
tests/oracle_pins.py.  Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import ssd_synth  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_f32_L256.json")
TIMES = [0, 1, 2, 3, 63, 64, 127, 200, 255]


def compute():
    wl = ssd_synth.WORKLOADS[0]
    prm = ssd_synth.make_params(wl)
    u = ssd_synth.make_u(wl).numpy()
    dt = ssd_synth.make_dt(wl, prm["dt_bias"]).numpy()
    out = oracle.layer(u, prm["w"].numpy(), dt, prm["A"].numpy(), prm["D"].numpy(),
                       prm["bias"].numpy(), None, None, H=wl.H, P=wl.P, N=wl.N, G=wl.G,
                       s=wl.s, io_round="f32")
    return wl, out


def main():
    wl, out = compute()
    doc = {
        "workload": wl.name,
        "source": "oracle/ssd_oracle.c via tests/golden/make_golden.py (no page prints a worked example)",
        "times": TIMES,
        "y_at_times": out["y"][0, TIMES].tolist(),
        "h_final": out["h_final"][0].tolist(),
        "h_ckpt_fro": [float(np.linalg.norm(out["h_ckpt"][0, k])) for k in range(out["h_ckpt"].shape[1])],
        "v_sum": float(out["v"].astype(np.float64).sum()),
        "tail_out": out["tail_out"][0].tolist(),
    }
    with open(OUT, "w") as f:
        json.dump(doc, f, indent=0)
    print("wrote", OUT)


if __name__ == "__main__":
    main()
