"""Write the router bias of the skewed-routing workload.

The skewed Nano workload (hidden 1024, 64 experts, top-2, T=16384) asks for a
router bias under which expert popularity follows Zipf(s=1.2): expert e (rank
e+1) should receive a share p_e = (e+1)^-s / sum_r r^-s of the T*K routing
slots.  The bias is an *input* of that workload; this script derives it with
the oracle's own router and selection (the bias only changes the selection
key s + bias, never the routing weights).

Procedure: draw a seeded calibration batch (same distributions as the
workload: x bf16 N(0,1), router W N(0, 0.02^2)), compute the sigmoid scores
once with the oracle, then repeat for a fixed number of iterations
    load_e = number of slots the oracle's top-K selection gives expert e
    bias_e += eta * (ln target_e - ln max(load_e, 0.5))
with target_e = T*K*p_e.  The final bias is written with 9 significant
digits to ``workloads/data/zipf_bias_e64_s1.2.txt`` together with the loads it
achieves on the calibration batch.

Run: ``python -m oracle.calibrate_zipf_bias`` (about a minute, single core).
"""
from __future__ import annotations

import os
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
import workloads  # noqa: E402

ZIPF_S = 1.2
CALIB_T = 16384
ITERS = 300
ETA = 0.02


def zipf_targets(E: int, slots: int, s: float = ZIPF_S) -> np.ndarray:
    p = np.arange(1, E + 1, dtype=np.float64) ** (-s)
    return slots * p / p.sum()


def main() -> None:
    wl = workloads.WORKLOADS["nano_zipf_t16384"]
    shape = wl.shape
    E, K = shape.E, shape.K
    layer = workloads.make_layer(shape, wl.wid, 0, device="cpu", bias_mode="zero", experts=[])
    x = workloads.make_x(shape, CALIB_T, wl.wid, batch=999, device="cpu")
    r = oracle.route(x, layer["router_w"], layer["router_bias"], K, shape.routed_scaling)
    scores = r["scores"]
    target = zipf_targets(E, CALIB_T * K)
    bias = np.zeros(E, np.float32)
    for _ in range(ITERS):
        idx, _m = oracle.select_topk(scores, bias, K)
        load = np.bincount(idx.reshape(-1), minlength=E).astype(np.float64)
        bias = (bias + ETA * (np.log(target) - np.log(np.maximum(load, 0.5)))).astype(np.float32)
    idx, _m = oracle.select_topk(scores, bias, K)
    load = np.bincount(idx.reshape(-1), minlength=E)
    path = workloads.zipf_bias_path(E, ZIPF_S)
    os.makedirs(os.path.dirname(path), exist_ok=True)
    with open(path, "w") as f:
        f.write(f"# router bias for Zipf(s={ZIPF_S}) expert popularity, E={E}, K={K}\n")
        f.write(f"# written by oracle/calibrate_zipf_bias.py: {ITERS} iterations, eta={ETA}, "
                f"calibration batch T={CALIB_T}\n")
        f.write("# columns: bias  (comment: achieved load on the calibration batch / Zipf target)\n")
        for e in range(E):
            f.write(f"{float(bias[e]):.9g}  # {int(load[e])} / {target[e]:.1f}\n")
    print(f"wrote {path}; hottest {load.max()}, coldest {load.min()}")


if __name__ == "__main__":
    main()
