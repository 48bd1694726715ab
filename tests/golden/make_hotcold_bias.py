"""Write tests/golden/hotcold_bias.json: the router bias of the hot/cold layer.

The expert-aware quantisation page ("Expert-aware quantisation: near-Q4 quality
at near-Q2 size?") profiles routing and finds it concentrated: per layer a Gini
coefficient of about 0.61, and the 32 most used of 256 experts take about half
of all routings; it keeps the 64 most used experts at high precision.  With no
trained model to profile, the hot/cold layer gets a seeded Zipf-like router
bias b[pi(r)] = -beta * ln(1 + r) (pi a seeded permutation of the experts),
with beta bisected so that the top-32 share on a seeded batch of 65,536 tokens
is 0.50.  The 64 experts with the highest counts (ties to the lower index) form
the hot set.  Counts come from the CPU oracle's router and top-k only.

Run:  python tests/golden/make_hotcold_bias.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import gen  # noqa: E402
import oracle  # noqa: E402

H, E, K_TOP, T_CAL, SEED = 2048, 256, 8, 65536, 0


def bias_for(beta, pi):
    b = np.zeros(E, np.float64)
    b[pi] = -beta * np.log1p(np.arange(E, dtype=np.float64))
    return b.astype(np.float32)


def stats(counts):
    c = np.sort(counts.astype(np.float64))[::-1]
    top32 = c[:32].sum() / c.sum()
    gini = np.abs(c[:, None] - c[None, :]).sum() / (2 * E * c.sum())
    return float(top32), float(gini)


def main():
    x = gen.normal_bf16_bits(SEED, gen.TID_X, 0, T_CAL * H).reshape(T_CAL, H)
    Wr = gen.normal_f32(SEED, gen.TID_ROUTER_W, 0, E * H, 0.02).reshape(E, H)
    pi = gen.permutation(SEED, gen.TID_PERM, E)
    logits0 = oracle.router(x, Wr, None)

    def share(beta):
        lg = (logits0 + bias_for(beta, pi)[None, :]).astype(np.float32)
        idx, _ = oracle.topk_softmax(lg, K_TOP)
        return stats(np.bincount(idx.ravel(), minlength=E))[0]

    lo, hi = 0.0, 4.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if share(mid) < 0.5:
            lo = mid
        else:
            hi = mid
    beta = 0.5 * (lo + hi)
    b = bias_for(beta, pi)
    idx, _ = oracle.topk_softmax(oracle.router(x, Wr, b), K_TOP)
    counts = np.bincount(idx.ravel(), minlength=E)
    top32, gini = stats(counts)
    hot = sorted(sorted(range(E), key=lambda e: (-int(counts[e]), e))[:64])
    out = {
        "source": __doc__.strip().splitlines()[0],
        "recipe": "b[pi(r)] = float32(-beta*ln(1+r)); pi = gen.permutation(seed 0, tid 4, 256); "
                  "calibration tokens x = gen tid 1 seed 0, [65536, 2048]; router W = gen tid 2 sigma 0.02",
        "beta": beta,
        "bias": [float(v) for v in b],
        "hot_experts": hot,
        "top32_share": top32,
        "gini": gini,
        "calibration_tokens": T_CAL,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "hotcold_bias.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(f"beta={beta:.6f} top32={top32:.4f} gini={gini:.4f} -> {path}")


if __name__ == "__main__":
    main()
