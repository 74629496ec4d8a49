"""Write tests/golden/draft_noise.json: the noise level of the synthetic draft logits.

Synthetic draft logits are y = z + N(0, sigma^2) noise on target logits z ~ N(0, 1) over a
262144-token vocabulary.  The acceptance probability of a draft drawn from q is
alpha = sum_v min(p_v, q_v) (p = softmax z, q = softmax y).  The Gemma 4 MTP serving guide,
section 2, reports acceptance of about 47% at position 0 and 24% for both of the first two
drafts, i.e. a conditional 0.24 / 0.47 = 0.51 at position 1 (decaying exponentially with
depth, same section).  This script bisects sigma for alpha = 0.47 and alpha = 0.51 using
only the oracle's softmax, and stores both.

Run:  python tests/golden/tune_draft_noise.py
"""
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
from oracle.accept import softmax  # noqa: E402

V = 262144
ROWS = 8


def alpha(sigma, seed=0):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((ROWS, V))
    y = z + sigma * rng.standard_normal((ROWS, V))
    return float(np.minimum(softmax(z), softmax(y)).sum(axis=-1).mean())


def solve(target):
    lo, hi = 0.01, 5.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if alpha(mid) > target:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def main():
    s0, s1 = solve(0.47), solve(0.51)
    out = dict(vocab=V, target_logit_std=1.0,
               source="Gemma 4 MTP serving guide, section 2: position 0 ~47%, "
                      "both of the first two drafts ~24% (conditional 0.51)",
               sigma_pos0=s0, alpha_pos0=alpha(s0, seed=1),
               sigma_later=s1, alpha_later=alpha(s1, seed=1))
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "draft_noise.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
