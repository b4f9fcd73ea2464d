"""Write full-size float64 oracle values for the large FLCE workloads.

Calls only `oracle/` (and the seeded input generators).  For each workload it
stores every row's logsumexp and label logit, the loss and the token counts,
so the GPU parity tests can compare all rows at full size and take sampled
dHidden / dWeight rows from the oracle's own lse.

    python tests/golden/make_oracle_fullsize.py [name ...]
"""
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import flce_inputs as fi  # noqa: E402
import oracle  # noqa: E402

NAMES = ["v32k_mean", "v131k_zipf", "v256k_softcap", "microbatch"]


def path_for(name: str) -> str:
    return os.path.join(HERE, f"oracle_{name}.npz")


def main(names):
    for name in names:
        t = time.time()
        w = fi.WORKLOADS[name]
        inp = fi.make_inputs(w)
        h, W, y = inp.hidden, inp.weight, inp.labels
        f = oracle.forward(h, W, y, fi.IGNORE_INDEX, w.softcap, w.reduction, chunk=256)
        extra = {}
        if w.microbatches > 1:
            losses, counts = [], []
            for sl in inp.microbatch_slices():
                valid = y[sl] != fi.IGNORE_INDEX
                losses.append(float(f["row_loss"][sl].sum()))
                counts.append(int(valid.sum()))
            extra = dict(mb_loss=np.array(losses), mb_count=np.array(counts))
        np.savez_compressed(path_for(name), lse=f["lse"], label_logit=f["label_logit"],
                            loss=np.float64(f["loss"]), num_tokens=np.int64(f["num_tokens"]),
                            num_valid=np.int64(f["num_valid"]), **extra)
        print(f"{name}: loss={f['loss']:.10g} n={f['num_valid']} ({time.time() - t:.1f}s)",
              flush=True)


if __name__ == "__main__":
    main(sys.argv[1:] or NAMES)
