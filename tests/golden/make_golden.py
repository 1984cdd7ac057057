"""Writes tiny_oracle.json: the fp64 oracle's loss and gradients on the tiny
workload (seeded synthetic inputs).  Calls only the oracle and the seeded
input generator; rerun it only when the oracle's arithmetic changes."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from rnn_joint_network_02_b200 import synth  # noqa: E402


def main():
    batch = synth.workload("tiny")
    f, g, W_f, W_g, W_o, b_o = (t.numpy() for t in batch.float64())
    res = oracle.fwd_bwd(f, g, W_f, W_g, W_o, b_o, batch.labels.numpy(), batch.T_len.numpy(),
                         batch.U_len.numpy())
    out = {"workload": "tiny", "seed": 1000, "status": res.status,
           "loss": res.loss.tolist()}
    for name in ("df", "dg", "dW_f", "dW_g", "dW_o", "db_o"):
        out[name] = getattr(res, name).reshape(-1).tolist()
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as fh:
        json.dump(out, fh)


if __name__ == "__main__":
    main()
