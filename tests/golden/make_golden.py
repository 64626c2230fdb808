"""Write the oracle's kv lists for the tiny workload (regression fixture).

The pages print no worked example, so this fixture is the oracle's own output
on seeded CPU inputs; it guards the oracle against unintended change. It calls
only oracle/ and the seeded input generator.
Usage: python tests/golden/make_golden.py
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from block_sparse_attention_softmax_b200.workloads import WORKLOADS, make_inputs  # noqa: E402


def main():
    wl = WORKLOADS["tiny"]
    x = make_inputs(wl, "cpu")
    lines = ["# hybrid Top-k(10%) + Top-p(0.9) block mask of the 'tiny' workload",
             "# (B=1 H=2 N=1024 d=64, 64x64 blocks), seeded CPU inputs.",
             "# Follows SpargeAttention2 §2(1) and SLA2 提案手法 ①; written by make_golden.py.",
             "# head:row:kv_cnt:kv_idx..."]
    for h in range(wl.H):
        out = oracle.build_mask(oracle.as_f64(x["q"][0, h]), oracle.as_f64(x["k"][0, h]),
                                wl.bq, wl.bk, wl.topk, wl.topp)
        idx, cnt = oracle.kv_lists(out["mask"])
        for r in range(idx.shape[0]):
            lines.append(f"{h}:{r}:{cnt[r]}:" + " ".join(str(t) for t in idx[r, :cnt[r]]))
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_kv_lists.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
