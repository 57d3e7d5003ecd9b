"""Write the oracle's outputs on the tiny fp32 workload as a text fixture.

Calls only the oracle and the seeded input generator.  The fixture guards the
oracle against silent drift: any later change of its arithmetic must either
reproduce these numbers or rewrite them with this script, with the reason.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from kv_cache_attention_qkv_b200 import workloads  # noqa: E402


def main():
    inp = workloads.generate("tiny_fp32")
    res = oracle.flashcache_step(inp.x, inp.w_qkv, inp.q_pos, inp.cu_seqlens_q, inp.cu_seqlens_k,
                                 inp.k_cache, inp.v_cache, inp.n_heads, inp.head_dim,
                                 inp.rope_theta, "fp32")
    tracked = oracle.topk_tracked(res["importance"], inp.cu_seqlens_k, inp.cand_lo, inp.cand_hi,
                                  inp.topk, int(inp.topk.max()))
    pos = inp.q_pos
    doc = {
        "what": "oracle outputs of one Flash-Cache step on workload tiny_fp32 (seed 0)",
        "source": "tests/golden/make_golden.py (calls oracle/ only)",
        "q_pos": pos.tolist(),
        "out": res["out"].reshape(-1).tolist(),
        "k_rows_written": res["k_cache"][pos].reshape(-1).tolist(),
        "v_rows_written": res["v_cache"][pos].reshape(-1).tolist(),
        "importance": res["importance"].tolist(),
        "tracked": tracked.reshape(-1).tolist(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_fp32_step.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=0)
        f.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
