"""Write the stored expected values for the 16-token "tiny" workload.

Calls only the CPU oracle and the seeded input generators; nothing here comes
from the CUDA path.  Re-run after a justified change to the oracle:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import workloads as wl  # noqa: E402


def tiny_expectations():
    cfg = wl.config("tiny")
    x = wl.activations_bf16(cfg)
    ids = oracle.mask_padding(wl.routing(cfg), cfg.real)
    idx = oracle.create_indices(ids, cfg.E)
    recv, counts = oracle.dispatch_mxfp4(x, cfg.top_k, cfg.E, idx)
    R = int(idx["expert_start_indices"][-1])
    wq, sfw, gw = oracle.quantize_weights_nvfp4(wl.all_expert_weights_f32(cfg))
    xq, sfa = oracle.nvfp4_quantize_bf16(x, 1.0)
    rng = np.random.default_rng(0)
    samples = [[int(m), int(j), int(n)] for m, j, n in zip(rng.integers(0, cfg.real, 24),
                                                           rng.integers(0, cfg.top_k, 24),
                                                           rng.integers(0, cfg.N_out, 24))]
    y16 = oracle.gemv_elements("w4a16", ids, wq, sfw, gw, samples, act_bf16=x)
    y4 = oracle.gemv_elements("w4a4", ids, wq, sfw, gw, samples, xq=xq, sfa=sfa)
    return {
        "workload": "tiny: N=16 (13 real), K=256, E=8, top_k=2, N_out=256, seed 101",
        "masked_topk_ids": ids.tolist(),
        "token_expert_order": idx["token_expert_order"].tolist(),
        "expert_start_indices": idx["expert_start_indices"].tolist(),
        "restore_token_order": idx["restore_token_order"].tolist(),
        "expert_ids": idx["expert_ids"].tolist(),
        "expert_usage_stats": idx["expert_usage_stats"].tolist(),
        "recv_counts": counts.tolist(),
        "recv_rows_sha256": __import__("hashlib").sha256(recv[:R].tobytes()).hexdigest(),
        "w_global": [float(v) for v in gw],
        "gemv_samples": samples,
        "gemv_w4a16": [float(v) for v in y16],
        "gemv_w4a4": [float(v) for v in y4],
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_pipeline.json"), "w") as f:
        json.dump(tiny_expectations(), f, indent=1)
        f.write("\n")
