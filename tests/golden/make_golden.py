"""Write the stored expected values of the full-size workloads.

    python tests/golden/make_golden.py [llama7b-8k llama7b-16k varlen-10k llama13b-32k]

Calls only the CPU oracle (``oracle/``) and the seeded input generators
(``contextual_token_sparsity_b200.synth``); nothing here touches the GPU
path.  For every layer of each workload it stores the oracle's token-block
scores (float64 as decimal strings of full precision), the keep-ratio
threshold derived from them, and sha256 digests of the generated input bytes
so a test can confirm it regenerated exactly the same inputs.
"""

import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from contextual_token_sparsity_b200 import synth  # noqa: E402


def golden_for(key: str) -> dict:
    w = synth.WORKLOADS[key]
    out = {"workload": key, "name": w.name, "lengths": list(w.lengths), "H": w.H, "dh": w.dh,
           "block": w.block, "d": w.d, "layers": []}
    for layer in range(w.layers):
        t0 = time.time()
        inp = synth.make_workload(key, layer, with_x=True)
        M = oracle.score_blocks(inp["q"], inp["k"], inp["cu_seqlens"], w.H, w.dh, w.block)
        sc = oracle.column_scores(M)
        theta = oracle.threshold_for_keep_ratio(sc, w.keep[layer])
        rec = {
            "layer": layer,
            "seed": int(w.seeds[layer]),
            "keep_ratio": w.keep[layer],
            "digest_qk": synth.digest(inp["q"], inp["k"], inp["cu_seqlens"]),
            "digest_x": synth.digest(inp["x"], inp["y_out"]),
            "scores": [repr(float(v)) for v in sc],
            "theta": repr(float(theta)),
            "kept_blocks": int(oracle.keep_mask(sc, theta).sum()),
        }
        if w.predictor_rank:
            cu = inp["cu_seqlens"]
            reps = oracle.block_representatives(inp["x"], cu, w.block)
            qh = oracle.predictor_embeddings(reps, inp["w1q"], inp["w2q"])
            kh = oracle.predictor_embeddings(reps, inp["w1k"], inp["w2k"])
            _, ps = oracle.predict_scores(qh, kh, cu, w.block, w.H, w.dh)
            ptheta = oracle.threshold_for_keep_ratio(ps, w.keep[layer])
            rec["digest_pred"] = synth.digest(inp["w1q"], inp["w2q"], inp["w1k"], inp["w2k"])
            rec["pred_scores"] = [repr(float(v)) for v in ps]
            rec["pred_theta"] = repr(float(ptheta))
            rec["recall"] = oracle.recall(oracle.keep_mask(ps, ptheta),
                                          oracle.keep_mask(sc, theta))
        rec["oracle_seconds"] = round(time.time() - t0, 1)
        out["layers"].append(rec)
        print(f"{key} layer {layer}: {rec['oracle_seconds']} s", flush=True)
    return out


def main(keys):
    for key in keys:
        g = golden_for(key)
        with open(os.path.join(HERE, f"{key}.json"), "w") as f:
            json.dump(g, f, indent=1)
            f.write("\n")


if __name__ == "__main__":
    main(sys.argv[1:] or ["llama7b-8k", "varlen-10k", "llama7b-16k", "llama13b-32k"])
