"""Write tests/golden/oracle_digests.json: SHA-256 digests of the oracle's
outputs on small seeded cases of every mode, both 16-bit formats and several
partial counts, and of the bf16 output of hc_mix on a few shapes.  Calls only oracle/ (and the seeded input generator).  Run it
again, and say why in the commit, only when the oracle's arithmetic is meant
to change; tests/test_oracle_digests.py checks the stored digests.

    python tests/golden/make_oracle_digests.py
"""
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

CASES = [  # (mode, M, H, P, residual, io)
    (0, 5, 256, 1, True, 0), (1, 4, 512, 2, True, 0), (2, 6, 224, 4, True, 0),
    (2, 3, 96, 3, False, 0), (0, 7, 64, 8, True, 0), (1, 2, 1024, 1, False, 0),
    (0, 4, 128, 2, True, 1), (1, 3, 256, 1, True, 1), (2, 5, 160, 4, False, 1),
]
HC_CASES = [(1, 4, 64, 8), (3, 4, 128, 16), (16, 4, 32, 64)]  # (M, hc, C, r); bf16 u


def digests():
    import torch

    import oracle
    from mxfp4_quantization_b200 import synth
    out = {}
    for mode, M, H, P, res, io in CASES:
        wl = synth.RowWorkload("digest", M=M, H=H, P=P, mode=mode, eps=1e-6, seed=M * H + P,
                               residual=res, outlier_frac=0.02, channel_decades=1.0 if P > 1 else 0.0,
                               dtype=torch.float16 if io else torch.bfloat16)
        inp = wl.inputs(device="cpu")
        parts = [synth.to_bits(p) for p in inp["parts"]]
        r = synth.to_bits(inp["residual"]) if res else None
        o = oracle.rmsnorm_quant(parts, r, synth.to_bits(inp["weight"]), wl.eps, mode, io=io)
        h = hashlib.sha256()
        for k in ("q", "scale", "residual_out", "y"):
            h.update(o[k].tobytes())
        out[f"mode{mode}_M{M}_H{H}_P{P}_{'res' if res else 'nores'}_{'fp16' if io else 'bf16'}"] = h.hexdigest()
    for M, hc, C, r in HC_CASES:
        wl = synth.HCWorkload("digest", M=M, hc=hc, C=C, r=r, seed=M + C + r)
        inp = wl.inputs(device="cpu")
        _, ub = oracle.hc_mix(synth.to_bits(inp["x"]), synth.to_bits(inp["w_down"]),
                              synth.to_bits(inp["w_up"]), hc, C, r)
        out[f"hc_mix_M{M}_hc{hc}_C{C}_r{r}"] = hashlib.sha256(ub.tobytes()).hexdigest()
    return out


if __name__ == "__main__":
    path = os.path.join(HERE, "oracle_digests.json")
    with open(path, "w") as fh:
        json.dump({"about": "SHA-256 of the oracle's (q, scale, residual_out, y) on seeded cases, "
                            "and of hc_mix's bf16 output; written by "
                            "tests/golden/make_oracle_digests.py", "cases": digests()},
                  fh, indent=1)
    print(path)
