"""Writes tests/golden/codebook16.json: the 16-entry 4-bit codebook (standard-normal
quantiles normalised to [-1, 1], as fp32) computed by the oracle.  The codebook is an
input of the 4-bit kernels; this file lets the product path read it without importing
the oracle.  Run: python tests/golden/make_codebook.py"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import quant4_ref  # noqa: E402

if __name__ == "__main__":
    c = quant4_ref.codebook16()
    out = {"_source": "oracle/quant4_ref.codebook16(): q_i = Phi^-1((i + 0.5) / 16) / max|q|, rounded to fp32",
           "codebook_f32_hex": [float(x).hex() for x in c.astype("float64")],
           "codebook": [float(x) for x in c]}
    with open(os.path.join(HERE, "codebook16.json"), "w") as fh:
        json.dump(out, fh, indent=1)
    print("wrote", os.path.join(HERE, "codebook16.json"))
