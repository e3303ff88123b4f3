"""Writes sphere_codebooks_b7_b8.json: the oracle's Lloyd-Max codebooks of the sphere-coordinate marginal
(oracle.tq_oracle.sphere_codebook) at 7 and 8 bits for d = 64, 128 and 256.  Their plain fixed-point iteration
takes minutes per codebook, so the tests read these stored levels; the file is written by the oracle alone
(python tests/golden/make_sphere_codebooks.py), and a test recomputes one of them to tie it to the oracle."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import tq_oracle as o  # noqa: E402


def main():
    out = {"source": "oracle.tq_oracle.sphere_codebook(d, bits), fp64 levels as float.hex", "codebooks": {}}
    for d in (64, 128, 256):
        for bits in (7, 8):
            c = o.sphere_codebook(d, bits)
            out["codebooks"][f"{d}/{bits}"] = [float(v).hex() for v in c]
            print(d, bits, flush=True)
    with open(os.path.join(HERE, "sphere_codebooks_b7_b8.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
