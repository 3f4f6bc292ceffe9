"""Write the stored expected values under tests/golden/ (calls only the oracle and synth).

    python tests/golden/make_golden.py

int8_div.json: the Int8 divisor K of the 8192x8192 Laplace workload (scale = absmax(row) / K)
that puts the symbol entropy at 2.00 bits, found by bisection with the oracle's quantiser, and
rounded to 4 decimals (the constant synth.INT8_DIV_LAPLACE_8K must equal it).
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import synth  # noqa: E402


def main():
    w = synth.WORKLOADS["int8_8k"].tensors[0].generate()
    k = round(oracle.int8_div_for_entropy(w, 2.0, lo=2.0, hi=8.0, iters=30), 4)
    s, _ = oracle.quantize(w, oracle.INT8, k)
    rec = {"workload": "int8_8k", "int8_div": k, "entropy_bits": oracle.entropy_bits(s),
           "cite": "Int8 8192x8192 Laplace workload: per-row scales chosen so the symbol entropy is about 2.0 bits"}
    with open(os.path.join(HERE, "int8_div.json"), "w") as f:
        json.dump(rec, f, indent=1)
    print(rec)


if __name__ == "__main__":
    main()
