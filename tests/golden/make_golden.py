"""Write the oracle-derived regression fixtures in this folder.

Calls only ``oracle/`` and the seeded input generator; run from the repo root:
    python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import qlora_inputs as qi  # noqa: E402
from oracle import nf4  # noqa: E402


def main():
    cb = nf4.nf4_codebook()
    with open(os.path.join(HERE, "nf4_codebook_f32.txt"), "w") as fh:
        fh.write("# NF4 levels as fp32 bit patterns (hex) and decimal, ascending; from oracle.nf4\n")
        for v in cb:
            fh.write(f"{int(np.float32(v).view(np.uint32)):08x} {float(v):.9g}\n")
    W = qi.make_linear(qi.SMALL)["W"].numpy()
    q = nf4.quantize_nf4(W)
    with open(os.path.join(HERE, "small_quant_digest.json"), "w") as fh:
        json.dump({"case": qi.SMALL.name,
                   "codes_sha256": hashlib.sha256(q["codes"].tobytes()).hexdigest(),
                   "absmax_q": q["absmax_q"].tolist(),
                   "group_scale_hex": [float(x).hex() for x in q["group_scale"]]}, fh, indent=1)


if __name__ == "__main__":
    main()
