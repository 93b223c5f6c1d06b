"""Write ``oracle_digests.json``: SHA-256 digests of the seeded fp16 inputs and
of the oracle's outputs for the small workloads.

The pages print no numeric worked example for the GEMM + ReLU, so the stored
values here are the oracle's own (after it passed its pins), kept to detect
any later drift in the input recipe or the oracle across machines.  This
script calls only ``oracle/`` and the input generator.

    python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from tiled_tensor_core_05_b200 import workloads  # noqa: E402

NAMES = ("cube256", "ragged1000", "cube1024")


def sha(x) -> str:
    if hasattr(x, "numpy"):
        x = x.contiguous().view(dtype=__import__("torch").int16).numpy()
    return hashlib.sha256(np.ascontiguousarray(x).tobytes()).hexdigest()


def digests(name):
    a, b = workloads.workload_inputs(name)
    out = {"a": sha(a), "b": sha(b)}
    out["relu"] = sha(oracle.gemm_relu(a, b).view(np.uint16))
    out["plain"] = sha(oracle.gemm(a, b).view(np.uint16))
    return out


def main():
    data = {n: digests(n) for n in NAMES}
    with open(os.path.join(HERE, "oracle_digests.json"), "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")
    print(json.dumps(data, indent=1))


if __name__ == "__main__":
    main()
