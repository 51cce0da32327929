"""Write tests/golden/oracle_digests.json: SHA-256 digests of the oracle's blobs and decodes.

The pages print no numeric results for their usage example ("EntroPack lattice compression",
section "Usage"), so these fixtures come from the oracle alone: this script calls only oracle/
(and the seeded inputs of cases.py). They pin the exact bytes of the format and of its decodes,
so a change that moved the oracle, the encoders and the kernel together still shows. Run from
the repository root:  python tests/golden/make_golden.py
"""
from __future__ import annotations

import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path[:0] = [ROOT, HERE]

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import workloads as W  # noqa: E402
from cases import CASES, matrix  # noqa: E402


def sha(a) -> str:
    return hashlib.sha256(bytes(a) if isinstance(a, (bytes, bytearray)) else np.ascontiguousarray(a).tobytes()).hexdigest()


def main() -> None:
    out = {"source": "written by tests/golden/make_golden.py from oracle/ only; the pages print no numeric "
                     "results for their usage example (EntroPack lattice compression, section Usage)",
           "cases": {}}
    for name, (what, pb, rate, dtypes) in CASES.items():
        m = matrix(name)
        blob = oracle.compress(m.bits, m.dtype, rate, prob_bits=pb)
        info = oracle.blob_info(blob)
        entry = {"what": what, "prob_bits": pb, "target_bpp": rate, "rows": int(m.bits.shape[0]),
                 "cols": int(m.bits.shape[1]), "dtype": W.DTYPE_NAME[m.dtype], "blob_bytes": len(blob),
                 "blob_sha256": sha(blob), "steps_per_tile": int(info["S"]), "n_tiles": int(info["n_tiles"]),
                 "decoded_sha256": {W.DTYPE_NAME[dt]: sha(oracle.decompress(blob, dt)) for dt in dtypes}}
        pay, sig = oracle.decompress_rowscaled(blob)
        entry["rowscaled_payload_sha256"] = sha(pay)
        entry["rowscaled_sigma_sha256"] = sha(np.asarray(sig, np.float32))
        out["cases"][name] = entry
    path = os.path.join(HERE, "oracle_digests.json")
    with open(path, "w") as fh:
        json.dump(out, fh, indent=1)
        fh.write("\n")
    print(path)


if __name__ == "__main__":
    main()
