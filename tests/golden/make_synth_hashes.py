"""Writes synth_sha256.json: SHA-256 of the generator's bf16 bytes for the small workload.

Pins the input generator's determinism (same seed -> same bytes on every machine).
Calls only the generator module; no method arithmetic is involved.
"""
import hashlib
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
import synth  # noqa: E402

if __name__ == "__main__":
    out = {}
    for name in ["mha4-L2048-B64"]:
        x = synth.make_inputs(synth.WORKLOADS[name])
        out[name] = {k: hashlib.sha256(x[k].tobytes()).hexdigest() for k in ("q", "k", "v")}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "synth_sha256.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
