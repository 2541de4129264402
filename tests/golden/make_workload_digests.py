"""Writes tests/golden/workload_digests.json: the SHA-256 of every synthetic input
buffer the benchmark and the full-size parity tests use.  It calls only the seeded
generators in workloads.py (no selection arithmetic, nothing from the CUDA path).

Run from the repository root: ``python tests/golden/make_workload_digests.py``.
``tests/test_workload_digests.py`` regenerates the buffers and compares, so a
change to a generator, a seed or numpy's PCG64 stream shows up as a failure.
"""
import hashlib
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

OUT = os.path.join(HERE, "workload_digests.json")


def cases():
    """(name, thunk returning a dict of named numpy buffers) for every workload."""
    yield "pr1_duplicates", lambda: {"x": W.pr1_duplicates().x}
    yield "indexer_drift", lambda: {"x": W.indexer_drift().x}

    def varlen():
        w = W.indexer_varlen()
        return {"x": w.x, "end": w.end}
    yield "indexer_varlen", varlen
    for b in (1, 8, 64, 256):
        def sampler(b=b):
            w = W.sampler_logits(b, 1024)     # k does not change the buffers
            out = {"x": w.x, "uniforms": W.uniforms(b)}
            if w.end is not None:
                out["end"] = w.end
            return out
        yield f"sampler_logits_{b}", sampler
    for rows, n in ((1, 1 << 28), (16, 1 << 24)):
        for variant in ("uniform", "desc", "equal"):
            yield f"long_rows_{rows}x{n}_{variant}", (lambda rows=rows, n=n, variant=variant:
                                                      {"x": W.long_rows(rows, n, 4096, variant).x})

        def nan(rows=rows, n=n):
            w = W.long_rows(rows, n, 1000, "uniform", inject_nan=True)
            return {"x": w.x, "nan_rows": w.nan_rows}
        yield f"long_rows_{rows}x{n}_uniform_nan", nan


def digest(buffers):
    return {name: {"sha256": hashlib.sha256(b.tobytes()).hexdigest(), "dtype": str(b.dtype),
                   "shape": list(b.shape)} for name, b in buffers.items()}


def main():
    out = {name: digest(thunk()) for name, thunk in cases()}
    with open(OUT, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
        f.write("\n")
    print(OUT)


if __name__ == "__main__":
    main()
