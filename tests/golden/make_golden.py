"""Write tests/golden/oracle_digests.json from the oracle alone.

Records, for the small weight sets, the SHA-256 of each generated input and of
each part of the oracle's container (stream, gaps, offsets, sign|fraction
bytes, lengths). tests/test_synth.py checks the input digests on the CPU;
test_encode_matches_stored_oracle_digests (tests/test_gpu_parity.py) checks
every part of the CUDA encoder's container against them. Run from the
repository root:

    python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from lossless_bf16_weight_huffman_b200 import synth  # noqa: E402


def sha(a) -> str:
    return hashlib.sha256(memoryview(a).cast("B")).hexdigest()


def main():
    out = {"about": "written by tests/golden/make_golden.py from the oracle only", "tensors": []}
    picks = [("single_1024x4096", 0), ("llama_layer", 1), ("llama_layer", 7), ("heavy_tail_64m", 0)]
    picks += [("mixed_2000", i) for i in (0, 1, 2, 3, 4, 5)]
    for set_name, idx in picks:
        spec = synth.weight_set(set_name)[idx]
        w = synth.generate(spec)
        for max_len in (32, 12):
            if max_len == 12 and set_name != "heavy_tail_64m":
                continue
            enc = oracle.encode(w, max_len=max_len, chunk_bytes=32, threads_per_block=256)
            out["tensors"].append({
                "set": set_name, "index": idx, "name": spec.name, "n": int(w.size), "max_len": max_len,
                "chunk_bytes": 32, "threads_per_block": 256,
                "input_sha256": sha(w), "total_bits": int(enc.total_bits),
                "container_bytes": int(enc.container_bytes),
                "lengths_sha256": sha(enc.lengths), "stream_sha256": sha(enc.stream),
                "gaps_sha256": sha(enc.gaps), "offsets_sha256": sha(enc.offsets), "sm_sha256": sha(enc.sm),
            })
            print(set_name, idx, max_len, enc.total_bits, flush=True)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_digests.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
