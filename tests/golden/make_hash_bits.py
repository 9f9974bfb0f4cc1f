"""Write hash_bits.json: worked examples of the codec's random signs (the
randomized Hadamard transform's sign vector) and dither uniforms, derived step
by step from their definition below, using only the oracle's SplitMix64
output function mix64 -- itself pinned to the published SplitMix64 outputs in
splitmix64.json.

  H(seed, tag, a, b) = mix64(mix64(mix64(seed + gamma (tag + 1)) ^ a) ^ b)
  sign s_j[i]       = -1 iff bit (i mod 64) of H(seed, 1, j, floor(i / 64)) is 1
  uniform r(t, i)   = bits 16 (i mod 4) .. 16 (i mod 4) + 15 of H(seed, 2, t, floor(i / 4)), times 2^-16

The composition and the bit positions are restated here, independently of
the oracle's own hqo_hash / hqo_sign / hqo_uniform.

    python tests/golden/make_hash_bits.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402

GAMMA = 0x9E3779B97F4A7C15
MASK = (1 << 64) - 1


def H(seed, tag, a, b):
    key = oracle.mix64((seed + GAMMA * (tag + 1)) & MASK)
    return oracle.mix64(oracle.mix64(key ^ a) ^ b), key


def main():
    out = {"source": "H(seed, tag, a, b) = mix64(mix64(mix64(seed + gamma (tag + 1)) ^ a) ^ b); sign s_j[i] = -1 "
                     "iff bit i mod 64 of H(seed, 1, j, i div 64); uniform r(t, i) = bits 16 (i mod 4) .. +15 of "
                     "H(seed, 2, t, i div 4) times 2^-16; mix64 = SplitMix64 output function (Steele, Lea & Flood "
                     "2014), pinned by splitmix64.json",
           "signs": [], "uniforms": []}
    for seed, j, n in ((0, 0, 256), (42, 1, 256), (42, 7, 128), ((1 << 63) + 5, 3, 1024)):
        words, steps = [], []
        for b in range((n + 63) // 64):
            h, key = H(seed, 1, j, b)
            words.append(h)
            steps.append({"b": b, "key": f"{key:#018x}", "H": f"{h:#018x}"})
        s = "".join("-" if (words[i // 64] >> (i % 64)) & 1 else "+" for i in range(n))
        out["signs"].append({"seed": seed, "j": j, "n": n, "hash_words": steps, "signs": s})
    for seed, t, count in ((0, 0, 16), (42, 5, 32), (7, 123456789, 16)):
        vals, steps = [], []
        for i in range(count):
            h, key = H(seed, 2, t, i // 4)
            if i % 4 == 0:
                steps.append({"m": i // 4, "key": f"{key:#018x}", "H": f"{h:#018x}"})
            vals.append((h >> (16 * (i % 4))) & 0xFFFF)
        out["uniforms"].append({"seed": seed, "t": t, "hash_words": steps, "r_times_2^16": vals})
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "hash_bits.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
