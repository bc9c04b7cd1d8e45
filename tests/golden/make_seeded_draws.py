"""Writes seeded_draws.json: border shifts and Halo widths worked out from the
published SplitMix64 outputs, for pinning the oracle's seeded draws.

Derivation (no generator is run here; only the published outputs of
splitmix64.json and integer arithmetic are used):

* SplitMix64 seeded with state s returns, as its k-th output (k = 1, 2, ...),
  mix(s + k * gamma) mod 2^64, gamma = 0x9E3779B97F4A7C15 (Steele, Lea and
  Flood 2014; Vigna's reference splitmix64.c).  splitmix64.json holds the
  first three outputs for state 0.
* The library's reading of the pages' seed (border jitter and Halo widths are
  set by the seed: gpt-diffusion.com, "Como entra en tu pipeline", README
  notes) draws number stream * 2^32 + index of the sequence seeded with the
  seed: draw(seed, stream, index) = mix(seed + (stream * 2^32 + index + 1) *
  gamma).
* So with seed = -(stream * 2^32 + offset) * gamma mod 2^64, the draw of
  index offset + i is exactly published output i + 1 of state 0.
* Border shifts use stream 1, index 0 (rows) and 1 (columns): shift = draw mod
  w_e per axis, w_e = min(w, side), 0 when the window spans the axis.
* Halo widths use stream 2, index b * 2^20 + i for final window i of batch
  element b: width = draw mod (halo + 1).
"""
import json
import os

HERE = os.path.dirname(os.path.abspath(__file__))
GAMMA = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1


def seed_for(stream: int, offset: int) -> int:
    return (-(stream * (1 << 32) + offset) * GAMMA) & M64


def main():
    pub = json.load(open(os.path.join(HERE, "splitmix64.json")))
    assert pub["seed"] == 0
    out = [int(h, 16) for h in pub["outputs_hex"]]
    jitter = []
    for Hg, Wg, w in [(384, 128, 96), (256, 256, 72), (384, 128, 272)]:
        hy, wx = min(w, Hg), min(w, Wg)
        jitter.append({"Hg": Hg, "Wg": Wg, "w": w, "seed_hex": f"{seed_for(1, 0):016x}",
                       "sy": out[0] % hy if hy < Hg else 0,
                       "sx": out[1] % wx if wx < Wg else 0})
    halo = []
    for b in (0, 1):
        s = seed_for(2, b << 20)
        for h in (8, 4):
            halo.append({"b": b, "halo": h, "seed_hex": f"{s:016x}",
                         "windows": [0, 1, 2], "widths": [o % (h + 1) for o in out]})
    doc = {
        "source": "Worked out from the published SplitMix64 outputs of state 0 "
                  "(splitmix64.json) by the derivation in make_seeded_draws.py; the "
                  "draws are the library's reading of the pages' seed (gpt-diffusion.com "
                  "blog, 'Como entra en tu pipeline', README notes: the seed sets border "
                  "jitter and Halo widths).",
        "jitter": jitter,
        "halo": halo,
    }
    with open(os.path.join(HERE, "seeded_draws.json"), "w") as fh:
        json.dump(doc, fh, indent=1)
        fh.write("\n")


if __name__ == "__main__":
    main()
