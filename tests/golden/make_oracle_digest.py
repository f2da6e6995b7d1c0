"""Write tests/golden/oracle_tiny_digest.txt: the oracle's routing and a hash of
its output on the tiny seeded layer (H=512, I=1024, E=8, top-2, T=4, seed 0).

Run from the repository root: python tests/golden/make_oracle_digest.py
It calls only the oracle and the seeded input generator.
"""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from nvfp4_weight_only_route_b200 import synth  # noqa: E402
from oracle import oracle  # noqa: E402


def digest():
    shape = synth.SHAPES[0]
    layer = synth.make_layer(shape, 0)
    x = synth.make_x(shape, 0, 4)
    r = oracle.forward(layer, x, top_k=shape.k, intermediates=True)
    lines = [
        "# oracle output on the tiny seeded layer (H=512, I=1024, E=8, top-2, T=4, seed 0)",
        "# written by tests/golden/make_oracle_digest.py",
        "inputs " + " ".join(f"{k}={v}" for k, v in synth.layer_digest(layer).items()),
        "x " + hashlib.sha256(x.tobytes()).hexdigest()[:16],
        "ids " + " ".join(str(int(i)) for i in r["ids"].ravel()),
        "out_sha256 " + hashlib.sha256(r["out"].tobytes()).hexdigest(),
        "a_sha256 " + hashlib.sha256(r["a"].tobytes()).hexdigest(),
    ]
    return "\n".join(lines) + "\n"


if __name__ == "__main__":
    path = os.path.join(ROOT, "tests", "golden", "oracle_tiny_digest.txt")
    open(path, "w").write(digest())
    print(open(path).read())
