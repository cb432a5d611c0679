"""Reader for the hand-worked golden fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_hand_example(name):
    blocks, cur, meta = {}, None, {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head = line.split()
            if head[0] == "bits":
                meta["bits"] = int(head[1])
                continue
            if len(head) == 1 and head[0].isalpha():
                cur = head[0]
                blocks[cur] = []
                continue
            blocks[cur].append(head)
    out = {"bits": meta["bits"]}
    out["W"] = np.array([[float(v) for v in r] for r in blocks["W"]], dtype=np.float64)
    out["scale"] = np.array([float(v) for v in blocks["scale"][0]], dtype=np.float64)
    out["q"] = np.array([[int(v) for v in r] for r in blocks["q"]], dtype=np.int64)
    out["packed"] = np.array([[int(v, 16) for v in r] for r in blocks["packed"]], dtype=np.uint8)
    out["X"] = np.array([[float(v) for v in r] for r in blocks["X"]], dtype=np.float64)
    out["Y"] = np.array([[float(v) for v in r] for r in blocks["Y"]], dtype=np.float64)
    return out
