"""Reader for the small `key: value ...` fixtures under tests/golden/ (comments start with #)."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read(name):
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(":")
            nums = [float(x) for x in val.split()]
            out[key.strip()] = nums[0] if len(nums) == 1 else nums
    return out
