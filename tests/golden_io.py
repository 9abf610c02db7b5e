"""Reader for the hand-computed position fixtures under tests/golden/."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_positions(name):
    """Returns (types, grids, [t, h, w], next) from a golden positions file."""
    fields = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            fields[key.strip()] = val.strip()
    types = [int(v) for v in fields["types"].split()]
    grids = [tuple(int(v) for v in g.split()) for g in fields["grids"].split(";")]
    pos = [[int(v) for v in fields[a].split()] for a in ("t", "h", "w")]
    return types, grids, pos, int(fields["next"])


def all_position_files():
    return sorted(n for n in os.listdir(GOLDEN) if n.startswith("positions_"))
