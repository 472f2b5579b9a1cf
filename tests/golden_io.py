"""Readers for the hand-worked fixtures under tests/golden/."""

import json
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_kv(name):
    """``key = json-value`` lines; '#' starts a comment line."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split("=", 1)
            out[key.strip()] = json.loads(val.strip())
    return out


def _ints(s):
    return [int(x) for x in s.split(",") if x != ""]


def read_trace(name):
    """Allocator trace lines as tuples (see the fixture's header)."""
    ops = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            op = parts[0]
            if op == "pool":
                ops.append(("pool", int(parts[1]), int(parts[2]), _ints(parts[3])))
            elif op == "add":
                ops.append(("add", int(parts[2])))
            elif op == "append":
                sid = int(parts[1])
                if parts[3] == "OOM":
                    ops.append(("append", sid, "OOM", None))
                else:
                    cow = tuple(_ints(parts[5])) if len(parts) > 4 else None
                    ops.append(("append", sid, int(parts[3]), cow))
            elif op == "fork":
                ops.append(("fork", int(parts[1]), int(parts[3])))
            elif op == "free":
                ops.append(("free", int(parts[1])))
            elif op == "state":
                st = {"tables": {}, "lens": {}}
                for kv in parts[1:]:
                    k, v = kv.split("=")
                    if k == "rc":
                        st["rc"] = _ints(v)
                    elif k == "free":
                        st["free"] = _ints(v)
                    elif k.startswith("t"):
                        st["tables"][int(k[1:])] = _ints(v)
                    elif k.startswith("n"):
                        st["lens"][int(k[1:])] = int(v)
                ops.append(("state", st))
            else:
                raise ValueError(line)
    return ops
