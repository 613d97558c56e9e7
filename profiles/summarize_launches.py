"""Summarise an ncu launch list (--metrics gpu__time_duration.sum --csv) per kernel."""
import collections
import csv
import re
import sys


def kernel_label(full: str) -> str:
    full = full.replace("(anonymous namespace)::", "").replace("<unnamed>::", "")
    base = full.split("(")[0]
    base = re.sub(r"^void\s+", "", base)
    m = re.match(r"([\w:<>]*?)(\w+)<", base)
    name = base.split("<")[0]
    tail = name.split("::")[-1]
    if "cta::" in full:
        targs = base[base.find("<") + 1: base.rfind(">")] if "<" in base else ""
        return f"cta::{tail}<{targs}>" if targs else f"cta::{tail}"
    return tail


def main(path):
    rows = list(csv.reader(open(path)))
    hi = [i for i, r in enumerate(rows) if "Kernel Name" in r][0]
    h = rows[hi]
    ki, mi, ui, vi = (h.index(x) for x in ("Kernel Name", "Metric Name", "Metric Unit", "Metric Value"))
    scale = {"ns": 1e-3, "nsecond": 1e-3, "us": 1.0, "usecond": 1.0, "ms": 1e3, "msecond": 1e3}
    agg = collections.OrderedDict()
    for r in rows[hi + 1:]:
        if len(r) <= vi or r[mi] != "gpu__time_duration.sum":
            continue
        a = agg.setdefault(kernel_label(r[ki]), [0, 0.0])
        a[0] += 1
        a[1] += float(r[vi].replace(",", "")) * scale[r[ui]]
    tot = sum(t for _, t in agg.values())
    print(f"{'kernel':64s} {'launches':>8s} {'total us':>11s} {'mean us':>9s} {'share':>6s}")
    for k, (c, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        print(f"{k[:64]:64s} {c:8d} {t:11.1f} {t / c:9.2f} {100 * t / tot:5.1f}%")
    print(f"{'total':64s} {sum(c for c, _ in agg.values()):8d} {tot:11.1f}")


if __name__ == "__main__":
    main(sys.argv[1])
