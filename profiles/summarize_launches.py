"""Summarise an ncu --csv launch list (gpu__time_duration.sum) per kernel:
launches, total time and share. Usage: python profiles/summarize_launches.py launches.csv"""
import collections
import csv
import sys


def summarize(path):
    rows = list(csv.reader(open(path)))
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    h = rows[hi]
    ki, mi, vi, ui = h.index("Kernel Name"), h.index("Metric Name"), h.index("Metric Value"), h.index("Metric Unit")
    scale = {"ns": 1e-3, "nsecond": 1e-3, "us": 1.0, "usecond": 1.0, "ms": 1e3, "msecond": 1e3, "s": 1e6, "second": 1e6}
    agg = collections.OrderedDict()
    for r in rows[hi + 1:]:
        if len(r) <= vi or r[mi] != "gpu__time_duration.sum":
            continue
        name = r[ki].split("(")[0]
        a = agg.setdefault(name, [0, 0.0])
        a[0] += 1
        a[1] += float(r[vi].replace(",", "")) * scale.get(r[ui], 1.0)
    tot = sum(v[1] for v in agg.values())
    out = ["| kernel | launches | total us | share | avg us |", "|---|---|---|---|---|"]
    for n, (c, t) in sorted(agg.items(), key=lambda kv: -kv[1][1]):
        out.append(f"| `{n}` | {c} | {t:.1f} | {100 * t / tot:.1f}% | {t / c:.2f} |")
    return "\n".join(out)


if __name__ == "__main__":
    print(summarize(sys.argv[1]))
