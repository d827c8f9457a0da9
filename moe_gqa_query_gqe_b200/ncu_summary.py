"""Summarise ncu output for the committed profile notes.

  python -m moe_gqa_query_gqe_b200.ncu_summary launches <launches.csv>
      per kernel: launches, total time, share (from a gpu__time_duration.sum list)
  python -m moe_gqa_query_gqe_b200.ncu_summary traffic <raw.csv> <kernel-regex>
      dram__bytes_read.sum + dram__bytes_write.sum per matching launch
      (from `ncu -i report --page raw --csv`)
"""
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


def dram_traffic(path, pattern):
    import re
    rows = list(csv.reader(open(path)))
    h, u = rows[0], rows[1]
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    out = []
    for r in rows[2:]:
        if not re.search(pattern, r[h.index("Kernel Name")]):
            continue
        tot = 0.0
        for m in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            i = h.index(m)
            tot += float(r[i].replace(",", "")) * scale.get(u[i], 1)
        out.append(tot)
    return out


if __name__ == "__main__":
    if sys.argv[1] == "launches":
        print(summarize(sys.argv[2]))
    elif sys.argv[1] == "traffic":
        for v in dram_traffic(sys.argv[2], sys.argv[3]):
            print(f"{v:.0f}")
