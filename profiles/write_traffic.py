"""Record per-launch DRAM traffic of the libcta kernels from an ncu report.

    python profiles/write_traffic.py <report.ncu-rep> "<command that made it>"

Writes profiles/traffic.json with dram__bytes_read.sum + dram__bytes_write.sum
per kernel and a hash of the kernel sources, so bench.py can tell when the
counters no longer describe the code.
"""
import csv
import io
import json
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def main(rep, command):
    import bench
    raw = subprocess.run(["ncu", "-i", rep, "--page", "raw", "--csv"], capture_output=True,
                         text=True, check=True).stdout
    rows = list(csv.reader(io.StringIO(raw)))
    h, units, data = rows[0], rows[1], rows[2:]
    col = {name: h.index(name) for name in ("Kernel Name", "dram__bytes_read.sum",
                                            "dram__bytes_write.sum", "gpu__time_duration.sum")}
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    out = {}
    for r in data:
        name = r[col["Kernel Name"]]
        # score[_kv_tc]_kernel, select_kernel, gather[_tc]_kernel, finalize_tc_kernel
        key = next((k for k in ("score", "select", "gather", "finalize")
                    if re.search(rf"\b{k}(_kv)?(_tc)?_kernel\b", name)), None)
        if key is None:
            continue
        rd = float(r[col["dram__bytes_read.sum"]]) * scale[units[col["dram__bytes_read.sum"]]]
        wr = float(r[col["dram__bytes_write.sum"]]) * scale[units[col["dram__bytes_write.sum"]]]
        out[key] = {"dram_bytes_per_launch": rd + wr, "dram_read": rd, "dram_write": wr}
    rec = {"source_hash": bench.kernel_source_hash(), "command": command, "kernels": out}
    with open(os.path.join(ROOT, "profiles", "traffic.json"), "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps(rec, indent=1))


if __name__ == "__main__":
    main(sys.argv[1], sys.argv[2])
