"""Record per-launch DRAM traffic of the library's kernels from an ncu capture.

Reads the CSV that ``ncu -i <report> --page raw --csv`` prints, or the long
form that ``ncu --metrics ... --csv --log-file`` writes during a run (either
with ``dram__bytes_read.sum`` and ``dram__bytes_write.sum``), averages the
launches of each kernel, and stores them in ``profiles/traffic.json`` under the
workload name, keyed by the kernel's timing tag together with the hash of the
source file it was built from (bench.py ignores a record whose source changed).

    ncu -i report.ncu-rep --page raw --csv > raw.csv
    python -m fourier_neural_spectral_fno_b200.profile_traffic raw.csv \
        fno2d_f32_b16_w32_256sq_m16 [--scale S] [--only tag,...]
"""

from __future__ import annotations

import csv
import hashlib
import json
import os
import re
import sys
from collections import defaultdict

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "fourier_neural_spectral_fno_b200", "csrc")

# kernel symbol prefix -> (timing tag, source file)
KERNELS = {
    "k_epi_pipe": ("epi_block_fwd_pipe", "epilogue_pipe.cu"),
    "k_fwd_pipe": ("fwd_transform_pipe", "transform_pipe.cu"),
    "k_proj_pipe": ("proj_fwd_pipe", "proj_pipe.cu"),
    "k_epi_tc": ("epi_block_fwd_tc", "epilogue_tc.cu"),
    "k_s1_tc": ("fwd_transform_tc", "transform_tc.cu"),
    "k_proj_tc": ("proj_fwd_tc", "net_tc.cu"),
    "k_inv_slab": ("inv_slab", "epilogue_tc.cu"),
    "k_mix_fwd": ("mix_fwd", "mix.cu"),
    "k_fwd_finish": ("fwd_finish", "transform.cu"),
    "k_lift4": ("lift", "net.cu"),
    "k_lift": ("lift", "net.cu"),
    "k_proj_bwd": ("proj_bwd", "net.cu"),
    "k_lift_bwd": ("lift_bwd", "net.cu"),
    "k_lift_bwd16": ("lift_bwd", "net.cu"),        # the streaming form
    "k_fwd_fft": ("fwd_fft", "transform_fft.cu"),
    "k_inv_slab_img": ("inv_slab_img", "spec_mid.cu"),
    "k_inv_slab_fft": ("inv_slab_fft", "spec_mid.cu"),
    "k_epi_bwd_pipe": ("epi_block_bwd_pipe", "epilogue_pipe.cu"),
    "k_proj_bwd_pipe": ("proj_bwd_pipe", "proj_pipe.cu"),
    "k_mix_bwd_dx": ("mix_bwd_dx", "mix.cu"),
    "k_mix_bwd_dr": ("mix_bwd_dr", "mix.cu"),
    "k_mix_fwd_1": ("mix_fwd", "mix.cu"),          # the small-shape forms
    "k_mix_bwd_dx_1": ("mix_bwd_dx", "mix.cu"),
    "k_mix_bwd_dr_1": ("mix_bwd_dr", "mix.cu"),
}

# k_epilogue<T, MODE, ...>: the timing tag follows the epilogue mode
EPILOGUE_TAGS = {"0": "epi_spec", "1": "epi_block_fwd", "2": "epi_spec_bwd", "3": "epi_block_bwd"}

UNIT_SCALE = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}


def source_sha(fname: str) -> str:
    with open(os.path.join(CSRC, fname), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


_KERNEL_RE = re.compile(r"\b(k_\w+)\s*(?:<([^()]*)>)?")


def _kernel_key(name: str):
    """(timing tag, source file) of a kernel name as ncu prints it, or None.
    The name's namespaces vary between ncu pages; the kernel is the first
    identifier that starts with ``k_``."""
    m = _KERNEL_RE.search(name.split("(")[0])
    if not m:
        return None
    base, targs = m.group(1), m.group(2)
    if base == "k_fwd_plane":   # k_fwd_plane<TS, T, MP, DZ>: the dz form has its own tag
        args = [t.strip() for t in (targs or "").split(",")]
        dz = bool(args) and args[-1] in ("true", "1")
        return ("fwd_plane_dz" if dz else "fwd_plane", "transform_plane.cu")
    if base == "k_mix_tc_dr":
        return ("mix_bwd_dr_tc", "mix_tc.cu")
    if base == "k_mix_tc":      # k_mix_tc<MB, ADJ>: the adjoint has its own tag
        args = [t.strip() for t in (targs or "").split(",")]
        adj = bool(args) and args[-1] in ("true", "1")
        return ("mix_bwd_dx_tc" if adj else "mix_fwd_tc", "mix_tc.cu")
    if base == "k_epilogue":
        args = [t.strip() for t in (targs or "").split(",")]
        tag = EPILOGUE_TAGS.get(args[1]) if len(args) > 1 else None
        return (tag, "epilogue.cu") if tag else None
    return KERNELS.get(base)


def _parse_long(rows):
    """The long form (one row per launch and metric) that a live run with
    ``--metrics ... --csv --log-file`` writes."""
    col = {h: i for i, h in enumerate(rows[0])}
    per_launch = defaultdict(dict)
    names = {}
    for r in rows[1:]:
        if len(r) != len(rows[0]):
            continue
        m = r[col["Metric Name"]]
        if m not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        try:
            v = float(r[col["Metric Value"]].replace(",", ""))
        except ValueError:
            continue
        per_launch[r[col["ID"]]][m] = v * UNIT_SCALE.get(r[col["Metric Unit"]], 1.0)
        names[r[col["ID"]]] = r[col["Kernel Name"]]
    acc = defaultdict(lambda: [0.0, 0.0, 0])
    for i, mets in per_launch.items():
        key = _kernel_key(names[i])
        if key is None or len(mets) != 2:
            continue
        a = acc[key]
        a[0] += mets["dram__bytes_read.sum"]
        a[1] += mets["dram__bytes_write.sum"]
        a[2] += 1
    return acc


def parse(csv_path: str):
    rows = [r for r in csv.reader(open(csv_path)) if r and not r[0].startswith("==")]
    hdr = rows[0]
    if "Metric Name" in hdr:
        return _parse_long(rows)
    col = {h: i for i, h in enumerate(hdr)}
    acc = defaultdict(lambda: [0.0, 0.0, 0])
    for r in rows[2:]:                       # row 1 holds the units
        key = _kernel_key(r[col["Kernel Name"]])
        if key is None:
            continue
        try:
            rd = float(r[col["dram__bytes_read.sum"]])
            wr = float(r[col["dram__bytes_write.sum"]])
        except (KeyError, ValueError):
            continue
        units = rows[1]
        a = acc[key]
        a[0] += rd * UNIT_SCALE.get(units[col["dram__bytes_read.sum"]], 1.0)
        a[1] += wr * UNIT_SCALE.get(units[col["dram__bytes_write.sum"]], 1.0)
        a[2] += 1
    return acc


def main(argv) -> int:
    import argparse
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("csv")
    ap.add_argument("workload")
    ap.add_argument("--scale", type=float, default=1.0,
                    help="units of the workload's launch per unit of the captured launch "
                         "(a capture of a smaller batch, when traffic grows in proportion)")
    ap.add_argument("--only", default="", help="comma-separated timing tags to record")
    args = ap.parse_args(argv[1:])
    acc = parse(args.csv)
    only = {t for t in args.only.split(",") if t}
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        data = json.load(open(path))
    except Exception:
        data = {}
    wl = data.setdefault(args.workload, {})
    for (tag, src), (rd, wr, n) in sorted(acc.items()):
        if only and tag not in only:
            continue
        rd, wr = rd * args.scale, wr * args.scale
        wl[tag] = {"bytes_per_launch": (rd + wr) / n, "read_bytes": rd / n,
                   "write_bytes": wr / n, "launches": n, "source_sha": source_sha(src)}
        if args.scale != 1.0:
            wl[tag]["scaled_from_capture_by"] = args.scale
        print(f"{tag:22s} {src:18s} read {rd / n / 1e6:8.1f} MB  write {wr / n / 1e6:8.1f} MB")
    with open(path, "w") as f:
        json.dump(data, f, indent=1)
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv))
