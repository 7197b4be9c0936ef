"""Host-side measurement helpers: algorithmic bytes per call, nvidia-smi clock
sampling, peaks and ncu traffic lookup. Pure Python, with no GPU work."""
from __future__ import annotations

import csv
import hashlib
import re
import io
import json
import os
import statistics
import subprocess

from . import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "csrc")

FALLBACK_HBM_GBS = 6650.0  # an earlier B200 copy measurement, used only without MEASURED_PEAKS.json
NVLINK_PEER_GBS = 770.0  # measured B200 peer copy per direction over NVLink 5 (900 GB/s nominal)


# ---- algorithmic bytes -------------------------------------------------------
# What the method itself must move, per call. Implementation-only traffic is
# left out: the layout's per-chunk scratch and re-reads, and L2 misses.

def layout_bytes(w: wl.Workload, N: int | None = None) -> int:
    """Reads logits N*E*4. Writes topk_idx + topk_w + dst_row (N*K*12) and
    is_token_in_rank (N*R)."""
    N = w.N if N is None else N
    return N * w.E * 4 + N * w.K * 12 + N * w.R


def dispatch_bytes(w: wl.Workload, M: int, N: int | None = None) -> int:
    """Reads each token once (N*H*2) and its dst_row + topk_w (N*K*8).
    Writes M rows of H*b bytes (b = 1 FP8, 2 bf16), the FP8 scales
    (M*H/128*4) and recv_src + recv_w (M*8)."""
    N = w.N if N is None else N
    b = 1 if w.fp8 else 2
    scales = M * (w.H // 128) * 4 if w.fp8 else 0
    return N * w.H * 2 + N * w.K * 8 + M * w.H * b + scales + M * 8


def combine_bytes(w: wl.Workload, M: int, fused_fp8: bool = False, N: int | None = None) -> int:
    """Reads the M expert-output rows (bf16: M*H*2; fused FP8: M*H + scales)
    and dst_row + topk_w (N*K*8). Writes N*H*2."""
    N = w.N if N is None else N
    y = M * w.H + M * (w.H // 128) * 4 if fused_fp8 else M * w.H * 2
    return y + N * w.K * 8 + N * w.H * 2


# ---- multi-rank timing --------------------------------------------------------

def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings over the default process group
    (all ranks call it). Single process: the values unchanged."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(values, device=None):
    """Element-wise sum over the default process group (all ranks call it).
    Single process: the values unchanged."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.tolist()


# ---- peaks -------------------------------------------------------------------

def hbm_peak() -> tuple[float, str]:
    """(GB/s, source): the measured copy bandwidth in MEASURED_PEAKS.json, else the fallback."""
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ---- ncu traffic (profiles/traffic.json) -------------------------------------

# The source files each kernel is built from: its own .cu (kernel + launcher)
# and the shared headers. A stored traffic figure stays valid while these stay
# unchanged, whatever happens to the other kernels.
KERNEL_SOURCES = {
    "layout": ("layout.cu",),
    "dispatch": ("dispatch.cu",),
    "combine": ("combine.cu",),
    "dispatch_dedup": ("dedup.cu",),
    "permute": ("dedup.cu",),
    "local_reduce": ("dedup.cu",),
    "combine_dedup": ("dedup.cu",),
}
SHARED_SOURCES = ("common.cuh", "internal.h")

# ncu function names of each kernel (template instances share the name)
NCU_NAMES = {
    "layout": "layout_kernel",
    "dispatch": ("dispatch_bf16_kernel", "dispatch_fp8_kernel"),
    "combine": ("combine_bf16_kernel", "combine_fp8_kernel", "combine_bf16_k8_kernel", "combine_fp8_k8_kernel",
                "combine_bf16_tma_kernel"),
}


_COMMENT = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)


def code_of(text: str) -> str:
    """Source text without its comments and with every run of whitespace
    collapsed to one space: what the compiler sees. (The kernel sources hold
    no string literal with a comment marker in it.)"""
    return " ".join(_COMMENT.sub(" ", text).split())


def source_hash(kernel: str | None = None) -> str:
    """Hash of the code a kernel is built from (all kernel sources when
    `kernel` is None); a stored ncu traffic figure is only valid for the code
    it was captured from. Comments and layout do not count."""
    if kernel is None:
        names = sorted(n for n in os.listdir(CSRC) if n.endswith((".cu", ".cuh", ".h")))
    else:
        names = sorted(set(KERNEL_SOURCES[kernel]) | set(SHARED_SOURCES))
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(CSRC, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(code_of(f.read()).encode())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str) -> float | None:
    """dram read+write bytes per launch at the workload's full size, from the
    committed ncu capture of a smaller case of the same workload scaled by
    tokens (see record_traffic), or None if absent or captured from other
    sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            data = json.load(f)
    except (OSError, ValueError):
        return None
    ent = data.get(workload, {}).get(kernel)
    if not ent or ent.get("source_hash") != source_hash(kernel):
        return None
    return float(ent["dram_bytes_per_launch"])


def _ncu_num(v: str) -> float:
    return float(v.replace(",", ""))


def parse_ncu_metrics(text: str) -> list[dict]:
    """Rows of an `ncu --metrics ... --csv` log: one dict per (launch, metric)
    with the kernel name, the launch id, the metric name, unit and value."""
    lines = text.splitlines()
    start = next((i for i, l in enumerate(lines) if l.startswith('"ID"')), None)
    if start is None:
        return []
    rows = []
    for r in csv.DictReader(io.StringIO("\n".join(lines[start:]))):
        try:
            rows.append({"id": int(r["ID"]), "kernel": r["Kernel Name"], "metric": r["Metric Name"],
                         "unit": r["Metric Unit"], "value": _ncu_num(r["Metric Value"])})
        except (KeyError, ValueError):
            continue
    return rows


_UNIT_BYTES = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}


def traffic_from_ncu(text: str) -> dict:
    """Per kernel (layout / dispatch / combine): dram read and write bytes of
    the last captured launch."""
    per_launch: dict[int, dict] = {}
    for r in parse_ncu_metrics(text):
        ent = per_launch.setdefault(r["id"], {"kernel": r["kernel"]})
        if r["metric"] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            ent[r["metric"]] = r["value"] * _UNIT_BYTES.get(r["unit"], 1)
    out = {}
    for _, ent in sorted(per_launch.items()):
        for kern, prefixes in NCU_NAMES.items():
            names = (prefixes,) if isinstance(prefixes, str) else prefixes
            if any(f"::{n}<" in ent["kernel"] or f"::{n}(" in ent["kernel"] for n in names) \
                    and "dram__bytes_read.sum" in ent:
                rd = int(ent["dram__bytes_read.sum"])
                wr = int(ent.get("dram__bytes_write.sum", 0))
                out[kern] = {"dram_bytes_per_launch": rd + wr, "dram_read": rd, "dram_write": wr,
                             "source_hash": source_hash(kern)}
    return out


def record_traffic(csv_path: str, workload: str, kernel: str, command: str, captured_tokens: int) -> dict:
    """Writes one kernel's dram bytes from an ncu capture of a small case of
    `workload` (captured_tokens tokens per rank) into the traffic file. The
    capture is one kernel (-k) and one launch; the full-size figure scales it
    by tokens, workload T / captured_tokens: every byte the kernels move
    (token rows read or written, receive rows, logits, indices) grows in
    proportion to the tokens at a fixed routing distribution. Stamped with
    the kernel's source hash."""
    with open(csv_path) as f:
        got = traffic_from_ncu(f.read())
    if kernel not in got:
        raise ValueError(f"no {kernel} launch with dram counters in {csv_path}")
    k = got[kernel]
    scale = wl.WORKLOADS[workload].T / captured_tokens
    ent = {"dram_read": k["dram_read"], "dram_write": k["dram_write"], "captured_tokens_per_rank": captured_tokens,
           "scale_to_workload": scale, "dram_bytes_per_launch": int(round((k["dram_read"] + k["dram_write"]) * scale)),
           "source_hash": k["source_hash"], "command": command}
    try:
        with open(TRAFFIC_FILE) as f:
            data = json.load(f)
    except (OSError, ValueError):
        data = {}
    data.setdefault(workload, {})[kernel] = ent
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(data, f, indent=1, sort_keys=False)
        f.write("\n")
    return ent


# ---- clocks ------------------------------------------------------------------

CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

REASON_COLS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    """Samples the SM clock and clock-event (throttle) reasons from a thread
    (NVML, every 1 ms; power every 10th sample), with host timestamps, so the
    caller can keep the samples that fall inside its timed region. Without
    NVML it runs nvidia-smi every 200 ms. Read-only: no GPU setting is
    touched."""

    # NVML clock-event reason bits (nvml.h)
    _BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
             "hw_thermal_slowdown": 0x40}

    def __init__(self, pci_bus_id: str | None = None, interval_s: float = 0.001):
        self.pci_bus_id = pci_bus_id
        self.interval = interval_s
        self.proc = None
        self.thread = None
        self.samples = []  # (t, sm_mhz, max_mhz, power_w or None, reasons)
        self._stop = None
        self._read = None  # one NVML sample (the thread's body), also callable from the caller's thread
        self._last = 0.0

    def start(self):
        try:
            import threading
            import time

            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByPciBusId(self.pci_bus_id) if self.pci_bus_id
                 else pynvml.nvmlDeviceGetHandleByIndex(0))
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._stop = threading.Event()

            def read(with_power: bool):
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0 if with_power else None
                    self.samples.append((time.perf_counter(), sm, mx, pw, rs))
                except Exception:  # noqa: BLE001 - sampling is best effort
                    pass

            self._read = read

            def run():
                i = 0
                while not self._stop.is_set():
                    read(i % 10 == 0)
                    i += 1
                    self._stop.wait(self.interval)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return self
        except Exception:  # noqa: BLE001 - fall back to nvidia-smi
            self.thread = None
        cmd = ["nvidia-smi", f"--query-gpu={CLOCK_QUERY}", "--format=csv", "-lms", "200"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def sample_now(self, min_gap_s: float = 0.001) -> None:
        """One sample from the caller's thread, at most every min_gap_s. The
        bench calls it between step launches, so that the timed region holds
        samples even when the host loop keeps the sampling thread off the
        interpreter for its whole (short) duration."""
        import time
        if self._read is None:
            return
        now = time.perf_counter()
        if now - self._last >= min_gap_s:
            self._last = now
            self._read(False)

    def stop(self, t0: float | None = None, t1: float | None = None) -> dict | None:
        """Stops sampling. Summarises the samples taken in [t0, t1] (host
        perf_counter times), or all of them if none fall inside."""
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
            inside = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
            out = summarize_nvml([x[1:] for x in (inside or self.samples)], self._BITS)
            if out is not None:
                out["window"] = "timed region" if inside else "whole run (no sample inside the timed region)"
            return out
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return parse_clocks(out)


def summarize_nvml(samples, bits) -> dict | None:
    """samples: (sm_mhz, max_mhz, power_w or None, reasons)."""
    if not samples:
        return None
    sm = [s[0] for s in samples]
    pw = [s[2] for s in samples if s[2] is not None]
    reasons = sorted({name for s in samples for name, b in bits.items() if s[3] & b})
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(s[1] for s in samples),
            "reasons": reasons, "samples": len(samples), "power_w_max": max(pw) if pw else None,
            "source": "nvml"}


def _num(s: str) -> float | None:
    s = s.strip().split(" ")[0]
    try:
        return float(s)
    except ValueError:
        return None


def parse_clocks(text: str) -> dict | None:
    rows = list(csv.reader(io.StringIO(text)))
    if len(rows) < 2:
        return None
    head = [h.strip() for h in rows[0]]

    def col(name):
        for i, h in enumerate(head):
            if h.startswith(name):
                return i
        return None

    i_sm, i_max, i_pw = col("clocks.sm"), col("clocks.max.sm"), col("power.draw")
    sm, mx, power, reasons = [], [], [], set()
    for r in rows[1:]:
        if len(r) != len(head):
            continue
        v = _num(r[i_sm]) if i_sm is not None else None
        if v is not None:
            sm.append(v)
        m = _num(r[i_max]) if i_max is not None else None
        if m is not None:
            mx.append(m)
        p = _num(r[i_pw]) if i_pw is not None else None
        if p is not None:
            power.append(p)
        for name in REASON_COLS:
            i = col(f"clocks_event_reasons.{name}")
            if i is not None and r[i].strip().lower() == "active":
                reasons.add(name)
    if not sm:
        return None
    loaded = [s for s, p in zip(sm, power)] if power else sm
    return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx) if mx else None,
            "reasons": sorted(reasons), "samples": len(sm),
            "power_w_max": max(power) if power else None}


def clocks_rejected(clk: dict | None) -> str | None:
    """Why a measurement must be rejected, or None."""
    if not clk:
        return None
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"} & set(clk.get("reasons", []))
    if bad:
        return "throttled: " + ",".join(sorted(bad))
    if clk.get("sm_max_mhz") and clk["sm_mhz"] < 0.6 * clk["sm_max_mhz"] and not clk.get("reasons"):
        return "SM clock far below max with no reason (clock lock?)"
    return None


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser(description="record one kernel's ncu dram traffic, scaled to the full workload")
    ap.add_argument("csv")
    ap.add_argument("workload")
    ap.add_argument("kernel", choices=sorted(NCU_NAMES))
    ap.add_argument("--tokens", type=int, required=True, help="tokens per rank of the captured case")
    ap.add_argument("--command", required=True)
    a = ap.parse_args()
    print(json.dumps(record_traffic(a.csv, a.workload, a.kernel, a.command, a.tokens), indent=1))
