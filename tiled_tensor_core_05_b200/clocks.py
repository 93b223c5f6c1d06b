"""SM clock, power and clock-event reasons sampled through NVML (read-only
queries) while the GPU works, for timing records taken under the power cap.
Nothing here changes a GPU setting."""
from __future__ import annotations

import statistics
import threading
import time


class ClockSampler:
    """SM clock, power and clock-event reasons polled through NVML (read-only
    queries) every ~1 ms from a background thread while the GPU works."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, gpu_uuid: str, interval_s: float = 0.001):
        self.samples = []
        self.marks = {}
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(gpu_uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.bits = [(name, getattr(pynvml, attr)) for name, attr in self.REASONS]
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = repr(e)
            return
        self.interval = interval_s
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv, h = self.nv, self.h
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((time.monotonic(), sm, rs, pw))
            except Exception:
                pass
            time.sleep(self.interval)

    def wait_first(self, timeout=5.0):
        t0 = time.monotonic()
        while self.ok and not self.samples and time.monotonic() - t0 < timeout:
            time.sleep(0.005)

    def mark(self, name):
        self.marks[name] = time.monotonic()

    def stop(self):
        self._stop.set()
        if self.ok:
            self.thread.join(timeout=2)

    def summary(self, start="t0", end="t1"):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable: " + getattr(self, "err", "")}
        t0, t1 = self.marks.get(start, 0.0), self.marks.get(end, 1e30)
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "NVML samples taken during the timed region"
        if len(inside) < 3:
            w0 = self.marks.get("warm0", t0)
            inside = [s for s in self.samples if w0 <= s[0] <= t1]
            note = "timed region too short for 3 samples; warm-up + timed samples"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": "no sample during the busy period"}
        reasons = sorted({name for s in inside for name, bit in self.bits if s[2] & bit})
        return {"sm_mhz": statistics.median(s[1] for s in inside),
                "sm_mhz_min": min(s[1] for s in inside),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside),
                "power_w_max": round(max(s[3] for s in inside), 1), "note": note}


def gpu_id_for(dev_index: int) -> str:
    """NVML UUID string ("GPU-...") of a torch device index."""
    import torch
    s = str(torch.cuda.get_device_properties(dev_index).uuid)
    return s if s.startswith("GPU-") else "GPU-" + s
