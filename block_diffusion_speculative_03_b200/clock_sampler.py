"""Sample SM clocks, power and clock-event reasons of one GPU through NVML
until stdin closes; print one CSV line per sample.  Run as a separate process
so the sampling does not compete with the launching thread."""
import sys
import threading
import time


def main():
    idx = int(sys.argv[1]) if len(sys.argv) > 1 else 0
    period = float(sys.argv[2]) if len(sys.argv) > 2 else 0.01
    import pynvml as N
    N.nvmlInit()
    h = N.nvmlDeviceGetHandleByIndex(idx)
    max_sm = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
    stop = threading.Event()
    threading.Thread(target=lambda: (sys.stdin.read(), stop.set()), daemon=True).start()
    print("max_sm,%d" % max_sm, flush=True)
    while not stop.is_set():
        sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
        try:
            reasons = N.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception:
            reasons = N.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        try:
            pw = N.nvmlDeviceGetPowerUsage(h) / 1000.0
        except Exception:
            pw = -1.0
        print("%.4f,%d,%d,%.1f" % (time.time(), sm, reasons, pw), flush=True)
        time.sleep(period)


if __name__ == "__main__":
    main()
