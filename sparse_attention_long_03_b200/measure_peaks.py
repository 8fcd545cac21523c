"""Measure this GPU's dense FP8 (e4m3) matmul throughput, the denominator of the prefill
indexer's roofline, the same way as the pool's bf16 figure: an 8192^3 product with
torch._scaled_mm (per-tensor scales, bf16 output), best of 10 launches (burst) and
back-to-back launches for 4 s (sustained), timed with CUDA events.  The bf16 product is
measured beside it for comparison.  Prints one JSON line.

    python -m sparse_attention_long_03_b200.measure_peaks
"""

from __future__ import annotations

import json
import time

import torch


def _time_ms(fn, reps):
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def _measure(fn, flop):
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    burst = min(_time_ms(fn, 1) for _ in range(10))
    # sustained: batches of launches until 4 s have passed
    t_end = time.time() + 4.0
    total_ms, n = 0.0, 0
    while time.time() < t_end:
        total_ms += _time_ms(fn, 20) * 20
        n += 20
    return flop / (burst * 1e-3) / 1e12, flop / (total_ms / n * 1e-3) / 1e12


def main():
    n = 8192
    dev = torch.device("cuda", 0)
    flop = 2.0 * n ** 3
    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()  # column-major operand
    one = torch.ones((), device=dev, dtype=torch.float32)
    fp8 = _measure(lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one,
                                            out_dtype=torch.bfloat16), flop)
    x = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
    y = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
    bf16 = _measure(lambda: torch.matmul(x, y), flop)
    print(json.dumps({"fp8_e4m3_tflops": round(fp8[0], 1),
                      "fp8_e4m3_tflops_sustained": round(fp8[1], 1),
                      "bf16_tflops": round(bf16[0], 1), "bf16_tflops_sustained": round(bf16[1], 1),
                      "how": "torch._scaled_mm e4m3 8192^3 (per-tensor scales, bf16 out) and "
                             "torch.matmul bf16 8192^3: best of 10 (burst), back to back for "
                             "4 s (sustained), CUDA events",
                      "gpu": torch.cuda.get_device_name(dev)}))


if __name__ == "__main__":
    main()
