"""Time the activation quantisers on the GPU.

    python -m sparsity_sbl_quantize_b200.run_act T K [--rmsnorm] [--gains] [--iters 20] [--warmup 3]

Quantises seeded bf16 activations X ~ N(0, 1) [T, K] (the generator of
``workloads``) with ``sbl_quantize_act``, or with ``sbl_quantize_act_rmsnorm``
(eps = 1e-6, bf16 gains ~ N(1, 0.25) with ``--gains``), ``warmup + iters``
times, the L2 flushed by a 512 MiB write before each launch, and prints one
JSON line: the mean launch time (CUDA events on the launching stream) and the
algorithmic rate, 3 bytes per element (read 2, write 1) plus 4 per token,
against the measured HBM copy bandwidth when MEASURED_PEAKS.json is present.
"""
import argparse
import json
import os

import numpy as np
import torch

from . import sbl
from . import workloads as wl


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("T", type=int)
    ap.add_argument("K", type=int)
    ap.add_argument("--rmsnorm", action="store_true")
    ap.add_argument("--gains", action="store_true")
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    args = ap.parse_args()
    T, K = args.T, args.K
    x = torch.from_numpy(wl.activations(T, K, seed=1).view(np.int16)).view(torch.bfloat16).cuda()
    g = None
    if args.gains:
        rng = np.random.default_rng(K)
        g = torch.from_numpy(wl.f32_to_bf16_bits(rng.normal(1.0, 0.25, size=K).astype(np.float32)).view(np.int16))
        g = g.view(torch.bfloat16).cuda()
    q = torch.empty((T, K), dtype=torch.int8, device="cuda")
    d = torch.empty((max(T, 1),), dtype=torch.float32, device="cuda")
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    times = []
    for i in range(args.warmup + args.iters):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if args.rmsnorm:
            sbl.sbl_quantize_act_rmsnorm(x, T, K, g, 1e-6, q, d)
        else:
            sbl.sbl_quantize_act(x, T, K, q, d)
        e1.record(stream)
        e1.synchronize()
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    err = sbl.sbl_device_error(clear=True)
    if err:
        raise SystemExit(f"device error flag {err:#x}")
    ms = sum(times) / max(len(times), 1)
    alg = 3.0 * T * K + 4.0 * T
    line = {"kernel": "rmsnorm+quantise" if args.rmsnorm else "quantise", "T": T, "K": K, "gains": bool(g is not None),
            "iters": len(times), "ms_per_launch": round(ms, 5), "algorithmic_bytes": alg,
            "gbs": round(alg / (ms * 1e-3) / 1e9, 1)}
    peaks = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "MEASURED_PEAKS.json")
    if os.path.exists(peaks):
        with open(peaks) as f:
            hbm = json.load(f).get("hbm_gbs")
        if hbm:
            line["frac_of_measured_hbm"] = round(line["gbs"] / hbm, 3)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
