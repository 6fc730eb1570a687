"""Run one Sparse-BitLinear layer forward on the GPU and time it.

    python -m sparsity_sbl_quantize_b200.run_layer O K T[,T2,...] [--nm 2:4] [--format sp24|i8|pk2|t24|batch]
                                                   [--copies N] [--iters 20] [--warmup 3]

Packs a seeded synthetic layer (W ~ N(0, 0.02) fp32, X ~ N(0, 1) bf16, the
generators of ``workloads``), quantises the activations, then launches
``sbl_forward`` ``warmup + iters`` times in the given packed format (default:
the one ``sbl_forward_format`` recommends) and prints, per token count, one
JSON line with the mean launch time over the timed iterations (CUDA events on the launching
stream; L2 flushed before each launch), the dense-equivalent and kept-weight
int8 rates.  It is the single-layer unit a profiler can capture in isolation.
With ``--format batch`` the layer is packed ``--copies`` times (PK2) and one
``sbl_forward_batch`` launch runs all copies; the line then also gives the
algorithmic GB/s (2-bit weights, int8 X and scales read, bf16 Y written).
"""
import argparse
import json

import torch

from . import sbl
from . import workloads as wl

FORMATS = {"i8": sbl.SBL_FMT_I8, "pk2": sbl.SBL_FMT_PK2, "sp24": sbl.SBL_FMT_SP24, "t24": sbl.SBL_FMT_T24,
           "batch": -1}


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("O", type=int, help="out_features")
    ap.add_argument("K", type=int, help="in_features")
    ap.add_argument("T", help="tokens, or a comma-separated list of token counts run one after another")
    ap.add_argument("--nm", default="2:4", help="N:M pattern, e.g. 6:8")
    ap.add_argument("--format", choices=sorted(FORMATS), default=None)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--copies", type=int, default=40, help="--format batch: packed copies of the layer")
    args = ap.parse_args()
    n, m = (int(v) for v in args.nm.split(":"))
    O, K = args.O, args.K
    tokens = [int(t) for t in args.T.split(",")]

    dsc = sbl.desc(O, K, n, m)
    fmt = FORMATS[args.format] if args.format else sbl.sbl_forward_format(dsc, max(tokens))
    if fmt == 0:
        raise SystemExit(f"no forward format for O={O} K={K} {n}:{m}")
    w = torch.from_numpy(wl.master_weights(O, K, seed=args.seed)).cuda()
    batch = fmt == -1
    ws = sbl.alloc_workspace(sbl.sbl_workspace_bytes(dsc, 0, sbl.SBL_OP_QUANTIZE_MASK_PACK))
    copies = []
    for _ in range(args.copies if batch else 1):
        packed = sbl.alloc_packed(dsc, sbl.SBL_FMT_PK2 if batch else fmt)
        sbl.sbl_quantize_mask_pack(dsc, w, sbl.SBL_FMT_PK2 if batch else fmt, packed, ws)
        copies.append(packed)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    name = {v: k for k, v in FORMATS.items()}[fmt]
    for T in tokens:
        x = torch.from_numpy(wl.activations(T, K, seed=args.seed).view("int16")).view(torch.bfloat16).cuda()
        xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
        d = torch.empty((max(T, 1),), dtype=torch.float32, device="cuda")
        sbl.sbl_quantize_act(x, T, K, xq, d)
        y = torch.empty((T, O), dtype=torch.bfloat16, device="cuda")
        if batch:
            ys = [torch.empty((T, O), dtype=torch.bfloat16, device="cuda") for _ in copies]
            arr = sbl.batch_array([sbl.batch_layer(dsc, p, yy, xq, d) for p, yy in zip(copies, ys)])
            bws = sbl.alloc_workspace(sbl.sbl_forward_batch_workspace_bytes(arr, len(copies), T))
        times = []
        for i in range(args.warmup + args.iters):
            flush.fill_(i & 0xFF)
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record(stream)
            if batch:
                sbl.sbl_forward_batch(arr, len(copies), T, bws)
            else:
                sbl.sbl_forward(dsc, xq, d, T, packed, fmt, y)
            end.record(stream)
            end.synchronize()
            if i >= args.warmup:
                times.append(start.elapsed_time(end))
        err = sbl.sbl_device_error(clear=True)
        if err:
            raise SystemExit(f"device error flag {err:#x}")
        ms = sum(times) / max(len(times), 1)
        dense_ops = 2.0 * T * O * K * len(copies)
        line = {"O": O, "K": K, "T": T, "nm": f"{n}:{m}", "format": name, "iters": len(times),
                "ms_per_launch": round(ms, 5),
                "dense_equivalent_tops": round(dense_ops / (ms * 1e-3) / 1e12, 2),
                "kept_tops": round(dense_ops * n / m / (ms * 1e-3) / 1e12, 2)}
        if batch:
            alg = len(copies) * (O * K / 4 + T * K + 4 * T + 2 * T * O)
            line.update(copies=len(copies), algorithmic_bytes=alg, gbs=round(alg / (ms * 1e-3) / 1e9, 1))
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
