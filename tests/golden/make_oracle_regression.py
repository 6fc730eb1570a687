"""Write tests/golden/oracle_regression_16x32.txt: every stage of the oracle
on one small seeded layer, so that any later change to the oracle's
arithmetic shows up as a changed fixture (and has to say why).

Calls only oracle/ (and the seeded input generators).  The inputs are stored
in the file as bit patterns, so the check does not depend on the random
generator.  Run from the repository root:

    python tests/golden/make_oracle_regression.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from sparsity_sbl_quantize_b200 import workloads as wl  # noqa: E402

OUT = os.path.join(ROOT, "tests", "golden", "oracle_regression_16x32.txt")
O, K, T, SEED = 16, 32, 5, 11
PATTERNS = [(6, 8), (2, 4)]


def hex32(a):
    return " ".join(f"{v:08x}" for v in np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).ravel())


def hex16(a):
    return " ".join(f"{v:04x}" for v in np.ascontiguousarray(a, dtype=np.uint16).ravel())


def hex8(a):
    return " ".join(f"{v:02x}" for v in np.ascontiguousarray(a).view(np.uint8).ravel())


def ints(a):
    return " ".join(str(int(v)) for v in np.asarray(a).ravel())


def f64(a):
    return " ".join(float(v).hex() for v in np.asarray(a, dtype=np.float64).ravel())


def stages(w, x, dy, g_bits):
    """Every oracle stage on (w, x, dy), as key -> text."""
    out = {}
    for n, m in PATTERNS:
        tag = f"{n}of{m}"
        layer = oracle.Layer(w, n, m)
        out[f"{tag}.gamma"] = hex32([layer.gamma])
        out[f"{tag}.mask"] = ints(layer.mask)
        out[f"{tag}.weff"] = ints(layer.weff)
        out[f"{tag}.pk2"] = hex8(oracle.pack_pk2(layer.weff))
        vals, bm = oracle.pack_nm(layer.weff, layer.mask, n, m)
        out[f"{tag}.nm_values"] = hex8(vals)
        out[f"{tag}.nm_bitmap"] = hex8(bm)
        if n <= 2:
            sv, sm = oracle.pack_sp24(layer.weff, layer.mask)
            out[f"{tag}.sp24_values"] = hex8(sv)
            out[f"{tag}.sp24_meta"] = hex8(sm)
            lo, hi = oracle.pack_t24(layer.weff)
            out[f"{tag}.t24_lo"] = hex8(lo)
            out[f"{tag}.t24_hi"] = hex8(hi)
        q, d, acc, y, yb = layer.forward(x)
        out[f"{tag}.q"] = ints(q)
        out[f"{tag}.d"] = hex32(d)
        out[f"{tag}.acc"] = ints(acc)
        out[f"{tag}.y"] = hex32(y)
        out[f"{tag}.y_bf16"] = hex16(yb)
        e, eb = oracle.epilogue(y, relu2=True, residual_bf16_bits=np.ascontiguousarray(x[:, :O]))
        out[f"{tag}.epilogue_relu2_residual"] = hex32(e)
        out[f"{tag}.epilogue_relu2_residual_bf16"] = hex16(eb)
        dx, dw = oracle.backward(dy, layer.weff, layer.gamma, q, d)
        out[f"{tag}.dx"] = f64(dx)
        out[f"{tag}.dw"] = f64(dw)
    qn, dn = oracle.rmsnorm_quantize_act(x, g_bits, 1e-5)
    out["rmsnorm.q"] = ints(qn)
    out["rmsnorm.d"] = hex32(dn)
    return out


def inputs():
    w = wl.master_weights(O, K, seed=SEED)
    x = wl.activations(T, K, seed=SEED, outlier_frac=0.05)
    dy = wl.output_grad(T, O, seed=SEED)
    g = wl.activations(1, K, seed=SEED + 1)[0]
    return w, x, dy, g


def main():
    w, x, dy, g = inputs()
    lines = [
        "# Every oracle stage on one seeded 16 x 32 layer (T = 5), written by",
        "# tests/golden/make_oracle_regression.py, which calls only oracle/.  Inputs are",
        "# stored as bit patterns (w fp32, x / dy / rmsnorm gains bf16); floats as hex",
        "# bits, fp64 gradients as C99 hex floats.  A change to this file is a change to",
        "# the oracle's arithmetic.",
        f"shape: {O} {K} {T}",
        f"w: {hex32(w)}",
        f"x: {hex16(x)}",
        f"dy: {hex16(dy)}",
        f"rmsnorm.g: {hex16(g)}",
    ]
    for k, v in stages(w, x, dy, g).items():
        lines.append(f"{k}: {v}")
    with open(OUT, "w") as f:
        f.write("\n".join(lines) + "\n")
    print(OUT)


if __name__ == "__main__":
    main()
