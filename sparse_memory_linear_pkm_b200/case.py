"""Runs the layer (selection, recurrence, optional epilogue) on one seeded
synthetic workload, a few times, on cuda:0 — the unit a profiler captures.

    python -m sparse_memory_linear_pkm_b200.case d2048_h16_n1024_dv128 B=2 [T=... H=... sqrt_n=...]
        [--repeat 2] [--variant auto|resident|streaming|pipelined] [--tile K] [--epilogue] [--backward]

Size overrides (B, T, H) shrink a named workload while keeping its slot
count, row width, entry counts and dtypes; sqrt_n=... also changes the slot
count (a smaller state with the same launch grid).
"""

from __future__ import annotations

import argparse

import torch

from . import layer_forward, make_shape, pkm_topk, scan_backward, scan_describe, synth


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("workload", choices=sorted(synth.WORKLOADS))
    ap.add_argument("sizes", nargs="*", help="overrides such as B=2 T=1024 H=4")
    ap.add_argument("--repeat", type=int, default=2)
    ap.add_argument("--variant", default="auto", choices=["auto", "resident", "streaming", "pipelined"])
    ap.add_argument("--tile", type=int, default=0)
    ap.add_argument("--epilogue", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="run the backward (sdm_scan_backward on the layer's selection, random dy) instead")
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args(argv)
    kw = {}
    for item in args.sizes:
        key, val = item.split("=")
        if key not in ("B", "T", "H", "sqrt_n"):
            raise SystemExit(f"unknown size override {key!r} (B, T, H or sqrt_n)")
        kw[key] = int(val)
    shape = synth.WORKLOADS[args.workload].replace(**kw)
    inp = synth.make_inputs(shape, seed=args.seed, device="cuda", with_gate=args.epilogue)
    if args.backward:
        idx_w, w_w = pkm_topk(inp["kp"], shape.W)
        idx_r, w_r = pkm_topk(inp["qp"], shape.R)
        gen = torch.Generator(device="cuda").manual_seed(args.seed)
        dy = torch.randn((shape.B, shape.T, shape.H, shape.d_v), generator=gen, device="cuda")
        M0 = inp["M0"].float().contiguous()
        for _ in range(args.repeat):
            scan_backward(idx_w, w_w, idx_r, w_r, inp["v"], inp["alpha"], inp["beta"], M0, dy)
        torch.cuda.synchronize()
        print("ok backward", shape)
        return
    y = torch.empty((shape.B, shape.T, shape.H, shape.d_v), dtype=torch.float32, device="cuda")
    M = torch.empty((shape.B,) + tuple(inp["M0"].shape), dtype=inp["M0"].dtype, device="cuda")
    for _ in range(args.repeat):
        layer_forward(inp["kp"], inp["qp"], inp["v"], inp["alpha"], inp["beta"], inp["M0"], shape.W, shape.R,
                      g=inp.get("g"), variant=args.variant, y=y, M_out=M, tile=args.tile)
    torch.cuda.synchronize()
    sh = make_shape(shape.B, shape.T, shape.H, shape.sqrt_n, shape.W, shape.R, shape.d_v, shape.torch_in(),
                    shape.torch_state(), variant=args.variant, tile=args.tile)
    print("ok", shape, "recurrence:", scan_describe(sh))


if __name__ == "__main__":
    main()
