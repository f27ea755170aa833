"""Run a few optimizer steps on (the first weights of) a workload, for a
profiler to capture.

  python -m shampoo_second_order_b200.run_steps [--config transformer_big_b1024]
      [--params 6] [--steps 3] [--gemm-tiles pair|single] [--roots fp64|int8]

Takes the first --params parameters of the named workload (default: the six
weights of Transformer-big layer 0, 20 blocks of 1024 x 1024), creates a
context on cuda:0 and runs --steps steps (roots on the first), with the
seeded synthetic inputs of the workloads module.  Small enough for an ncu
capture of individual launches; the kernels are those of the full workload.
"""
from __future__ import annotations

import argparse

from . import workloads as wl


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="transformer_big_b1024", choices=sorted(wl.CONFIGS))
    ap.add_argument("--params", type=int, default=6)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--gemm-tiles", default="pair", choices=["pair", "single"])
    ap.add_argument("--roots", default="fp64", choices=["fp64", "int8"])
    args = ap.parse_args(argv)
    import torch
    from .optimizer import Shampoo
    c = wl.CONFIGS[args.config]
    shapes = c["shapes"][:args.params]
    gdt = torch.bfloat16 if c["grad_dtype"] == "bf16" else torch.float32
    W = [torch.from_numpy(w).cuda() for w in wl.make_params(shapes, c["seed"])]
    G = [torch.from_numpy(g).cuda().to(gdt)
         for g in wl.make_grads(shapes, c["seed"], 0, c["grad_std"], c["grad_dtype"])]
    opt = Shampoo(shapes, c["block_size"], c["beta2"], c["eps"], c["p"], c["graft"], c["momentum"],
                  c["grad_dtype"])
    opt.set_gemm_tiles(args.gemm_tiles == "pair")
    opt.set_root_method(args.roots)
    for t in range(args.steps):
        opt.step(W, G, c["lr"], t == 0)
    torch.cuda.synchronize()
    opt.close()
    print(f"{args.steps} steps of {len(shapes)} parameters of {args.config} ({args.gemm_tiles} tiles) done")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
