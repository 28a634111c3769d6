"""Time the library's bf16 projection kernels through its C ABI (rlt_gemm_bf16).

    python -m cross_token_latent_b200.gemm_bench --shapes 512x1024x1024,64x2048x2048 --kernels 0,2,8
    python -m cross_token_latent_b200.gemm_bench --shapes 512x1024x1024 --kernels 2,8,9,4 --launches 2 --no-timing

Kernel ids are those of rlt_gemm_bf16: 0 = the library's own choice for the shape, 1 = CUDA
cores, 2 + v = row-tile variant v, 11 + s = few-row kernel (s: 0 chosen, 1..4 = split 1/2/4/8),
16 = the weight-streaming CUDA-core kernel (M <= 4), 17 = the persistent row-tile kernel,
18 + p = the CTA-pair tiles 256 x (64 << p).
The weight matrix cycles through enough copies (> 256 MB) that every launch reads it from
HBM, as one decoder step does; the activation panel stays L2-resident.  Launches are queued
behind a device-side sleep so that the host's launch rate does not limit the timing.  With
--no-timing every kernel id runs --launches times and nothing is timed (for profilers).
Prints one line per shape: {kernel id: [us per launch, TFLOP/s]}.
"""
from __future__ import annotations

import argparse
import json
from types import SimpleNamespace

import torch

from .rlt import RLTModel


def _handle_model() -> RLTModel:
    # rlt_gemm_bf16 needs a model handle only for its stream-ordered error flags
    cfg = SimpleNamespace(V=64, d=64, n_heads=4, head_dim=16, L_E=1, L_D=1, F=128, W=2, G=1, dtype="bf16",
                          rms_eps=1e-6, rope_base=10000.0)
    return RLTModel(cfg, max_pos=8)


def main() -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--shapes", required=True, help="comma-separated MxNxK")
    ap.add_argument("--kernels", default="0")
    ap.add_argument("--launches", type=int, default=200)
    ap.add_argument("--no-timing", action="store_true")
    args = ap.parse_args()
    model = _handle_model()
    kernels = [int(k) for k in args.kernels.split(",")]
    for shape in args.shapes.split(","):
        M, N, K = (int(x) for x in shape.split("x"))
        gen = torch.Generator(device="cuda").manual_seed(0)
        A = torch.randn(M, K, device="cuda", generator=gen).to(torch.bfloat16)
        W = (torch.randn(N, K, device="cuda", generator=gen) * 0.05).to(torch.bfloat16)
        n_copies = 2 if args.no_timing else max(1, min(200, (256 << 20) // (N * K * 2) + 1))
        Ws = [W] + [W.clone() for _ in range(n_copies - 1)]
        C = torch.empty(M, N, device="cuda")
        row = {}
        for k in kernels:
            for i in range(3 if not args.no_timing else args.launches):
                model.gemm_bf16(A, Ws[i % n_copies], k, out=C)
            torch.cuda.synchronize()
            if args.no_timing:
                continue
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(20_000_000)
            a.record()
            for i in range(args.launches):
                model.gemm_bf16(A, Ws[i % n_copies], k, out=C)
            b.record()
            torch.cuda.synchronize()
            us = a.elapsed_time(b) * 1e3 / args.launches
            row[k] = [round(us, 2), round(2.0 * M * N * K / us / 1e6, 1)]
        ref = A.float() @ Ws[(args.launches - 1) % n_copies].float().t()     # the last launch's weights
        err = float((C - ref).abs().max())
        model.check_device_errors()
        print(json.dumps({"shape": [M, N, K], "us_tflops": row, "max_abs_err_last": err}), flush=True)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
