"""Run one workload of the library a fixed number of times, for profilers.

    python -m up_projection_b200.profile_case decode  --M 8 --K 1536 --N 6912 --copies 4 --launches 3
    python -m up_projection_b200.profile_case decode  --M 32 --K 4096 --N 11008 --copies 4 --launches 3
        (9 <= M <= 128 with K a multiple of 64: the tcgen05 weight stream)
    python -m up_projection_b200.profile_case prefill --M 4096 --K 4096 --N 14336 --launches 3
    python -m up_projection_b200.profile_case dswiglu --n 117440512 --launches 3
    python -m up_projection_b200.profile_case fp32    --M 2048 --K 5120 --N 13824 --launches 2
    python -m up_projection_b200.profile_case floor   --K 1536 --N 6912 --copies 4 --launches 3
    python -m up_projection_b200.profile_case fp8     --M 4096 --K 4096 --N 14336 --launches 2
    python -m up_projection_b200.profile_case bwd_dx  --M 4096 --K 4096 --N 14336 --launches 2
    python -m up_projection_b200.profile_case bwd_dw  --M 4096 --K 4096 --N 14336 --launches 2

Each launch of the profiled kernel is preceded by nothing else of this
library, so `ncu -k regex:<name> -s <skip> -c <count>` selects launches by
index.  Decode launches rotate over `copies` distinct weight buffers so each
reads its weights cold.  Exits non-zero if a kernel reports a device-side
timeout.
"""
from __future__ import annotations

import argparse
import sys

import torch


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["decode", "prefill", "dswiglu", "fp32", "floor", "bwd_dx",
                                       "bwd_dw", "bwd_all", "fp8"])
    ap.add_argument("--M", type=int, default=8)
    ap.add_argument("--K", type=int, default=1536)
    ap.add_argument("--N", type=int, default=6912)
    ap.add_argument("--n", type=int, default=8192 * 14336)
    ap.add_argument("--copies", type=int, default=4)
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--fp32", action="store_true",
                    help="bwd_dx / bwd_dw / bwd_all: fp32 (3xTF32) operands")
    ap.add_argument("--weights-stable", action="store_true",
                    help="decode: SWIGLU_FLAG_WEIGHTS_STABLE (programmatic dependent launch)")
    a = ap.parse_args(argv)

    import up_projection_b200 as up
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    L = a.launches
    if a.case in ("decode", "floor"):
        Wg = [(torch.randn((a.N, a.K), generator=g, device=dev) / a.K ** 0.5).to(torch.bfloat16)
              for _ in range(a.copies)]
        Wu = [(torch.randn((a.N, a.K), generator=g, device=dev) / a.K ** 0.5).to(torch.bfloat16)
              for _ in range(a.copies)]
        X = torch.randn((a.M, a.K), generator=g, device=dev).to(torch.bfloat16)
        H = torch.empty((a.M, a.N), dtype=torch.bfloat16, device=dev)
        sink = torch.empty(4096, dtype=torch.int32, device=dev)
        for i in range(L):
            c = i % a.copies
            if a.case == "decode":
                up.swiglu_fwd(X, Wg[c], Wu[c], H, weights_stable=a.weights_stable)
            else:
                up.swiglu_read_floor(Wg[c], Wu[c], sink)
    elif a.case in ("prefill", "fp32"):
        dt = torch.bfloat16 if a.case == "prefill" else torch.float32
        X = torch.randn((a.M, a.K), generator=g, device=dev).to(dt)
        Wg = (torch.randn((a.N, a.K), generator=g, device=dev) / a.K ** 0.5).to(dt)
        Wu = (torch.randn((a.N, a.K), generator=g, device=dev) / a.K ** 0.5).to(dt)
        H = torch.empty((a.M, a.N), dtype=dt, device=dev)
        for _ in range(L):
            up.swiglu_fwd(X, Wg, Wu, H)
    elif a.case == "fp8":
        bf = torch.bfloat16
        X = torch.randn((a.M, a.K), generator=g, device=dev).to(bf)
        Wg = (torch.randn((a.N, a.K), generator=g, device=dev) / a.K ** 0.5).to(bf)
        Wu = (torch.randn((a.N, a.K), generator=g, device=dev) / a.K ** 0.5).to(bf)
        for _ in range(L):
            up.swiglu_fwd_fp8(X, Wg, Wu)
    elif a.case in ("bwd_dx", "bwd_dw", "bwd_all"):
        bf = torch.float32 if a.fp32 else torch.bfloat16
        dG = torch.randn((a.M, a.N), generator=g, device=dev).to(bf)
        dU = torch.randn((a.M, a.N), generator=g, device=dev).to(bf)
        if a.case == "bwd_all":
            # dX, dWg and dWu in one launch (swiglu_bwd_gemms)
            X = torch.randn((a.M, a.K), generator=g, device=dev).to(bf)
            Wg = (torch.randn((a.N, a.K), generator=g, device=dev) / a.K ** 0.5).to(bf)
            Wu = (torch.randn((a.N, a.K), generator=g, device=dev) / a.K ** 0.5).to(bf)
            for _ in range(L):
                up.swiglu_bwd_gemms(dG, dU, Wg, Wu, X)
        elif a.case == "bwd_dx":
            Wg = (torch.randn((a.N, a.K), generator=g, device=dev) / a.K ** 0.5).to(bf)
            Wu = (torch.randn((a.N, a.K), generator=g, device=dev) / a.K ** 0.5).to(bf)
            dX = torch.empty((a.M, a.K), dtype=bf, device=dev)
            for _ in range(L):
                up.swiglu_bwd_dx(dG, dU, Wg, Wu, dX)
        else:
            X = torch.randn((a.M, a.K), generator=g, device=dev).to(bf)
            dWg = torch.empty((a.N, a.K), dtype=bf, device=dev)
            dWu = torch.empty((a.N, a.K), dtype=bf, device=dev)
            for _ in range(L):
                up.swiglu_bwd_dw(dG, dU, X, dWg, dWu)
    else:
        dH, G, U = (torch.randn(a.n, generator=g, device=dev).to(torch.bfloat16) for _ in range(3))
        dG, dU = torch.empty_like(G), torch.empty_like(U)
        for _ in range(L):
            up.dswiglu_bwd(dH, G, U, dG, dU)
    torch.cuda.synchronize()
    st = up.swiglu_sync_status()
    if st != 0:
        print("device status:", up.status_string(st), file=sys.stderr)
        return 1
    print(f"{a.case}: {L} launches ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
