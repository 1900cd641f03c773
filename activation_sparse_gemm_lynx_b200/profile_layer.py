"""Run one Lynx layer a few times, for profilers (ncu) and quick checks.

    python -m activation_sparse_gemm_lynx_b200.profile_layer WORKLOAD [REPS] [--dense]

WORKLOAD is one of the named DiT shapes (attn_out, mlp_up, mlp_down, tiny).
Each repetition writes a 256 MiB buffer (evicting the 126 MB L2) and then
calls lynx_linear on the workload's seeded inputs, so a profiler that skips
the first launches captures a call in the same cache state as bench.py's
timed steps.  Exits non-zero if the library reports a device error.
"""
import sys


def main(argv=None):
    import numpy as np
    import torch

    from . import lynx, workloads

    args = list(sys.argv[1:] if argv is None else argv)
    dense = "--dense" in args
    args = [a for a in args if a != "--dense"]
    if not args or args[0] not in workloads.CONFIGS:
        print(__doc__)
        return 2
    name = args[0]
    reps = int(args[1]) if len(args) > 1 else 3
    torch.cuda.set_device(0)
    lynx.library()
    c = workloads.CONFIGS[name]
    inp = workloads.make_config_inputs(name)

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    X, W, b, A, B = (dev(inp[k]) for k in ("X", "W", "bias", "A", "B"))
    Y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(lynx.lynx_workspace_bytes(c.M, c.N, c.K, c.r), dtype=torch.uint8, device="cuda")
    flush = torch.empty(64 << 20, dtype=torch.int32, device="cuda")
    for _ in range(reps):
        flush.zero_()
        lynx.lynx_linear(X, W, b, A, B, skip_sparsify=dense, Y=Y, workspace=ws)
    torch.cuda.synchronize()
    st, code = lynx.lynx_check_error()
    print(f"{name}: {reps} calls, status {st} code {code:#x}")
    return 0 if st == lynx.LYNX_OK else 1


if __name__ == "__main__":
    sys.exit(main())
