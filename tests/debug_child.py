"""Child process of test_gpu_debug_build: runs the layer on small odd shapes through ONE
library file (the release or the bounds-checking debug build of libsvdq) and saves every
output, so that the test can compare the two builds bit for bit.

    python tests/debug_child.py <library.so> <out.npz>
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

# (M, K, N, rank): ragged M, K % 256 == 128 (the FP4 GEMM's two-load fallback), a single
# row, rank 0, and a small batch that takes the prologue's K split
SHAPES = [(129, 384, 384, 16), (1, 256, 128, 0), (300, 640, 640, 48), (40, 2048, 256, 16)]
FORMATS = ["nvfp4", "int4", "mxfp4", "w8a8"]


def main(lib_path: str, out: str) -> None:
    import torch

    from bit_w4a4_quantized_group_b200 import binding as B
    from bit_w4a4_quantized_group_b200 import prepare as P
    from bit_w4a4_quantized_group_b200.layer import W4A4LowRankLinear

    B.load(lib_path)
    dev = torch.device("cuda", 0)
    res = {}
    for fmt in FORMATS:
        for (M, K, N, rank) in SHAPES:
            rng = np.random.default_rng(M * 7 + K + N + rank)
            X = rng.standard_normal((M, K)).astype(np.float32)
            X[:, rng.integers(0, K, 4)] *= 30.0                      # a few outlier channels
            prep = {"lam": rng.uniform(0.5, 4.0, K).astype(np.float32),
                    "R_nk": (rng.standard_normal((N, K)) * 0.02).astype(np.float32),
                    "L1_rk": (rng.standard_normal((rank, K)) * 0.05).astype(np.float32),
                    "L2_nr": (rng.standard_normal((N, rank)) * 0.05).astype(np.float32),
                    "act_gscale": 1.0}
            bias = (rng.standard_normal(N) * 0.1).astype(np.float32)
            lin = W4A4LowRankLinear(fmt, N, K, P.pack(fmt, prep), prep["lam"], 1.0, bias, device=dev)
            Xd = torch.from_numpy(X).to(dev).to(torch.bfloat16)
            Y = lin.forward(Xd, check=True)                          # raises on a device error
            torch.cuda.synchronize()
            res[f"{fmt}_{M}_{K}_{N}_{rank}"] = Y.view(torch.int16).cpu().numpy()
    st, site = B.svdq_get_last_device_error(None)
    res["device_error"] = np.array([st, site])
    np.savez(out, **res)


if __name__ == "__main__":
    main(sys.argv[1], sys.argv[2])
