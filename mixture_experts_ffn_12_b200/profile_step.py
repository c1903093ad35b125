"""A few eager calls of the GPT-OSS-20B-shaped layer at T tokens, for ncu captures.

    python -m mixture_experts_ffn_12_b200.profile_step T

Uploads the seeded synthetic layer (the same weights as the prefill workload), takes
the decode recipe's T activation rows and runs four layer calls on cuda:0 (each call
launches the gate/up and down GEMMs once, so `ncu -k regex:decode_gemm_kernel -s 4 -c 2`
captures the third call's two expert GEMMs).  Run from the repository root.
"""
from __future__ import annotations

import sys


def main(argv=None) -> None:
    import torch
    import workloads as W
    from . import api
    T = int((argv or sys.argv[1:] or ["1"])[0])
    spec = W.GPTOSS20B_PREFILL
    d = api.upload_layer(W.make_layer(spec, seed=0))
    layer = api.MoELayer(api.config_from_spec(spec), d["w_router"], d["b_router"], api.expert_weights_from(d))
    x = api.to_torch(W.make_layer(W.gptoss20b_decode(T), seed=0, with_experts=False)["x"]).cuda()
    y = torch.empty_like(x)
    for _ in range(4):
        layer(x, y=y)
    torch.cuda.synchronize()
    print("ok", api.last_device_error())


if __name__ == "__main__":
    main()
