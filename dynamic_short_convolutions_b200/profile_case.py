"""One layer of a workload, forward + backward, for profiling a kernel under ncu.

    python -m dynamic_short_convolutions_b200.profile_case --config c4_all_linear_2b_block \\
        --layer 2 --batch 2 [--repeats 2] [--rope] [--layout channel_first]

runs the layer's forward and backward `repeats` times on seeded inputs (the
workload's recipe with `batch` sequences of its length), checks the device status
and prints the problem.  With ``--rope`` the QKV layer of the 150M / 2B
workloads fuses RoPE after the conv (base 10000); ``--layout channel_first`` stores
u, y, g and du as [batch, C, seqlen].  Meant for captures such as
``ncu --set full -k regex:lowrank_bwd_kernel -s 1 -c 1 python -m ...``: a
reduced batch keeps the capture small while the inputs stay above L2.
"""
from __future__ import annotations

import argparse
import os
import sys

def build_parser() -> argparse.ArgumentParser:
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="c4_all_linear_2b_block")
    ap.add_argument("--layer", type=int, default=0)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--repeats", type=int, default=2)
    ap.add_argument("--rope", action="store_true")
    ap.add_argument("--layout", default="token_major", choices=["token_major", "channel_first"])
    return ap


def main(argv=None) -> int:
    args = build_parser().parse_args(argv)
    import torch

    from . import _lib as L, ops, workloads as W

    L.load()
    w0 = W.CONFIGS[args.config]
    w = W.scaled(w0, args.batch, w0.seqlen, name=f"{w0.name}_profile")
    layer = w.layers[args.layer]
    t = W.make_inputs(w, layer, args.layer, device="cuda")
    kind = L.LOWRANK if w.kind == W.LOWRANK else L.HEADWISE
    rope = W.ROPE_QKV.get(w0.name) if args.rope and layer.name == "qkv" else None
    table = ops.rope_table(w.seqlen, rope[1], device="cuda") if rope else None
    batch, seqlen = (1, w.tokens) if w.varlen else (w.batch, w.seqlen)
    cf = args.layout == "channel_first"
    if cf:                  # u and g stored [batch, C, seqlen]
        for k in ("u", "g"):
            t[k] = t[k].reshape(batch, seqlen, layer.channels).transpose(1, 2).contiguous()
    plan = ops.DynConvPlan(kind, W.storage_dtype(w), batch, seqlen, layer.d_model, layer.channels, w.ksize, w.rank,
                           w.head_dim, device="cuda", layout=L.CHANNEL_FIRST if cf else L.TOKEN_MAJOR,
                           rope_channels=rope[0] if rope else 0,
                           rope_head_dim=rope[1] if rope else 0, rope_table=table)
    BW = t["B"] if kind == L.LOWRANK else t["W"]
    R = w.rank if kind == L.LOWRANK else (layer.channels // w.head_dim) * w.ksize
    z = torch.empty((w.tokens, R), dtype=W.storage_dtype(w), device="cuda")
    cu = t["cu_seqlens"] if w.varlen else None
    for _ in range(args.repeats):
        plan.forward(t["u"], t["h"], t.get("A"), BW, cu, z_save=z)
        plan.backward(t["g"], t["u"], t["h"], t.get("A"), BW, cu, z_saved=z)
    torch.cuda.synchronize()
    st = L.dynconv_device_status(plan.ws)
    if st != 0:
        print("device status", st, L.dynconv_last_error(), file=sys.stderr)
        return 1
    print(f"{w.name} layer {layer.name}: tokens {w.tokens}, d {layer.d_model}, C {layer.channels}, K {w.ksize}, "
          f"r {w.rank}, head_dim {w.head_dim}, rope {rope}, layout {args.layout}, repeats {args.repeats}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
