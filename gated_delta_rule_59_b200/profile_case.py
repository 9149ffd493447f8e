"""A few launches of one workload through the library, for profiler captures.

    python -m gated_delta_rule_59_b200.profile_case gated --launches 2
    python -m gated_delta_rule_59_b200.profile_case small --launches 2
    python -m gated_delta_rule_59_b200.profile_case decode --launches 3
    python -m gated_delta_rule_59_b200.profile_case gated --launches 2 --chunk-states

``gated``: the gated prefill workload (B=2, T=8192, Hqk=16, Hv=32, d=128, bf16 in,
fp32 o); ``small``: the same shape family at B=2, T=2048, Hqk=2, Hv=4; ``decode``: one
decode step at B=256, H=32, d=128 with an fp32 state.  ``--chunk-states``: the prefill also
returns the state after every 64-token chunk.  Inputs come from the seeded
generators in ``inputs``; nothing else runs, so an ncu capture with ``-s 1 -c 1`` sees
exactly one warm launch.
"""
import argparse

import torch

from . import chunk_fwd, device_status, recurrent_step
from . import inputs


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["gated", "small", "decode"])
    ap.add_argument("--launches", type=int, default=2)
    ap.add_argument("--chunk-states", action="store_true")
    args = ap.parse_args(argv)
    dev = torch.device("cuda:0")
    if args.case == "decode":
        state, steps = inputs.decode_config(n_steps=1, B=256)
        state, step = state.to(dev), steps[0].to(dev)
        for _ in range(args.launches):
            o = recurrent_step(step.q, step.k, step.v, step.g, step.beta, state)
    else:
        B, T, Hqk, Hv = (2, 8192, 16, 32) if args.case == "gated" else (2, 2048, 2, 4)
        p = inputs.prefill(B, T, Hqk, Hv, 128, 128, torch.bfloat16, gated=True, state_std=0.02,
                           seed=5).to(dev)
        for _ in range(args.launches):
            o = chunk_fwd(p.q, p.k, p.v, p.g, p.beta, p.state_in, None,
                          output_chunk_states=args.chunk_states)[0]
    torch.cuda.synchronize()
    if device_status() != 0:
        raise SystemExit("device status %d" % device_status())
    print("ok", float(o.float().abs().sum()))


if __name__ == "__main__":
    main()
