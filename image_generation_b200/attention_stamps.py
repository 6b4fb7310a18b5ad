"""Per-phase timing of the attention kernel from its own clock stamps.

    python -m image_generation_b200.build --stamps
    python -m image_generation_b200.attention_stamps [--head-dim 96 128]

Runs the diagnostic build of the library (libh3dit_stamps.so, selected
through H3DIT_LIB) on the 4096^2 sequence (16,896 tokens, 56 heads, random
Q|K|V) and prints, as JSON, medians over steps 10 .. 249 of the stamped CTA's
264 steps of 64 keys, in SM clocks:
  - each phase of a softmax warp: waiting for S, loading the scores, the row
    max, the exponentials (with sums and the bf16 pack), storing P, handing
    P back; and the period of a step;
  - how far apart the four softmax warps of a query tile hand P back;
  - each MMA issuer: from the last hand-back to the issuer seeing P, issuing
    PV, waiting for K two steps ahead, issuing that S, and until the softmax
    sees it;
  - the phase of query tile 1's steps against tile 0's.
Measurement only: the stamped kernel is the product kernel with clock64()
stores at those points.
"""
from __future__ import annotations

import argparse
import ctypes as C
import json
import os
import sys

D, H, N = 5376, 56, 16896
FIRST, LAST = 10, 250


def _median(x):
    import numpy as np

    return float(np.median(x))


def analyse(st) -> dict:
    """st: int64 [steps, slots] stamps with the layout attention.cu documents."""
    import numpy as np

    a, b = FIRST, LAST
    names = ["S_seen", "scores_loaded", "row_max", "exponentials", "P_stored", "P_handed_back"]
    res = {}
    for t in (0, 1):
        base = 6 * t
        ph = {f"{names[i - 1]}_to_{names[i]}": _median(st[a:b, base + i] - st[a:b, base + i - 1])
              for i in range(1, 6)}
        ph["wait_for_next_S"] = _median(st[a + 1:b + 1, base] - st[a:b, base + 5])
        ph["period"] = _median(st[a + 1:b + 1, base] - st[a:b, base])
        arr = st[a:b, 20 + 4 * t:24 + 4 * t]
        ph["hand_back_after_first_warp"] = [_median(arr[:, k] - arr.min(axis=1)) for k in range(4)]
        ph["hand_back_spread"] = _median(arr.max(axis=1) - arr.min(axis=1))
        res[f"softmax_tile{t}"] = ph
        iss = 12 + 3 * t
        res[f"issuer_tile{t}"] = {
            "last_hand_back_to_P_seen": _median(st[a:b, iss] - arr.max(axis=1)),
            "issue_PV": _median(st[a:b, iss + 1] - st[a:b, iss]),
            "wait_K_two_steps_ahead": _median(st[a + 2:b + 2, 28 + t] - st[a:b, iss + 1]),
            "issue_S_two_steps_ahead": _median(st[a:b, iss + 2] - st[a + 2:b + 2, 28 + t]),
            "S_issued_to_softmax_sees_it": _median(st[a + 2:b + 2, base] - st[a:b, iss + 2]),
        }
    d = st[a:b, 6] - st[a:b, 0]
    res["tile1_S_seen_minus_tile0"] = {"median": _median(d),
                                       "p10_p90": [float(np.percentile(d, 10)),
                                                   float(np.percentile(d, 90))]}
    res["tma_stage_period"] = _median(np.diff(st[a:b, 18]))
    return res


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--head-dim", type=int, nargs="+", default=[96, 128], choices=[96, 128])
    args = ap.parse_args()

    from . import build as B

    os.environ.setdefault("H3DIT_LIB", B.LIB_STAMPS)
    if not os.path.exists(os.environ["H3DIT_LIB"]):
        sys.exit(f"{os.environ['H3DIT_LIB']} is missing: python -m image_generation_b200.build --stamps")
    import numpy as np
    import torch

    from . import h3dit as Hb

    out = {"library": os.path.basename(Hb.LIB_PATH), "tokens": N, "heads": H}
    for dh in args.head_dim:
        I = H * dh
        g = torch.Generator(device="cuda")
        g.manual_seed(dh)
        qkv = torch.randn(N, 3 * I, device="cuda", generator=g).bfloat16()
        dummy = torch.zeros(1 << 16, device="cuda", dtype=torch.bfloat16)
        tw = {k: torch.zeros(D * 256 if k == "w_t1" else (D * D if k == "w_t2" else D),
                             device="cuda") for k in ("w_t1", "b_t1", "w_t2", "b_t2")}
        blk = {k: dummy for k in ("w_qkv", "w_o", "w_ff1", "w_ff2", "w_ada")}
        blk["b_ada"] = torch.zeros(6 * D, device="cuda")
        ctx = Hb.Context(Hb.make_config(D, H, dh, 14336, 1, N), tw, [blk])
        o = torch.empty(N, I, device="cuda", dtype=torch.bfloat16)
        for _ in range(4):  # warm-up; the table keeps the last launch
            ctx.attention(qkv[:, :I], qkv[:, I:2 * I], qkv[:, 2 * I:], 3 * I, o, I, N)
        torch.cuda.synchronize()
        if ctx.sync_status() != 0:
            sys.exit("attention failed")
        slots, steps = Hb.H3DIT_ATTN_STAMP_SLOTS, Hb.H3DIT_ATTN_STAMP_STEPS
        buf = (C.c_uint64 * (slots * steps))()
        Hb.check(None, Hb.lib.h3dit_attention_stamps(buf, slots, steps))
        st = np.frombuffer(buf, dtype=np.uint64).astype(np.int64).reshape(steps, slots)
        st = st[:(N + 63) // 64]
        st = st - st[st > 0].min()
        out[f"head_dim_{dh}"] = analyse(st)
        ctx.close()
    print(json.dumps(out, indent=1))


if __name__ == "__main__":
    main()
