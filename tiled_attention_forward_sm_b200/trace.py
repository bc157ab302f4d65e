"""Timeline of the attention kernel's roles from the tracing build.

    python -m tiled_attention_forward_sm_b200.build --trace
    python -m tiled_attention_forward_sm_b200.trace [--workload NAME] [--cta C]

The tracing library (``libattn_b200_trace.so``) is the same kernel with a
``clock64`` stamp at every hand-off between roles: the MMA warp issuing S and
the two halves of PV, each softmax group seeing S, having loaded it, having
its row maximum and publishing each half of P, and the producer issuing K
and V.  Stamps are taken for the first work item of the first 64 CTAs and
its first 72 K/V steps, into a device buffer registered with
``attn_trace_set_buffer``.  From them this module derives, per step, the
period of the S_0 -> S_0 chain and the median length of each segment; the
numbers explain where a step's time goes (see the step-time discussion of
the design notes).

Stamps are SM clock cycles of the CTA's own SM; differences within one CTA
are meaningful, across CTAs they are not.
"""
from __future__ import annotations

import argparse
import ctypes
import os
import re

import numpy as np
import torch

from .build import CSRC, TRACE_LIB, build_trace
from .inputs import WORKLOADS, make_workload_inputs

TRACE_CTAS = 64
TRACE_STEPS = 72


def event_names() -> list[str]:
    """The kernel's trace events in enum order (from its source, so the two
    cannot drift apart)."""
    src = open(os.path.join(CSRC, "attn_fwd_kernel.cuh")).read()
    body = re.search(r"enum TraceEvent : int \{(.*?)\};", src, re.S).group(1)
    names = [n.strip().split("=")[0].strip() for n in body.split(",")]
    names = [n[len("kTr"):] for n in names if n.startswith("kTr")]
    assert names[-1] == "NumEvents"
    return names[:-1]


def _library():
    path = build_trace()
    lib = ctypes.CDLL(path)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.attn_fwd.argtypes = [vp] * 5 + [i] * 5 + [f, vp]
    lib.attn_fwd.restype = i
    lib.attn_trace_set_buffer.argtypes = [vp]
    lib.attn_trace_set_buffer.restype = i
    lib.attn_last_device_error.argtypes = [vp]
    lib.attn_last_device_error.restype = i
    return lib


def record(q, k, v, causal: bool, scale: float, warmup: int = 3):
    """Run the traced kernel on CUDA bf16 [B,H,N,d] inputs; return the stamp
    array [CTA, event, step] (0 where nothing was stamped) and (o, lse)."""
    lib = _library()
    B, H, N, d = (int(x) for x in q.shape)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream

    def run():
        rc = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          B, H, N, d, int(bool(causal)), float(scale), stream)
        if rc != 0:
            raise RuntimeError(f"attn_fwd (trace build) returned {rc}")

    ev = event_names()
    buf = torch.zeros(TRACE_CTAS * len(ev) * TRACE_STEPS, dtype=torch.int64, device=q.device)
    for _ in range(warmup):
        run()
    if lib.attn_trace_set_buffer(ctypes.c_void_p(buf.data_ptr())) != 0:
        raise RuntimeError("attn_trace_set_buffer failed")
    run()
    torch.cuda.synchronize(q.device)
    if lib.attn_trace_set_buffer(None) != 0:
        raise RuntimeError("attn_trace_set_buffer failed")
    status = lib.attn_last_device_error(stream)
    if status != 0:
        raise RuntimeError(f"device status {status}")
    return buf.view(TRACE_CTAS, len(ev), TRACE_STEPS).cpu().numpy().astype(np.int64), (o, lse)


def segments(stamps: np.ndarray, cta: int) -> dict:
    """Median length (clk) of each segment of one CTA's steady state."""
    ev = {n: i for i, n in enumerate(event_names())}
    t = stamps[cta]
    s0 = t[ev["MmaS0"]]
    n = int((s0 > 0).sum())
    js = range(2, n - 2)
    if n < 6:
        return {"steps": n}

    def med(a, b, shift=0):
        return int(np.median([t[ev[b]][j + shift] - t[ev[a]][j] for j in js]))

    return {
        "steps": n,
        "period S0 -> S0": int(np.median(np.diff(s0[:n])[2:])),
        "S0 issue -> softmax 0 sees S": med("MmaS0", "Sm0Full"),
        "softmax 0: S loaded": med("Sm0Full", "Sm0Ld"),
        "softmax 0: row max": med("Sm0Ld", "Sm0Max"),
        "softmax 0: first P half": med("Sm0Max", "Sm0Pa"),
        "softmax 0: second P half": med("Sm0Pa", "Sm0Pb"),
        "first P half -> PV0 issued": med("Sm0Pa", "MmaPV0a"),
        "S0 issue (8 MMAs)": med("MmaS0", "MmaS0end"),
        "group 1 lag (sees S1 - sees S0)": med("Sm0Full", "Sm1Full"),
        "softmax 1: sees S -> second P half": med("Sm1Full", "Sm1Pb"),
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="b2h32n8192d128_causal", choices=sorted(WORKLOADS))
    ap.add_argument("--cta", type=int, default=0)
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    q, k, v = (t.cuda() for t in make_workload_inputs(w))
    stamps, _ = record(q, k, v, w.causal, w.scale)
    print(f"{TRACE_LIB}: workload {w.name}, CTA {args.cta}")
    for key, val in segments(stamps, args.cta).items():
        print(f"  {key:32s} {val}")


if __name__ == "__main__":
    main()
