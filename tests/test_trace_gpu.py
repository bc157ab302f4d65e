"""The tracing build: its stamps follow each step's hand-off order, and the
stamps do not change the arithmetic (the traced kernel's output equals the
product library's bitwise)."""
import numpy as np
import pytest
import torch

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200 import trace
from tiled_attention_forward_sm_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


def test_trace_orders_the_hand_offs_and_leaves_results_unchanged():
    B, H, N, d = 1, 16, 4096, 128
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, 2100))
    stamps, (o, lse) = trace.record(q, k, v, True, d ** -0.5)
    o_ref, l_ref = tab.attn_fwd(q, k, v, causal=True)
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    ev = {n: i for i, n in enumerate(trace.event_names())}
    t = stamps[0]
    n = int((t[ev["MmaS0"]] > 0).sum())
    assert n >= 8
    for j in range(1, n - 1):
        chain = [t[ev[e]][j] for e in ("MmaS0", "Sm0Full", "Sm0Ld", "Sm0Max", "Sm0Pa", "Sm0Pb")]
        assert all(a < b for a, b in zip(chain, chain[1:])), (j, chain)
        assert t[ev["Sm0Pa"]][j] < t[ev["MmaPV0a"]][j] < t[ev["MmaS0"]][j + 1]
    seg = trace.segments(stamps, 0)
    assert seg["period S0 -> S0"] > 0
