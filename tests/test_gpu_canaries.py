"""Out-of-bounds write detection without a sanitizer: every device buffer the
library writes (the bound cache, the decode workspace, the outputs, the regrade
scratch, the dequantize outputs) is surrounded by 1 MiB guard regions holding a
seeded byte pattern, the whole path runs -- appends through the tail into the
pages, decode of every sequence and layer, prefill on both paths, dequantize and a
VBR regrade -- and every guard must come back unchanged.  Workloads: the VBR mix
(F16 and block layers, `_1` codecs, a tail, GQA 6), the per-head projection, and
the batched KVarN case (ragged lengths, tail).
"""
import numpy as np
import pytest
import torch

from quantized_kv_cache_15_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu

GUARD = 1 << 20


class Guarded:
    """A device buffer of `nbytes` (256-byte aligned) between two guard regions."""

    def __init__(self, nbytes, seed):
        g = torch.Generator().manual_seed(seed)
        self.buf = torch.empty(GUARD + nbytes + 256 + GUARD, dtype=torch.uint8, device="cuda")
        self.off = GUARD + (-(self.buf.data_ptr() + GUARD)) % 256
        self.n = nbytes
        pat = torch.randint(0, 256, (self.buf.numel(),), dtype=torch.uint8, generator=g)
        self.buf.copy_(pat.cuda())
        self.lo = self.buf[:self.off].clone()
        self.hi = self.buf[self.off + nbytes:].clone()

    def view(self, dtype=torch.uint8, shape=None):
        v = self.buf[self.off:self.off + self.n]
        if dtype != torch.uint8:
            v = v.view(dtype)
        return v if shape is None else v.view(*shape)

    def intact(self):
        return torch.equal(self.buf[:self.off], self.lo) and torch.equal(self.buf[self.off + self.n:], self.hi)


@pytest.mark.parametrize("cfg", [3, 4, 5])
def test_no_write_leaves_its_buffer(cfg):
    w = W.make_workload(cfg, "small")
    plan = H.make_plan(w)
    cache = Guarded(plan.cache_bytes(), 1)
    plan.bind(cache.view())
    H.fill(plan, w, chunk=300)
    torch.cuda.synchronize()
    guards = {"cache": cache}
    nseq = w.batch
    ws = Guarded(max(plan.workspace_bytes(max(nseq, 256)), 16), 2)
    ws.view().zero_()
    guards["workspace"] = ws
    out = Guarded(nseq * w.n_q_heads * 128 * 4, 3)
    guards["decode out"] = out
    for layer in range(w.n_layers):
        q = torch.stack([w.queries(layer, s, 0, "cuda") for s in range(nseq)]).contiguous()
        plan.decode(layer, list(range(nseq)), q, out.view(torch.float32, (nseq, w.n_q_heads, 128)), ws.view())
    seq = int(np.argmax(w.ctx))
    n_q = min(w.ctx[seq], 200)
    pq = torch.stack([w.queries(w.n_layers - 1, seq, i, "cuda") for i in range(n_q)]).contiguous()
    for path in (0, 1):
        plan.debug_set_prefill_path(path)
        pout = Guarded(n_q * w.n_q_heads * 128 * 4, 10 + path)
        guards[f"prefill out (path {path})"] = pout
        for layer in range(w.n_layers):
            plan.prefill(layer, seq, pq, pout.view(torch.float32, (n_q, w.n_q_heads, 128)), ws.view())
    plan.debug_set_prefill_path(0)
    n = w.ctx[seq]
    dk = Guarded(n * w.n_kv_heads * 128 * 4, 20)
    dv = Guarded(n * w.n_kv_heads * 128 * 4, 21)
    guards["dequantize K"], guards["dequantize V"] = dk, dv
    plan.dequantize(0, seq, 0, n, dk.view(torch.float32), dv.view(torch.float32))
    if w.rot != W.ROT_PROJECTION:
        layer = w.n_layers - 1
        nk = [W.Q2_0 if c != W.F16 else W.F16 for c in w.k_codec[layer]]
        nv = [W.Q2_1 if c != W.F16 else W.F16 for c in w.v_codec[layer]]
        sc = Guarded(max(plan.regrade_bytes(layer, nk, nv), 16), 30)
        guards["regrade scratch"] = sc
        plan.regrade(layer, nk, nv, sc.view())
        q = torch.stack([w.queries(layer, s, 0, "cuda") for s in range(nseq)]).contiguous()
        plan.decode(layer, list(range(nseq)), q, out.view(torch.float32, (nseq, w.n_q_heads, 128)), ws.view())
    torch.cuda.synchronize()
    plan.check_device_error()
    broken = [k for k, g in guards.items() if not g.intact()]
    assert not broken, broken
