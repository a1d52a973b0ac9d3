"""Device copies of a synthetic hybrid batch, run through the C ABI.

Marshalling only: torch allocates the device tensors (Q, the paged K/V pools,
block table, lengths, outputs, workspace) and the calls go through the
binding's Plan; there is no attention arithmetic here.  Used by the tests,
``bench.py`` and ``__graft_entry__.smoke()``."""
from __future__ import annotations

import numpy as np


def bits_to_bf16(torch, a: np.ndarray, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.view(torch.bfloat16).to(device)


class _LayoutBatch:
    """Host-side description of a batch whose values live only on the GPU."""

    def __init__(self, w, lay):
        self.workload = w
        self.kv_lens = lay.kv_lens
        self.block_table = lay.block_table
        self.num_blocks = lay.num_blocks
        self.scale = w.softmax_scale
        self.prefill_len = w.prefill_len
        self.prefill_ctx = w.prefill_ctx
        self.num_prefill = w.num_prefill
        self.prefill_qo_lens = [P for P, _ in w.prefill_requests]
        self.prefill_kv_lens = [int(x) for x in lay.kv_lens[:w.num_prefill]]

    @property
    def decode_lens(self):
        return self.kv_lens[self.num_prefill:]


class DeviceBatch:
    @classmethod
    def generated_on_device(cls, torch, w, device="cuda"):
        """Same lengths, block layout and poison as synth.make_batch, but the
        normal values are drawn on the GPU by torch.Generator(seed) (for large
        performance-only batches; the values differ from the NumPy recipe)."""
        import synth
        lay = synth.make_layout(w)
        gen = torch.Generator(device=device)
        gen.manual_seed(w.seed)
        Hq, Hkv, d, P, B = w.num_q_heads, w.num_kv_heads, w.head_dim, w.prefill_rows, w.num_decode

        def normal(*shape):
            return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)

        self = cls.__new__(cls)
        self.b = _LayoutBatch(w, lay)
        self.torch = torch
        self.q_pre = normal(P, Hq, d) if P else None
        self.q_dec = normal(B, Hq, d) if B else None
        self.k = normal(lay.num_blocks, Hkv, synth.PAGE, d)
        self.v = normal(lay.num_blocks, Hkv, synth.PAGE, d)
        for r, L in enumerate(lay.kv_lens.tolist()):
            n = (L + synth.PAGE - 1) // synth.PAGE
            if n and L % synth.PAGE:
                blk = int(lay.block_table[r, n - 1])
                self.k[blk, :, L % synth.PAGE:, :] = synth.POISON_K
                self.v[blk, :, L % synth.PAGE:, :] = synth.POISON_V
        for blk in lay.unused_blocks.tolist():
            self.k[blk] = synth.POISON_K
            self.v[blk] = synth.POISON_V
        self.bt = torch.from_numpy(lay.block_table).to(device)
        self.lens = torch.from_numpy(lay.kv_lens).to(device)
        self.o_pre = torch.empty_like(self.q_pre) if self.q_pre is not None else None
        self.o_dec = torch.empty_like(self.q_dec) if self.q_dec is not None else None
        return self

    def __init__(self, torch, b, device="cuda"):
        self.b = b
        w = b.workload
        self.torch = torch
        self.q_pre = bits_to_bf16(torch, b.q_prefill, device) if w.prefill_rows else None
        self.q_dec = bits_to_bf16(torch, b.q_decode, device) if w.num_decode else None
        self.k = bits_to_bf16(torch, b.k_pool, device)
        self.v = bits_to_bf16(torch, b.v_pool, device)
        self.bt = torch.from_numpy(b.block_table).to(device)
        self.lens = torch.from_numpy(b.kv_lens).to(device)
        self.o_pre = torch.empty_like(self.q_pre) if self.q_pre is not None else None
        self.o_dec = torch.empty_like(self.q_dec) if self.q_dec is not None else None

    def plan(self, pod, **kw):
        w = self.b.workload
        if w.prefill_reqs is not None:   # several prefill requests: the batched planner
            return pod.Plan(w.num_q_heads, w.num_kv_heads, w.head_dim, self.b.prefill_qo_lens,
                            self.b.prefill_kv_lens, self.b.decode_lens, **kw)
        P, C = w.prefill_len, w.prefill_ctx
        return pod.Plan(w.num_q_heads, w.num_kv_heads, w.head_dim, P, C + P, self.b.decode_lens, **kw)

    def workspace(self, plan):
        return self.torch.zeros(max(plan.workspace_bytes, 256), dtype=self.torch.uint8, device=self.k.device)

    def run(self, pod, plan, ws, trace=None, stream=None):
        plan.run(self.q_pre, self.q_dec, self.k, self.v, self.b.num_blocks, self.bt, self.bt.shape[1], self.lens,
                 self.b.scale, self.o_pre, self.o_dec, ws, trace=trace, stream=stream)

    def outputs(self):
        op = self.o_pre.float().cpu().numpy().astype(np.float64) if self.o_pre is not None else None
        od = self.o_dec.float().cpu().numpy().astype(np.float64) if self.o_dec is not None else None
        return op, od

    # ------------------------------------------------------------ e4m3 cache
    def attach_fp8(self, cache, device=None):
        """Device copies of an e4m3 cache made on the host (synth.fp8_cache)."""
        dev = self.k.device if device is None else device
        t = self.torch
        self.k8 = t.from_numpy(cache.k_pool).to(dev)
        self.v8 = t.from_numpy(cache.v_pool).to(dev)
        self.k_scale = t.from_numpy(cache.k_scale).to(dev)
        self.v_scale = t.from_numpy(cache.v_scale).to(dev)
        return self

    def fp8_on_device(self):
        """An e4m3 copy of the device pools made on the GPU (large batches): per kv head,
        scale = largest |value| outside the poison / 448; codes = the value / scale, clamped to
        +-448 and converted by torch (round to nearest even); poison slots get +448 (K) and
        -448 (V).  Input preparation only; the kernel sees nothing but the codes and scales."""
        import synth
        t = self.torch
        out = []
        for pool, poison, code in ((self.k, synth.POISON_K, synth.POISON_E4M3_K),
                                   (self.v, synth.POISON_V, synth.POISON_E4M3_V)):
            f = pool.float()
            bad = f == poison
            amax = t.where(bad, t.zeros_like(f), f.abs()).amax(dim=(0, 2, 3))
            scale = (amax / synth.E4M3_MAX).clamp_min(1e-8).to(t.float32)
            q = (f / scale[None, :, None, None]).clamp(-synth.E4M3_MAX, synth.E4M3_MAX)
            q = q.to(t.float8_e4m3fn).view(t.uint8)
            q[bad] = code
            out.append((q.contiguous(), scale))
            del f, bad
        (self.k8, self.k_scale), (self.v8, self.v_scale) = out
        return self

    def run_fp8(self, pod, plan, ws, trace=None, stream=None):
        """pod_attn_run_fp8kv: decodes read the e4m3 copy (same block table), prefill the bf16 pools."""
        plan.run_fp8kv(self.q_pre, self.q_dec, self.k, self.v, self.b.num_blocks, self.k8, self.v8,
                       self.k8.shape[0], self.k_scale, self.v_scale, self.bt, self.bt.shape[1], self.lens,
                       self.b.scale, self.o_pre, self.o_dec, ws, trace=trace, stream=stream)

    def error_word(self, plan, ws):
        off = plan.info.error_offset
        return int(ws[off:off + 4].view(self.torch.int32).item())
