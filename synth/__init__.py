"""Seeded synthetic hybrid batches (one prefill chunk + many decode requests).

This module only draws random inputs and lays them out the way the paged KV
cache is stored; it holds none of the attention arithmetic, so both the CPU
oracle (``oracle/``) and the CUDA path (through its tests and ``bench.py``) can
take their inputs from it without sharing any of the method's code.

Workload shapes follow the POD-Attention explainer ("The evaluation": Llama-3-8B
shapes, contexts 4K-20K, prefill chunks 512-2K) and the paged KV-cache layout of
the blog post "Prefill vs. Decode GPU Utilization Imbalance" (section "How the
KV cache turns the memory-bandwidth constraint into a capacity crisis": a
token's cache entry is K and V for every layer and kv head).

Recipe (every config):
  rng = numpy.random.default_rng(seed); draws in this order:
    1. decode lengths (fixed list, integer uniform with inclusive bounds, or
       lognormal: clip(round_half_even(exp(ln(median) + sigma * z)), lo, hi));
    2. block permutation rng.permutation(num_blocks); the prefill requests
       (one by default: request 0, kv_len = C + P; a batched workload lists
       several (P_i, C_i), rows 0..NP-1) take the first pages, then decodes in
       order; EXTRA_BLOCKS trailing blocks stay unreferenced;
    3. Q_prefill [sum P_i, Hq, d] (the requests' rows one after another);
    4. Q_decode [B, Hq, d];
    5. K pool [num_blocks, Hkv, 16, d]; 6. V pool (same shape);
  values are float32 standard normals drawn in chunks of CHUNK elements and
  rounded to bf16 (round to nearest even).  Slots past a request's length in its
  last page and every unreferenced block hold finite poison (K = +30, V = -30),
  so a kernel that fails to mask them lands far outside tolerance.  Block-table
  entries past a request's last page point at an unreferenced (poison) block.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

PAGE = 16
EXTRA_BLOCKS = 2
POISON_K = 30.0
POISON_V = -30.0
CHUNK = 1 << 24


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (uint16), round to nearest, ties to even.

    Inputs are finite normals or poison constants, so no NaN/Inf handling."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit pattern (uint16) -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


E4M3_MAX = 448.0


def f64_to_e4m3_bits(v: np.ndarray) -> np.ndarray:
    """float64 -> e4m3 byte (uint8): round to nearest, ties to even, saturating at +-448.

    Input generation only (the FP8 cache is made from the bf16 values); the
    decoding that both sides compute with is the format's own definition."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    # quantum of the binade: 2^(e-3) for normals (|v| >= 2^-6), 2^-9 below
    _, ex = np.frexp(np.where(a > 0, a, 1.0))           # a = f 2^ex, f in [0.5, 1)
    e = np.clip(ex - 1, -6, 8)
    quantum = np.ldexp(1.0, (e - 3).astype(np.int64))
    q = np.minimum(np.rint(a / quantum) * quantum, E4M3_MAX)
    _, qx = np.frexp(np.where(q > 0, q, 1.0))
    qe = qx - 1
    normal = q >= 2.0 ** -6
    ebits = np.where(normal, qe + 7, 0)
    mant = np.where(normal, q / np.ldexp(1.0, qe.astype(np.int64)) * 8 - 8, q / 2.0 ** -9)
    bits = (ebits.astype(np.int64) << 3) | np.rint(mant).astype(np.int64)
    bits = np.where(np.signbit(v), bits | 0x80, bits)
    return bits.astype(np.uint8)


def _normal_bf16(rng: np.random.Generator, shape: Sequence[int]) -> np.ndarray:
    n = int(np.prod(shape, dtype=np.int64))
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, CHUNK):
        e = min(n, s + CHUNK)
        out[s:e] = f32_to_bf16_bits(rng.standard_normal(e - s, dtype=np.float32))
    return out.reshape(shape)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One hybrid batch: a prefill chunk of P query tokens over C prior tokens
    (request 0) plus B single-token decode requests."""
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    prefill_len: int          # P (0 = no prefill)
    prefill_ctx: int          # C, prior context of the prefill request
    num_decode: int           # B
    lens_kind: str            # "fixed" | "uniform" | "lognormal"
    lens_args: tuple          # fixed: the lengths; uniform: (lo, hi); lognormal: (median, sigma, lo, hi)
    seed: int
    scale: Optional[float] = None   # default 1/sqrt(head_dim)
    prefill_reqs: Optional[tuple] = None   # ((P_i, C_i), ...): several prefill requests, rows 0..NP-1

    @property
    def prefill_requests(self) -> List[tuple]:
        """(P_i, C_i) per prefill request; one request (row 0, P may be 0) unless batched."""
        if self.prefill_reqs is not None:
            return [(int(P), int(C)) for P, C in self.prefill_reqs]
        return [(self.prefill_len, self.prefill_ctx)]

    @property
    def num_prefill(self) -> int:
        return len(self.prefill_requests)

    @property
    def prefill_rows(self) -> int:
        return sum(P for P, _ in self.prefill_requests)

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.head_dim)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


def _draw_lengths(rng: np.random.Generator, w: Workload) -> np.ndarray:
    B = w.num_decode
    if B == 0:
        return np.zeros(0, dtype=np.int32)
    if w.lens_kind == "fixed":
        lens = np.asarray(w.lens_args, dtype=np.int64)
        assert lens.shape == (B,)
    elif w.lens_kind == "uniform":
        lo, hi = w.lens_args
        lens = rng.integers(lo, hi, size=B, endpoint=True)
    elif w.lens_kind == "lognormal":
        median, sigma, lo, hi = w.lens_args
        z = rng.standard_normal(B)
        lens = np.clip(np.rint(np.exp(math.log(median) + sigma * z)), lo, hi)
    else:
        raise ValueError(w.lens_kind)
    return lens.astype(np.int32)


@dataclasses.dataclass
class Batch:
    workload: Workload
    q_prefill: np.ndarray     # uint16 bf16 bits [sum P_i, Hq, d]
    q_decode: np.ndarray      # uint16 bf16 bits [B, Hq, d]
    k_pool: np.ndarray        # uint16 bf16 bits [num_blocks, Hkv, 16, d]
    v_pool: np.ndarray        # uint16 bf16 bits [num_blocks, Hkv, 16, d]
    block_table: np.ndarray   # int32 [NP + B, max_pages]; rows 0..NP-1 = prefill requests
    kv_lens: np.ndarray       # int32 [NP + B]; [i] = C_i + P_i, [NP + r] = L_r
    scale: float

    @property
    def prefill_len(self) -> int:
        return self.workload.prefill_len

    @property
    def prefill_ctx(self) -> int:
        return self.workload.prefill_ctx

    @property
    def num_prefill(self) -> int:
        return self.workload.num_prefill

    @property
    def prefill_qo_lens(self) -> List[int]:
        return [P for P, _ in self.workload.prefill_requests]

    @property
    def prefill_kv_lens(self) -> List[int]:
        return [int(x) for x in self.kv_lens[:self.num_prefill]]

    @property
    def decode_lens(self) -> np.ndarray:
        return self.kv_lens[self.num_prefill:]

    @property
    def num_blocks(self) -> int:
        return self.k_pool.shape[0]


@dataclasses.dataclass
class Layout:
    """Lengths and paged-block layout of a batch (draws 1 and 2 of the recipe)."""
    kv_lens: np.ndarray       # int32 [NP + B]
    block_table: np.ndarray   # int32 [NP + B, max_pages]
    num_blocks: int
    unused_blocks: np.ndarray # blocks no request references (poison)


def make_layout(w: Workload, rng: Optional[np.random.Generator] = None) -> Layout:
    B = w.num_decode
    rng = np.random.default_rng(w.seed) if rng is None else rng
    dec = _draw_lengths(rng, w)
    pre = [C + P if P > 0 else 0 for P, C in w.prefill_requests]
    kv_lens = np.concatenate([np.asarray(pre, dtype=np.int32), dec]).astype(np.int32)
    pages = (kv_lens.astype(np.int64) + PAGE - 1) // PAGE
    used = int(pages.sum())
    num_blocks = used + EXTRA_BLOCKS
    perm = rng.permutation(num_blocks).astype(np.int32)
    poison_block = int(perm[used])
    max_pages = max(1, int(pages.max()) if pages.size else 1)
    R = len(pre) + B
    bt = np.full((R, max_pages), poison_block, dtype=np.int32)
    off = 0
    for r in range(R):
        n = int(pages[r])
        bt[r, :n] = perm[off:off + n]
        off += n
    return Layout(kv_lens, bt, num_blocks, perm[used:])


def make_batch(w: Workload) -> Batch:
    Hq, Hkv, d = w.num_q_heads, w.num_kv_heads, w.head_dim
    P, B = w.prefill_rows, w.num_decode
    rng = np.random.default_rng(w.seed)
    lay = make_layout(w, rng)
    kv_lens, bt, num_blocks = lay.kv_lens, lay.block_table, lay.num_blocks
    pages = (kv_lens.astype(np.int64) + PAGE - 1) // PAGE
    used = int(pages.sum())
    perm_unused = lay.unused_blocks
    q_pre = _normal_bf16(rng, (P, Hq, d))
    q_dec = _normal_bf16(rng, (B, Hq, d))
    k_pool = _normal_bf16(rng, (num_blocks, Hkv, PAGE, d))
    v_pool = _normal_bf16(rng, (num_blocks, Hkv, PAGE, d))
    pk = f32_to_bf16_bits(np.float32(POISON_K)).item()
    pv = f32_to_bf16_bits(np.float32(POISON_V)).item()
    for r in range(len(kv_lens)):
        L, n = int(kv_lens[r]), int(pages[r])
        if n and L % PAGE:
            blk = bt[r, n - 1]
            k_pool[blk, :, L % PAGE:, :] = pk
            v_pool[blk, :, L % PAGE:, :] = pv
    for blk in perm_unused:
        k_pool[blk] = pk
        v_pool[blk] = pv
    return Batch(w, q_pre, q_dec, k_pool, v_pool, bt, kv_lens, w.softmax_scale)


@dataclasses.dataclass
class Fp8Cache:
    """The same paged cache stored as e4m3 bytes with one fp32 scale per kv head for K
    and for V; read by the decode requests (block-table rows from NP on)."""
    k_pool: np.ndarray        # uint8 [num_blocks, Hkv, 16, d]
    v_pool: np.ndarray        # uint8 [num_blocks, Hkv, 16, d]
    k_scale: np.ndarray       # float32 [Hkv]
    v_scale: np.ndarray       # float32 [Hkv]


POISON_E4M3_K = 0x7E          # +448: unused slots and blocks, as in the bf16 pools
POISON_E4M3_V = 0xFE          # -448


def fp8_cache(b: Batch) -> Fp8Cache:
    """Quantise a batch's K/V pools to e4m3 (no random draws: derived from the bf16 values).

    Scale of kv head h = (largest |value| of that head's pool outside the poison) / 448,
    rounded to float32; bytes = RNE(value / scale) saturated at 448; poison slots and
    blocks hold +448 (K) and -448 (V)."""
    out = []
    for pool, poison_bf16, poison8 in ((b.k_pool, POISON_K, POISON_E4M3_K), (b.v_pool, POISON_V, POISON_E4M3_V)):
        f = bf16_bits_to_f32(pool).astype(np.float64)
        is_poison = f == poison_bf16
        amax = np.where(is_poison, 0.0, np.abs(f)).max(axis=(0, 2, 3))
        scale = np.maximum(amax / E4M3_MAX, 1e-8).astype(np.float32)
        q = np.empty(pool.shape, dtype=np.uint8)
        for h in range(pool.shape[1]):
            q[:, h] = f64_to_e4m3_bits(f[:, h] / np.float64(scale[h]))
        q[is_poison] = poison8
        out.append((q, scale))
    return Fp8Cache(out[0][0], out[1][0], out[0][1], out[1][1])


# ---------------------------------------------------------------------------
# Named workloads (shapes of the POD-Attention evaluation; seeds fixed).
# ---------------------------------------------------------------------------

def tiny(seed: int = 0) -> Workload:
    """1 prefill chunk of 64 tokens over 128 prior + 4 decodes {64,100,180,256};
    4 q heads / 2 kv heads, head_dim 64, scale 1/8."""
    return Workload("tiny", 4, 2, 64, 64, 128, 4, "fixed", (64, 100, 180, 256), seed, 1.0 / 8.0)


def llama3_8b_mix(seed: int = 1) -> Workload:
    """Llama-3-8B layer: 32/8 heads, d=128; prefill 512 over 4096; 64 decodes U[1024,4096]."""
    return Workload("llama3_8b_mix", 32, 8, 128, 512, 4096, 64, "uniform", (1024, 4096), seed)


def long_context_mix(seed: int = 2) -> Workload:
    """32/8 heads, d=128; prefill 1024 over 12288; 128 decodes U[8192,16384]."""
    return Workload("long_context_mix", 32, 8, 128, 1024, 12288, 128, "uniform", (8192, 16384), seed)


def decode_heavy_mix(seed: int = 3) -> Workload:
    """32/8 heads, d=128; prefill 256 over 2048; 256 decodes lognormal(2048, 1.0) in [16, 32768]."""
    return Workload("decode_heavy_mix", 32, 8, 128, 256, 2048, 256, "lognormal", (2048, 1.0, 16, 32768), seed)


def sweep(prefill_len: int, num_decode: int, ctx: int, seed: int, prior: int = 4096) -> Workload:
    """Mix sweep point: 32/8 heads, d=128; prefill chunk over `prior` prior tokens;
    decode lengths uniform within +-25% of ctx (bounds rounded half-even)."""
    lo, hi = int(round(0.75 * ctx)), int(round(1.25 * ctx))
    return Workload(f"sweep_p{prefill_len}_b{num_decode}_c{ctx}", 32, 8, 128, prefill_len,
                    prior if prefill_len > 0 else 0, num_decode, "uniform", (lo, hi), seed)


def sweep_points() -> List[Workload]:
    pts = []
    seed = 10
    for P in (512, 1024, 2048):
        for B in (16, 64, 256):
            for ctx in (4096, 16384):
                pts.append(sweep(P, B, ctx, seed))
                seed += 1
    pts.append(sweep(1024, 0, 4096, seed))            # prefill only
    pts.append(sweep(0, 64, 4096, seed + 1))          # decode only
    return pts


def batched_llama3_8b_mix(seed: int = 4) -> Workload:
    """Batched hybrid batch: three prefill chunks (512 over 3584, 512 over 1536,
    256 over 0 prior tokens) + 64 decodes U[1024,4096]; 32/8 heads, d=128."""
    return Workload("batched_llama3_8b_mix", 32, 8, 128, 0, 0, 64, "uniform", (1024, 4096), seed,
                    prefill_reqs=((512, 3584), (512, 1536), (256, 0)))


NAMED = {
    "tiny": tiny,
    "llama3_8b_mix": llama3_8b_mix,
    "long_context_mix": long_context_mix,
    "decode_heavy_mix": decode_heavy_mix,
    "batched_llama3_8b_mix": batched_llama3_8b_mix,
}


def custom(name: str, Hq: int, Hkv: int, d: int, P: int, C: int, lens: Sequence[int], seed: int,
           scale: Optional[float] = None) -> Workload:
    """Small hand-sized batch (fixed decode lengths) for edge-case tests."""
    return Workload(name, Hq, Hkv, d, P, C if P > 0 else 0, len(lens), "fixed", tuple(int(x) for x in lens), seed, scale)


def custom_batched(name: str, Hq: int, Hkv: int, d: int, prefill_reqs: Sequence[tuple], lens: Sequence[int],
                   seed: int, scale: Optional[float] = None) -> Workload:
    """Small batched hybrid batch: prefill requests ((P_i, C_i), ...) in rows
    0..NP-1, fixed decode lengths after them."""
    return Workload(name, Hq, Hkv, d, 0, 0, len(lens), "fixed", tuple(int(x) for x in lens), seed, scale,
                    prefill_reqs=tuple((int(P), int(C)) for P, C in prefill_reqs))
