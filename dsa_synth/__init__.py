"""Seeded synthetic inputs for the DSA forward path.

This module is the ONLY code shared by the CUDA path's tests/benchmark and the fp64
oracle.  It draws random numbers and lays them out; it contains none of the method's
arithmetic (no scores, no selection, no attention).  The FP8 quantisation below is
input preparation: the FP8 indexer consumes e4m3 codes plus per-token scales that
arrive already quantised.

Workloads (shapes from the pages: 64 indexer heads x 128, index_topk 2048, 128 MLA
heads over a 576-d latent = 512 KV-LoRA + 64 RoPE, value = first 512 dims):

  ``pr_ref_256``       L=256 prefill, topk 64, q_I,k_I ~ N(0,1), w ~ N(0,1)/8,
                       q, kv ~ N(0,1)/sqrt(576)
  ``prefill_2k``       L=2048 prefill, topk 2048 (every causal key is selected: short sequence)
  ``prefill_4k``       L=4096 prefill, topk 2048, structured keys (below), q, kv ~ N(0,1)
  ``prefill_32k``      L=32768, otherwise as prefill_4k (the headline workload)
  ``decode_b64``       64 sequences, one query each, context ~ U[8192, 65536]
  ``prefill_128k_fp8`` L=131072, indexer inputs quantised to e4m3 with per-token scales

Structured keys: k_I = N(0,1) + Z @ B with Z [S,16] ~ N(0,1), B [16,128] ~ N(0,1)/4,
a rank-16 component shared by all keys so that index scores have structure.

Draw order per workload is fixed: q_I, k_I noise, Z, B, w, q, kv (decode: the context
lengths first).  All draws are float32 normals from one ``torch.Generator`` seeded with
``seed`` on ``device``, then rounded to the storage dtype.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Optional

import torch

N_IDX_HEADS = 64
IDX_DIM = 128
N_HEADS = 128
D_QK = 576
D_V = 512
SM_SCALE = 1.0 / (192.0 ** 0.5)   # 128 NoPE + 64 RoPE dims per query/key head
E4M3_MAX = 448.0


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill" or "decode"
    seq_len: int = 0          # prefill: L (queries = keys = L)
    batch: int = 1
    ctx_min: int = 0          # decode: context length range (inclusive)
    ctx_max: int = 0
    topk: int = 2048
    structured_keys: bool = True
    latent_std: float = 1.0   # std of q and kv entries
    fp8_indexer: bool = False
    chunk: int = 0            # queries per indexer/top-k chunk in the fused forward


WORKLOADS: Dict[str, Workload] = {
    "pr_ref_256": Workload("pr_ref_256", "prefill", seq_len=256, topk=64, structured_keys=False,
                           latent_std=1.0 / 24.0),
    "prefill_2k": Workload("prefill_2k", "prefill", seq_len=2048),
    "prefill_4k": Workload("prefill_4k", "prefill", seq_len=4096),
    "prefill_32k": Workload("prefill_32k", "prefill", seq_len=32768, chunk=8192),
    "decode_b64": Workload("decode_b64", "decode", batch=64, ctx_min=8192, ctx_max=65536),
    "prefill_128k_fp8": Workload("prefill_128k_fp8", "prefill", seq_len=131072, fp8_indexer=True,
                                 chunk=4096),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(g, shape, device, std=1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x


def quantize_e4m3_per_token(x: torch.Tensor):
    """Per-token e4m3 codes: scale[t] = amax(|x[t]|)/448 (1 if the row is 0), codes =
    round-to-nearest-even(x / scale) saturated to +-448.  Returns (codes uint8, scale f32)."""
    flat = x.reshape(x.shape[0], -1).float()
    amax = flat.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (flat / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(x.shape)
    return codes.contiguous(), scale.contiguous()


def quantize_e4m3_ue8m0_blocks(x: torch.Tensor):
    """Block-scaled e4m3 codes: one scale per 128-element block along the last dimension,
    a power of two stored as a ue8m0 byte (exponent + 127), the smallest power of two not
    below amax / 448 (so no code saturates); codes = round-to-nearest-even(x / scale).
    For q_I [T, H, 128] a block is one head of one token, for k_I [S, 128] one token.
    Returns (codes uint8 like x, scale bytes uint8 [..., blocks])."""
    assert x.shape[-1] % 128 == 0
    blocks = x.float().reshape(*x.shape[:-1], x.shape[-1] // 128, 128)
    amax = blocks.abs().amax(dim=-1)
    e = torch.ceil(torch.log2(torch.clamp(amax / E4M3_MAX, min=2.0 ** -126))).clamp_(-127, 127)
    scale = torch.exp2(e)
    y = (blocks / scale[..., None]).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(x.shape)
    sbytes = (e + 127).to(torch.uint8)
    if x.shape[-1] == 128:
        sbytes = sbytes[..., 0]
    return codes.contiguous(), sbytes.contiguous()


def make_prefill(L: int, topk: int = 2048, seed: int = 0, device="cpu", structured_keys: bool = True,
                 latent_std: float = 1.0, fp8_indexer: bool = False, T: Optional[int] = None,
                 with_latent: bool = True, fp8_blocks: bool = False):
    """One sequence of L tokens.  T (default L) queries are the last T tokens.

    ``with_latent=False`` skips the last draws (q, kv) and leaves the indexer inputs
    unchanged, for runs that only need the indexer side."""
    T = L if T is None else T
    g = _gen(seed, device)
    q_idx = _randn(g, (T, N_IDX_HEADS, IDX_DIM), device)
    k_idx = _randn(g, (L, IDX_DIM), device)
    if structured_keys:
        Z = _randn(g, (L, 16), device)
        B = _randn(g, (16, IDX_DIM), device, std=0.25)
        k_idx += Z @ B
    w = _randn(g, (T, N_IDX_HEADS), device, std=0.125)
    out = {}
    if with_latent:
        out["q"] = _randn(g, (T, N_HEADS, D_QK), device, std=latent_std).to(torch.bfloat16).contiguous()
        out["kv"] = _randn(g, (L, D_QK), device, std=latent_std).to(torch.bfloat16).contiguous()
    out.update(w=w.contiguous(), topk=topk,
               cu_q=torch.tensor([0, T], dtype=torch.int32, device=device),
               cu_k=torch.tensor([0, L], dtype=torch.int32, device=device),
               total_q=T, total_k=L, max_len_q=T, max_len_k=L, batch=1)
    if fp8_blocks:
        out["q_idx8"], out["q_scale_ue8m0"] = quantize_e4m3_ue8m0_blocks(q_idx)
        out["k_idx8"], out["k_scale_ue8m0"] = quantize_e4m3_ue8m0_blocks(k_idx)
    elif fp8_indexer:
        out["q_idx8"], out["q_scale"] = quantize_e4m3_per_token(q_idx)
        out["k_idx8"], out["k_scale"] = quantize_e4m3_per_token(k_idx)
    else:
        out["q_idx"] = q_idx.to(torch.bfloat16).contiguous()
        out["k_idx"] = k_idx.to(torch.bfloat16).contiguous()
    return out


def make_decode(batch: int, ctx_min: int, ctx_max: int, topk: int = 2048, seed: int = 0,
                device="cpu", structured_keys: bool = True, latent_std: float = 1.0, q_per_seq: int = 1):
    """``batch`` sequences with cached keys; ``q_per_seq`` new query tokens each (the last ones)."""
    g = _gen(seed, device)
    lens = torch.randint(ctx_min, ctx_max + 1, (batch,), generator=g, device=device, dtype=torch.int64)
    lens_cpu = lens.cpu()
    cu_k = torch.zeros(batch + 1, dtype=torch.int64)
    cu_k[1:] = torch.cumsum(lens_cpu, 0)
    S = int(cu_k[-1])
    T = batch * q_per_seq
    q_idx = _randn(g, (T, N_IDX_HEADS, IDX_DIM), device)
    k_idx = _randn(g, (S, IDX_DIM), device)
    if structured_keys:
        Z = _randn(g, (S, 16), device)
        B = _randn(g, (16, IDX_DIM), device, std=0.25)
        k_idx += Z @ B
    w = _randn(g, (T, N_IDX_HEADS), device, std=0.125)
    q = _randn(g, (T, N_HEADS, D_QK), device, std=latent_std).to(torch.bfloat16)
    kv = _randn(g, (S, D_QK), device, std=latent_std).to(torch.bfloat16)
    cu_q = torch.arange(0, T + 1, q_per_seq, dtype=torch.int32)
    return dict(q_idx=q_idx.to(torch.bfloat16).contiguous(), k_idx=k_idx.to(torch.bfloat16).contiguous(),
                w=w.contiguous(), q=q.contiguous(), kv=kv.contiguous(), topk=topk,
                cu_q=cu_q.to(device), cu_k=cu_k.to(torch.int32).to(device),
                total_q=T, total_k=S, max_len_q=q_per_seq, max_len_k=int(lens_cpu.max()), batch=batch)


def to_paged(inp: dict, page_size: int = 64, seed: int = 0, spare_pages: int = 3) -> dict:
    """The same problem with its key-side caches (k_idx / k_idx8 + k_scale, kv) laid out in
    pages of ``page_size`` rows placed in a seeded random order, plus the block table
    [B, max_pages] int32 that maps logical page j of sequence b to its physical page (-1 for
    unused entries).  ``spare_pages`` unused pages (filled with noise) are mixed in, so no
    sequence's pages are contiguous by accident.  Values are copied, never changed."""
    cu_k = inp["cu_k"].cpu().tolist()
    B = len(cu_k) - 1
    lens = [cu_k[b + 1] - cu_k[b] for b in range(B)]
    npages = [(n + page_size - 1) // page_size for n in lens]
    max_pages = max(1, max(npages))
    total = sum(npages) + spare_pages
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(total, generator=g)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    j = 0
    for b in range(B):
        for pg in range(npages[b]):
            table[b, pg] = int(perm[j])
            j += 1
    out = dict(inp)
    dev = inp["cu_k"].device
    for name in ("k_idx", "k_idx8", "k_scale", "kv"):
        if name not in inp:
            continue
        src = inp[name]
        shape = (total * page_size,) + tuple(src.shape[1:])
        dst = torch.zeros(shape, dtype=src.dtype, device=src.device)
        if src.dtype == torch.float32:
            dst.normal_(generator=torch.Generator(device=src.device).manual_seed(seed + 1))
        for b in range(B):
            for pg in range(npages[b]):
                r0 = cu_k[b] + pg * page_size
                n = min(page_size, cu_k[b + 1] - r0)
                d0 = int(table[b, pg]) * page_size
                dst[d0:d0 + n] = src[r0:r0 + n]
        out[name] = dst.contiguous()
    out.update(block_table=table.to(dev), page_size=page_size, max_pages=max_pages, phys_k=total * page_size)
    return out


def make_workload(name: str, seed: int = 0, device="cpu", with_latent: bool = True, **overrides):
    wl = WORKLOADS[name]
    if wl.kind == "decode":
        return make_decode(wl.batch, overrides.get("ctx_min", wl.ctx_min), overrides.get("ctx_max", wl.ctx_max),
                           topk=wl.topk, seed=seed, device=device, structured_keys=wl.structured_keys,
                           latent_std=wl.latent_std)
    return make_prefill(overrides.get("L", wl.seq_len), topk=wl.topk, seed=seed, device=device,
                        structured_keys=wl.structured_keys, latent_std=wl.latent_std,
                        fp8_indexer=wl.fp8_indexer, with_latent=with_latent)
