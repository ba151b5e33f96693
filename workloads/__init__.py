"""Seeded synthetic inputs for the DeepSeek Sparse Attention (DSA) hot path.

This module is shared by the CPU oracle (tests) and the CUDA path (tests,
bench). It draws random numbers and encodes them into the cache formats the
method consumes, and nothing else: it holds none of the method's arithmetic
(no dot products, no selection, no softmax).

Workloads follow the pages' description of the two DSA caches:
  * indexer key cache: 128 values per token, FP8 (page "DeepSeek-V3.2-Exp
    模型优势与 DSA 工作原理", section 3 "闪电索引器"; FP8 for the indexer:
    page "m.gxzdkb.com/media/457.html", section "秘密武器");
  * MLA latent cache: 512 values per token (same page 3, section 3 "稀疏多潜在
    注意力"), stored here as 512 latent + 64 rope dims in bf16.

FP8 encoding of a float tensor is per token: scale = amax / 448 over the
token's values (1 when amax = 0), code = e4m3(x / scale) with torch's
round-to-nearest-even cast after clamping to +-448.

Every generator takes a seed and a device. The same seed on the same device
type gives the same tensors; CPU and CUDA generators give different streams,
so a consumer that needs the values on the host copies them there.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

D_INDEX = 128          # indexer key/query width
D_LATENT = 512         # MLA latent (value) width
D_ROPE = 64            # MLA rope width carried next to the latent
D_QK = D_LATENT + D_ROPE
BLOCK = 64             # paged cache block size (tokens per block)
FP8_MAX = 448.0


@dataclass(frozen=True)
class Config:
    """One workload shape. ``kind`` is "prefill" or "decode"."""
    cid: int
    name: str
    kind: str
    k: int
    Hi: int
    H: int
    seed: int
    # prefill
    L: int = 0
    chunk: int = 0
    # decode
    B: int = 0
    ctx: int = 0
    ctx_lo: int = 0
    ctx_hi: int = 0
    nq: int = 1
    # value recipe
    grid: bool = False          # integer FP8 grid (exact fp32 scores)
    scale: float = 1.0 / math.sqrt(D_INDEX)
    sm_scale: float = 1.0 / math.sqrt(D_QK)
    plant_block: int = 0        # queries per planting block
    plant_n: int = 0            # planted keys per block
    plant_prefix: bool = False  # planted keys drawn from the block's prefix
    extra: dict = field(default_factory=dict)


CONFIGS = {
    1: Config(1, "tiny_prefill_L1024_k256", "prefill", k=256, Hi=4, H=8, seed=0,
              L=1024, grid=True, scale=1.0 / 16, sm_scale=1.0 / 24),
    2: Config(2, "prefill_L16384_k2048", "prefill", k=2048, Hi=64, H=128, seed=1,
              L=16384, plant_block=1024, plant_n=64),
    3: Config(3, "decode_B64_ctx32768", "decode", k=2048, Hi=64, H=128, seed=2,
              B=64, ctx=32768, nq=1),
    4: Config(4, "prefill_L131072_chunk4096", "prefill", k=2048, Hi=64, H=128, seed=3,
              L=131072, chunk=4096, plant_block=4096, plant_n=32, plant_prefix=True),
    5: Config(5, "decode_varlen_B128_nq2", "decode", k=2048, Hi=64, H=128, seed=4,
              B=128, ctx_lo=512, ctx_hi=131072, nq=2),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def fp8_per_token(x: torch.Tensor, token_dims: int):
    """Encode ``x`` to e4m3 bytes with one fp32 scale per token.

    ``token_dims`` trailing dims form one token (1 for a key row [.., 128],
    2 for a query [.., Hi, 128]). Returns (uint8 codes, float32 scales).
    """
    flat = x.reshape(*x.shape[: x.dim() - token_dims], -1).float()
    amax = flat.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
    y = (flat / scale.unsqueeze(-1)).clamp_(-FP8_MAX, FP8_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(x.shape)
    return codes.contiguous(), scale.float().contiguous()


def _normal(shape, g, device, dtype=torch.float32):
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(dtype)


def _plant(q: torch.Tensor, k: torch.Tensor, cfg: Config, g, device, t0q: int = 0, L: int = 0):
    """Correlate each block of queries with a few keys along a random direction.

    For block b (``plant_block`` queries), draw a unit vector u_b in R^128 and
    ``plant_n`` key positions, uniform in [0, block_end) (or in the block's
    prefix [0, block_start), the first block using [0, block_end)). Add a*u_b
    to every head of every query in the block and to each planted key, with
    a^2 = 3*sqrt(128), so a planted pair's dot product gains +3 sigma.
    ``q`` may hold only the query rows [t0q, t0q + len(q)) of an L-token
    prefill (L = 0: all rows); every block's keys are planted all the same.
    """
    L = L or q.shape[0]
    a = math.sqrt(3.0 * math.sqrt(D_INDEX))
    nblk = (L + cfg.plant_block - 1) // cfg.plant_block
    for b in range(nblk):
        t0 = b * cfg.plant_block
        t1 = min(L, t0 + cfg.plant_block)
        u = torch.randn(D_INDEX, generator=g, device=device)
        u = u / u.norm()
        hi = t0 if (cfg.plant_prefix and t0 > 0) else t1
        pos = torch.randint(0, hi, (cfg.plant_n,), generator=g, device=device)
        r0, r1 = max(t0, t0q) - t0q, min(t1, t0q + q.shape[0]) - t0q
        if r0 < r1:
            q[r0:r1] += a * u
        k.index_add_(0, pos, (a * u).expand(cfg.plant_n, D_INDEX).contiguous())


def make_prefill(cfg: Config, device="cpu", L: int | None = None, rows=None):
    """Inputs for a causal prefill of ``L`` tokens (default: the config's L).

    Returns a dict with
      q8 [L][Hi][128] uint8 (e4m3), q_scale [L] f32 or None,
      k8 [L][128] uint8 (e4m3), k_scale [L] f32 or None, w [L][Hi] f32,
      q [L][H][576] bf16, kv [L][576] bf16,
      plus scale, sm_scale, k, q_pos0 (=0), T, S.
    With ``rows`` = (t0, t1), the query-side tensors (q8, q_scale, w, q) hold
    only the rows t0 .. t1-1 of that prefill (T = t1 - t0, q_pos0 = t0) and
    the caches all L keys: the same shapes and distributions, drawn in
    another order than the whole prefill's (so not the same values).
    """
    L = cfg.L if L is None else L
    t0, t1 = rows if rows is not None else (0, L)
    T = t1 - t0
    g = _gen(cfg.seed, device)
    Hi, H = cfg.Hi, cfg.H
    if cfg.grid:
        assert rows is None, "the integer grid is drawn for whole prefills only"
        q8 = torch.randint(-8, 9, (L, Hi, D_INDEX), generator=g, device=device)
        k8 = torch.randint(-8, 9, (L, D_INDEX), generator=g, device=device)
        q8 = q8.float().to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
        k8 = k8.float().to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
        w = torch.randint(-4, 5, (L, Hi), generator=g, device=device).float() / 4.0
        q_scale = k_scale = None
    else:
        qi = _normal((T, Hi, D_INDEX), g, device)
        ki = _normal((L, D_INDEX), g, device)
        if cfg.plant_block:
            _plant(qi, ki, cfg, g, device, t0q=t0, L=L)
        q8, q_scale = fp8_per_token(qi, 2)
        k8, k_scale = fp8_per_token(ki, 1)
        del qi, ki
        w = _normal((T, Hi), g, device) / 8.0        # N(0, 1/64)
    q = _normal((T, H, D_QK), g, device, torch.bfloat16)
    kv = _normal((L, D_QK), g, device, torch.bfloat16)
    return dict(q8=q8, q_scale=q_scale, k8=k8, k_scale=k_scale, w=w.contiguous(),
                q=q.contiguous(), kv=kv.contiguous(), scale=cfg.scale,
                sm_scale=cfg.sm_scale, k=cfg.k, q_pos0=t0, T=T, S=L,
                Hi=Hi, H=H)


def decode_lengths(cfg: Config, g, device="cpu", B: int | None = None):
    B = cfg.B if B is None else B
    if cfg.ctx:
        return torch.full((B,), cfg.ctx, dtype=torch.int32)
    lo, hi = math.log(cfg.ctx_lo), math.log(cfg.ctx_hi)
    u = torch.rand(B, generator=g, device=device, dtype=torch.float64).cpu()
    lens = torch.exp(lo + (hi - lo) * u).floor().clamp_(cfg.ctx_lo, cfg.ctx_hi)
    return lens.to(torch.int32)


def make_decode(cfg: Config, device="cpu", B: int | None = None,
                lens: torch.Tensor | None = None):
    """Inputs for batched decode over a paged cache (block size 64).

    Sequence b holds ``seq_len[b]`` tokens; its ``nq`` new queries sit at
    positions seq_len-nq .. seq_len-1 (their keys are already in the cache).
    Physical blocks are a random permutation of the pool.

    Returns a dict with
      q8 [B][nq][Hi][128] u8, q_scale [B][nq] f32, w [B][nq][Hi] f32,
      q [B][nq][H][576] bf16,
      k8_pool [nblk][64][128] u8, k_scale_pool [nblk][64] f32,
      kv_pool [nblk][64][576] bf16,
      block_table [B][max_blocks] int32 (-1 past the end), seq_len [B] int32,
      plus scale, sm_scale, k, nq, B, max_blocks, nblk.
    """
    g = _gen(cfg.seed, device)
    if lens is None:
        B = cfg.B if B is None else B
        lens = decode_lengths(cfg, g, device, B)
    else:
        lens = lens.to(torch.int32).cpu()
        B = int(lens.numel())
    nq, Hi, H = cfg.nq, cfg.Hi, cfg.H
    nblocks = [(int(n) + BLOCK - 1) // BLOCK for n in lens.tolist()]
    nblk = sum(nblocks)
    max_blocks = max(nblocks)
    perm = torch.randperm(nblk, generator=g, device=device).cpu().to(torch.int32)
    table = torch.full((B, max_blocks), -1, dtype=torch.int32)
    off = 0
    for b, nb in enumerate(nblocks):
        table[b, :nb] = perm[off: off + nb]
        off += nb
    ki = _normal((nblk, BLOCK, D_INDEX), g, device)
    k8, k_scale = fp8_per_token(ki, 1)
    del ki
    kv = _normal((nblk, BLOCK, D_QK), g, device, torch.bfloat16)
    qi = _normal((B, nq, Hi, D_INDEX), g, device)
    q8, q_scale = fp8_per_token(qi, 2)
    w = _normal((B, nq, Hi), g, device) / 8.0
    q = _normal((B, nq, H, D_QK), g, device, torch.bfloat16)
    return dict(q8=q8, q_scale=q_scale, w=w.contiguous(), q=q.contiguous(),
                k8_pool=k8, k_scale_pool=k_scale, kv_pool=kv.contiguous(),
                block_table=table.to(device), seq_len=lens.to(device),
                scale=cfg.scale, sm_scale=cfg.sm_scale, k=cfg.k, nq=nq, B=B,
                max_blocks=max_blocks, nblk=nblk, Hi=Hi, H=H)


def rope_table(T: int, q_pos0: int = 0, base: float = 10000.0, device="cpu") -> torch.Tensor:
    """(cos, sin) of the rotary angles for positions q_pos0 .. q_pos0 + T - 1 and the
    64 dimension pairs of a 128-wide head: [T][64][2] float32, angle (p * base^(-i/64)
    for pair i), evaluated in float64. The projection kernel and the oracle both
    take it as input data."""
    pos = torch.arange(q_pos0, q_pos0 + T, dtype=torch.float64).unsqueeze(1)
    inv = base ** (-torch.arange(64, dtype=torch.float64) / 64.0)
    ang = pos * inv.unsqueeze(0)
    return torch.stack([ang.cos(), ang.sin()], dim=-1).float().contiguous().to(device)


def make_projection(T: int, d: int, Hi: int, seed: int, device="cpu"):
    """Hidden states h ~ N(0, 1) [T][d] and weights [Hi*128 + 128 + Hi][d] ~ N(0, 1/d),
    both bf16 (so each output is about N(0, 1)), plus the rotary table of positions 0..T-1."""
    g = torch.Generator(device=device).manual_seed(seed)
    N = Hi * D_INDEX + D_INDEX + Hi
    h = _normal((T, d), g, device, torch.bfloat16)
    wt = (torch.randn(N, d, generator=g, device=device) / math.sqrt(d)).to(torch.bfloat16)
    return dict(h=h, wt=wt, rope=rope_table(T, device=device), T=T, d=d, Hi=Hi)
