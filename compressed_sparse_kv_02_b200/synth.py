"""Seeded synthetic inputs for the CSA / HCA path (tests and benchmark).

Only random inputs live here: raw token streams, gate logits, queries,
indexer weights, and compressed caches synthesised directly in stored form
for the long-context decode workloads. Nothing here computes any step of
the method; the GPU library and the CPU oracle each take these same tensors.

Workloads (shapes and distributions of the five benchmark configurations):
  tiny     B=1, n=8192, 8 consecutive decode queries, H=16, d=128 (K=V) bf16,
           raw KV ~N(0,1)/sqrt(d), gate logits ~N(0,1), CSA m=4 top-512,
           HCA m'=128, window 128, indexer 4 heads x 64, w ~U(0,1); seed 0.
  flash    B=32, n=131072, H=32, d=128, CSA top-512, indexer 4 x 64; seed 1.
  pro      B=8, n=1048576, H=128, d_qk=576 (512 + 64 RoPE), d_v=512, CSA
           top-1024, indexer 8 x 128, 1% planted high-similarity indexer keys;
           seed 2.
  prefill  65536 new tokens on 65536 cached, H=64, d=128, indexer 4 x 64,
           top-512; seed 3.
  mixed    B=64, n log-uniform in [4096, 1048576], FP8 e4m3 KV with an fp32
           scale per entry, FP4 e2m1 indexer keys/queries with e4m3 scales per
           16, top-1024, 2 CSA + 2 HCA layers; seed 4.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Config:
    name: str
    batch: int
    ctx: int            # tokens in each stream; the decode query sits at t = ctx - 1
    heads: int
    d_qk: int
    d_v: int
    heads_idx: int
    d_idx: int
    k: int
    seed: int
    m_csa: int = 4
    m_hca: int = 128
    n_win: int = 128
    page_size: int = 64
    planted_frac: float = 0.0
    kv_dtype: str = "bf16"
    idx_dtype: str = "bf16"


CONFIGS = {
    "tiny": Config("tiny", 1, 8192, 16, 128, 128, 4, 64, 512, seed=0),
    "flash": Config("flash", 32, 131072, 32, 128, 128, 4, 64, 512, seed=1),
    "pro": Config("pro", 8, 1 << 20, 128, 576, 512, 8, 128, 1024, seed=2, planted_frac=0.01),
    "prefill": Config("prefill", 1, 131072, 64, 128, 128, 4, 64, 512, seed=3),
    "mixed": Config("mixed", 64, 1 << 20, 128, 576, 512, 8, 128, 1024, seed=4, kv_dtype="fp8", idx_dtype="fp4"),
}


def generator(seed: int, stream: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream * 7919) % (1 << 63))
    return g


def normal(shape, std: float, g: torch.Generator, device="cpu", dtype=torch.bfloat16, chunk_rows: int = 1 << 16):
    """~N(0, std^2), rounded to `dtype`, generated in row chunks to bound temporaries."""
    shape = tuple(shape)
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1, shape[-1]) if len(shape) > 1 else out.view(1, -1)
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(r0 + chunk_rows, flat.shape[0])
        flat[r0:r1] = (torch.randn((r1 - r0, flat.shape[1]), generator=g, device=device) * std).to(dtype)
    return out


def uniform(shape, lo: float, hi: float, g: torch.Generator, device="cpu"):
    return torch.rand(tuple(shape), generator=g, device=device) * (hi - lo) + lo


def raw_stream(batch: int, n: int, d: int, seed: int, stream: int, device="cpu", gate_cols=None):
    """Raw latent rows x ~N(0,1)/sqrt(d) and per-channel gate logits z ~N(0,1), both bf16."""
    gc = d if gate_cols is None else gate_cols
    x = normal((batch, n, d), 1.0 / math.sqrt(d), generator(seed, stream, device), device)
    z = normal((batch, n, gc), 1.0, generator(seed, stream + 1, device), device)
    return x, z


def decode_queries(batch: int, heads: int, d_qk: int, heads_idx: int, d_idx: int, seed: int, stream: int,
                   device="cpu", q_scale: float = 1.0):
    """Attention queries q ~N(0,1)*q_scale, indexer queries ~N(0,1) (bf16) and weights w ~U(0,1) (fp32)."""
    q = normal((batch, heads, d_qk), q_scale, generator(seed, stream, device), device)
    q_idx = normal((batch, heads_idx, d_idx), 1.0, generator(seed, stream + 1, device), device)
    w = uniform((batch, heads_idx), 0.0, 1.0, generator(seed, stream + 2, device), device)
    return q, q_idx, w


def page_permutation(n_pages: int, seed: int, stream: int, device="cpu") -> torch.Tensor:
    return torch.randperm(n_pages, generator=generator(seed, stream, "cpu")).to(torch.int32).to(device)


def planted_keys(keys: torch.Tensor, q_idx: torch.Tensor, w: torch.Tensor, frac: float, n_cand: int, seed: int,
                 stream: int) -> torch.Tensor:
    """Plant frac * n_cand of the first n_cand keys along u = unit(sum_h w_h q_h): K <- 0.5 K + 2 sqrt(d) u.

    keys [n_entries, d] of one sequence; q_idx [heads_idx, d]; w [heads_idx].
    Returns the planted entry ids.
    """
    d = keys.shape[-1]
    n_plant = int(frac * n_cand)
    if n_plant == 0:
        return torch.empty(0, dtype=torch.int64, device=keys.device)
    ids = torch.randperm(n_cand, generator=generator(seed, stream, "cpu"))[:n_plant].to(keys.device)
    u = (w.float()[:, None] * q_idx.float()).sum(0)
    u = u / u.norm()
    keys[ids] = (0.5 * keys[ids].float() + 2.0 * math.sqrt(d) * u).to(keys.dtype)
    return ids


def decode_layer_state(cfg: Config, kind: str, device="cpu", stream_base: int = 0):
    """Synthesised state of one decode layer at t = ctx - 1, all sequences.

    kind "csa" or "hca". Returns a dict of tensors:
      entries [B, E, d_qk] bf16 stored compressed entries (~N(0,1)/sqrt(d_qk)),
      idx_entries [B, E, d_idx] bf16 (CSA; ~N(0,1), planted if cfg asks),
      ring_x / ring_z (and ring_xi / ring_zi for CSA): the raw rows of positions
      t-128 .. t-1 at ring slot p % n_win,
      new_x / new_z (new_xi / new_zi): the rows of the decode token t,
      q, q_idx, w: the decode queries.
    """
    B, t = cfg.batch, cfg.ctx - 1
    m = cfg.m_csa if kind == "csa" else cfg.m_hca
    E = cfg.ctx // m
    s = cfg.seed
    base = stream_base + (0 if kind == "csa" else 100)
    out = {}
    out["entries"] = normal((B, E, cfg.d_qk), 1.0 / math.sqrt(cfg.d_qk), generator(s, base + 1, device), device)
    ring_x, ring_z = raw_stream(B, cfg.n_win, cfg.d_qk, s, base + 3, device)
    new_x, new_z = raw_stream(B, 1, cfg.d_qk, s, base + 5, device)
    q, q_idx, w = decode_queries(B, cfg.heads, cfg.d_qk, cfg.heads_idx, cfg.d_idx, s, base + 7, device)
    # ring slot of position p is p % n_win: rows generated in position order t-128 .. t-1
    slots = torch.tensor([(t - cfg.n_win + i) % cfg.n_win for i in range(cfg.n_win)], device=device)
    out["ring_x"] = torch.empty_like(ring_x)
    out["ring_x"][:, slots] = ring_x
    out["ring_z"] = torch.empty_like(ring_z)
    out["ring_z"][:, slots] = ring_z
    out.update(new_x=new_x, new_z=new_z, q=q, q_idx=q_idx, w=w)
    if kind == "csa":
        ie = normal((B, E, cfg.d_idx), 1.0, generator(s, base + 2, device), device)
        n_cand = E - cfg.n_win // m  # plant among entries older than one window
        planted = []
        for b in range(B):
            planted.append(planted_keys(ie[b], q_idx[b], w[b], cfg.planted_frac, n_cand, s, base + 50 + b))
        out["idx_entries"] = ie
        out["planted"] = planted
        rxi, rzi = raw_stream(B, cfg.n_win, cfg.d_idx, s, base + 9, device)
        out["ring_xi"] = torch.empty_like(rxi)
        out["ring_xi"][:, slots] = rxi
        out["ring_zi"] = torch.empty_like(rzi)
        out["ring_zi"][:, slots] = rzi
        out["new_xi"], out["new_zi"] = raw_stream(B, 1, cfg.d_idx, s, base + 11, device)
    return out


def mixed_lengths(cfg: Config, lo: int = 4096, hi: int = None) -> list:
    """Per-sequence stream lengths n_b = round(exp(U(ln lo, ln hi))) (hi defaults to cfg.ctx)."""
    hi = cfg.ctx if hi is None else hi
    u = torch.rand(cfg.batch, generator=generator(cfg.seed, 900, "cpu"), dtype=torch.float64)
    return [int(round(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo))))) for x in u]


def e4m3_codes(shape, std: float, g: torch.Generator, device="cpu") -> torch.Tensor:
    """E4M3 code bytes of ~N(0, std^2) values (torch's float8_e4m3fn rounding; never NaN)."""
    v = (torch.randn(tuple(shape), generator=g, device=device) * std).clamp(-448.0, 448.0)
    return v.to(torch.float8_e4m3fn).view(torch.uint8)


def e2m1_codes(shape, g: torch.Generator, device="cpu") -> torch.Tensor:
    """Random bytes of two E2M1 codes each (every 4-bit pattern is a finite value)."""
    return torch.randint(0, 256, tuple(shape), generator=g, device=device, dtype=torch.int32).to(torch.uint8)


def e4m3_block_scales(shape, g: torch.Generator, device="cpu") -> torch.Tensor:
    """Positive E4M3 scale bytes between 0.5 and 2 (codes 0x30 .. 0x40)."""
    return torch.randint(0x30, 0x41, tuple(shape), generator=g, device=device, dtype=torch.int32).to(torch.uint8)


def stored_sequence_state(cfg: Config, kind: str, b: int, n_b: int, device="cpu", stream_base: int = 0) -> dict:
    """Synthesised quantised state of one sequence of one decode layer at t = n_b - 1 (FP8 KV, FP4 indexer).

    kv_codes [E, d_qk] E4M3 bytes with kv_scale [E] fp32 (stored value = code x scale, ~N(0,1)/sqrt(d_qk));
    CSA also idx_codes [E, d_idx/2] E2M1 bytes with idx_scales [E, d_idx/16] E4M3 bytes;
    ring_x / ring_z [n_win, d] bf16 rows of positions t-128 .. t-1 at slot p % n_win (CSA: ring_xi / ring_zi).
    """
    m = cfg.m_csa if kind == "csa" else cfg.m_hca
    E = n_b // m
    t = n_b - 1
    s = cfg.seed
    base = stream_base + (0 if kind == "csa" else 100) + 1000 * (b + 1)
    out = {"kv_codes": e4m3_codes((E, cfg.d_qk), 1.0, generator(s, base + 1, device), device),
           "kv_scale": torch.full((E,), 1.0 / math.sqrt(cfg.d_qk), dtype=torch.float32, device=device)}
    slots = torch.tensor([(t - cfg.n_win + i) % cfg.n_win for i in range(cfg.n_win)], device=device)
    rx, rz = raw_stream(1, cfg.n_win, cfg.d_qk, s, base + 3, device)
    out["ring_x"] = torch.empty_like(rx[0])
    out["ring_x"][slots] = rx[0]
    out["ring_z"] = torch.empty_like(rz[0])
    out["ring_z"][slots] = rz[0]
    if kind == "csa":
        out["idx_codes"] = e2m1_codes((E, cfg.d_idx // 2), generator(s, base + 2, device), device)
        out["idx_scales"] = e4m3_block_scales((E, cfg.d_idx // 16), generator(s, base + 4, device), device)
        rxi, rzi = raw_stream(1, cfg.n_win, cfg.d_idx, s, base + 9, device)
        out["ring_xi"] = torch.empty_like(rxi[0])
        out["ring_xi"][slots] = rxi[0]
        out["ring_zi"] = torch.empty_like(rzi[0])
        out["ring_zi"][slots] = rzi[0]
    return out


def stored_step_inputs(cfg: Config, device="cpu", stream_base: int = 0) -> dict:
    """New rows and decode queries of one step for a quantised layer pair (FP4 indexer queries)."""
    B, s = cfg.batch, cfg.seed
    base = stream_base + 5000
    out = {}
    out["csa_x"], out["csa_z"] = raw_stream(B, 1, cfg.d_qk, s, base + 1, device)
    out["csa_xi"], out["csa_zi"] = raw_stream(B, 1, cfg.d_idx, s, base + 3, device)
    out["hca_x"], out["hca_z"] = raw_stream(B, 1, cfg.d_qk, s, base + 5, device)
    out["q_csa"] = normal((B, cfg.heads, cfg.d_qk), 1.0, generator(s, base + 7, device), device)
    out["q_hca"] = normal((B, cfg.heads, cfg.d_qk), 1.0, generator(s, base + 8, device), device)
    out["q_idx"] = e2m1_codes((B, cfg.heads_idx, cfg.d_idx // 2), generator(s, base + 9, device), device)
    out["q_idx_scale"] = e4m3_block_scales((B, cfg.heads_idx, cfg.d_idx // 16), generator(s, base + 10, device),
                                           device)
    out["w"] = uniform((B, cfg.heads_idx), 0.0, 1.0, generator(s, base + 11, device), device)
    return out
