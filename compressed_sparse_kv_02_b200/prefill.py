"""One prefill chunk through a CSA and an HCA layer, as a fixed sequence of
C-ABI calls (DeepSeek-V4 report digest, section 3; 10100.com article,
section 2.1: the chunk is compressed, then every position of it is indexed
and attended).

A sequence holds `cached` tokens (compressed caches plus the last n_win raw
rows in the rings) and receives `chunk` new raw tokens at positions
cached .. cached+chunk-1. One pass:
  CSA: csa_compress_kv over the chunk (latent and indexer-key streams)
  HCA: hca_compress_kv over the chunk
  per block of up to 4096 query positions:
       csa_index_score_topk -> csa_attend (window rows from the chunk or the ring)
       hca_attend
  cskv_cache_append (ring only) of the chunk's last n_win rows.
The pass starts by writing the cached tail back into the rings (a ring-only
append of the n_win rows before the chunk), so that it can be repeated on
the same state. Argument blocks are marshalled once (`prepare`).
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional

import torch

from . import _binding as B
from . import synth
from .decode import _Call


class PrefillModel:
    def __init__(self, cfg: synth.Config, cached: int, chunk: int, device="cuda", q_block: int = 4096):
        if cached % cfg.m_hca or chunk % cfg.m_hca or cached < cfg.n_win:
            raise ValueError("cached and chunk must be multiples of m' and cached >= n_win")
        self.cfg, self.device = cfg, device
        self.cached, self.chunk, self.q_block = cached, chunk, min(q_block, chunk)
        n = cached + chunk
        P = cfg.page_size
        self.layers = []
        for kind, m in ((B.LAYER_CSA, cfg.m_csa), (B.LAYER_HCA, cfg.m_hca)):
            pages = -(-(n // m) // P)
            L = B.Layer.allocate(kind, m, cfg.d_qk, cfg.d_v, n_seqs=1, n_pages=pages, max_pages_per_seq=pages,
                                 page_size=P, n_win=cfg.n_win, d_idx=cfg.d_idx, device=device)
            L.set_pages(0, synth.page_permutation(pages, cfg.seed, 600 + kind, device))
            self.layers.append(L)
        self.max_pos = n - 1
        self.seq = torch.zeros(1, dtype=torch.int32, device=device)
        self.q_pos = torch.arange(cached, n, dtype=torch.int64, device=device)
        self.q_seq = torch.zeros(chunk, dtype=torch.int32, device=device)
        H, k = cfg.heads, cfg.k
        self.idx = torch.zeros(chunk, k, dtype=torch.int32, device=device)
        self.cnt = torch.zeros(chunk, dtype=torch.int32, device=device)
        self.o_csa = torch.zeros(chunk, H, cfg.d_v, dtype=torch.bfloat16, device=device)
        self.o_hca = torch.zeros(chunk, H, cfg.d_v, dtype=torch.bfloat16, device=device)
        csa, hca = self.layers
        qb = self.q_block
        self.ws_index = torch.empty(B.csa_index_ws_bytes(csa, qb, cfg.heads_idx, self.max_pos, k), dtype=torch.uint8,
                                    device=device)
        self.ws_csa = torch.empty(B.cskv_attend_ws_bytes(csa, qb, H, self.max_pos, k), dtype=torch.uint8,
                                  device=device)
        self.ws_hca = torch.empty(B.cskv_attend_ws_bytes(hca, qb, H, self.max_pos), dtype=torch.uint8,
                                  device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.inputs = None
        self._calls = None

    def fill_synthetic(self):
        """Cached entries in stored form, the cached tail and the chunk as raw rows, and the chunk's queries."""
        cfg, dev, c0, T = self.cfg, self.device, self.cached, self.chunk
        s = cfg.seed
        csa, hca = self.layers
        d, di = cfg.d_qk, cfg.d_idx
        csa.write_entries(0, 0, kv=synth.normal((c0 // cfg.m_csa, d), 1.0 / math.sqrt(d), synth.generator(s, 1, dev),
                                                dev),
                          idx=synth.normal((c0 // cfg.m_csa, di), 1.0, synth.generator(s, 2, dev), dev))
        hca.write_entries(0, 0, kv=synth.normal((c0 // cfg.m_hca, d), 1.0 / math.sqrt(d), synth.generator(s, 3, dev),
                                                dev))
        inp = {}
        # raw rows of the cached tail (positions c0 - n_win .. c0 - 1) and of the chunk, per layer
        for name, dd, st in (("x", d, 10), ("xi", di, 20), ("x_h", d, 30)):
            tail_x, tail_z = synth.raw_stream(1, cfg.n_win, dd, s, st, dev)
            x, z = synth.raw_stream(1, T, dd, s, st + 2, dev)
            inp["tail_" + name], inp["tail_z" + name[1:]] = tail_x, tail_z
            inp[name], inp["z" + name[1:]] = x, z
        inp["q"] = synth.normal((T, cfg.heads, d), 1.0, synth.generator(s, 40, dev), dev)
        inp["q_h"] = synth.normal((T, cfg.heads, d), 1.0, synth.generator(s, 41, dev), dev)
        inp["q_idx"] = synth.normal((T, cfg.heads_idx, di), 1.0, synth.generator(s, 42, dev), dev)
        inp["w"] = synth.uniform((T, cfg.heads_idx), 0.0, 1.0, synth.generator(s, 43, dev), dev)
        self.inputs = inp
        torch.cuda.synchronize()

    def prepare(self):
        L = B.lib()
        cfg, inp, c0, T, qb = self.cfg, self.inputs, self.cached, self.chunk, self.q_block
        csa, hca = self.layers
        sm = 1.0 / math.sqrt(cfg.d_qk)
        keep = [csa.struct, hca.struct]
        lc, lh = ctypes.pointer(keep[0]), ctypes.pointer(keep[1])
        calls = []
        tail_pos = torch.tensor([c0 - cfg.n_win], dtype=torch.int64, device=self.device)
        end_pos = torch.tensor([c0 + T - cfg.n_win], dtype=torch.int64, device=self.device)
        self._pos = (tail_pos, end_pos)
        last = slice(T - cfg.n_win, T)
        self._last = {k_: inp[k_][:, last].contiguous() for k_ in ("x", "z", "xi", "zi", "x_h", "z_h")}
        # restore the rings to the cached state (so that the pass can be repeated)
        calls.append(_Call(L.cskv_cache_append, B.AppendArgs(
            ctypes.sizeof(B.AppendArgs), lc, 1, cfg.n_win, B._ptr(self.seq), B._ptr(tail_pos), B._ptr(inp["tail_x"]),
            B._ptr(inp["tail_z"]), B._ptr(inp["tail_xi"]), B._ptr(inp["tail_zi"]), 1, B._ptr(self.status)),
            where="cskv_cache_append"))
        calls.append(_Call(L.cskv_cache_append, B.AppendArgs(
            ctypes.sizeof(B.AppendArgs), lh, 1, cfg.n_win, B._ptr(self.seq), B._ptr(tail_pos),
            B._ptr(inp["tail_x_h"]), B._ptr(inp["tail_z_h"]), None, None, 1, B._ptr(self.status)),
            where="cskv_cache_append"))
        calls.append(_Call(L.csa_compress_kv, B.CompressArgs(
            ctypes.sizeof(B.CompressArgs), lc, 1, B._ptr(self.seq), c0, T, B._ptr(inp["x"]), B._ptr(inp["z"]),
            B._ptr(inp["xi"]), B._ptr(inp["zi"]), B._ptr(self.status)), where="csa_compress_kv"))
        calls.append(_Call(L.hca_compress_kv, B.CompressArgs(
            ctypes.sizeof(B.CompressArgs), lh, 1, B._ptr(self.seq), c0, T, B._ptr(inp["x_h"]), B._ptr(inp["z_h"]),
            None, None, B._ptr(self.status)), where="hca_compress_kv"))
        xc, xh = inp["x"][0], inp["x_h"][0]
        for q0 in range(0, T, qb):
            sl = slice(q0, min(T, q0 + qb))
            n = sl.stop - sl.start
            ia = B._index_args(csa, self.q_seq[sl], self.q_pos[sl], self.max_pos, inp["q_idx"][sl], inp["w"][sl],
                               cfg.k, self.idx[sl], self.cnt[sl], None, None, self.status)
            ia.layer = lc
            calls.append(_Call(L.csa_index_score_topk, ia, self.ws_index, "csa_index_score_topk"))
            aa = B._attend_args(csa, self.q_seq[sl], self.q_pos[sl], self.max_pos, inp["q"][sl], self.idx[sl],
                                self.cnt[sl], cfg.k, sm, self.o_csa[sl], None, xc, c0, self.status)
            aa.layer = lc
            calls.append(_Call(L.csa_attend, aa, self.ws_csa, "csa_attend"))
            ha = B._attend_args(hca, self.q_seq[sl], self.q_pos[sl], self.max_pos, inp["q_h"][sl], None, None, 0, sm,
                                self.o_hca[sl], None, xh, c0, self.status)
            ha.layer = lh
            calls.append(_Call(L.hca_attend, ha, self.ws_hca, "hca_attend"))
            assert n > 0
        # the rings take the chunk's last n_win rows (the state the next chunk starts from)
        last_ = self._last
        calls.append(_Call(L.cskv_cache_append, B.AppendArgs(
            ctypes.sizeof(B.AppendArgs), lc, 1, cfg.n_win, B._ptr(self.seq), B._ptr(end_pos), B._ptr(last_["x"]),
            B._ptr(last_["z"]), B._ptr(last_["xi"]), B._ptr(last_["zi"]), 1, B._ptr(self.status)),
            where="cskv_cache_append"))
        calls.append(_Call(L.cskv_cache_append, B.AppendArgs(
            ctypes.sizeof(B.AppendArgs), lh, 1, cfg.n_win, B._ptr(self.seq), B._ptr(end_pos), B._ptr(last_["x_h"]),
            B._ptr(last_["z_h"]), None, None, 1, B._ptr(self.status)), where="cskv_cache_append"))
        self._keep = keep
        self._calls = calls
        return calls

    def step(self, stream=None):
        """Run one prefill pass of the chunk on `stream` (default: torch's current stream)."""
        if self._calls is None:
            self.prepare()
        st = B._stream(stream)
        for c in self._calls:
            c(st)

    def check_status(self) -> int:
        return B.cskv_get_status(self.status)

    def flops(self) -> dict:
        """Algorithmic flops of one pass: indexer sum_t |E_csa(t)| H_I d_I 2, attention per key and head
        2 (d_qk + d_v) over the window and the selected (CSA) or visible (HCA) entries."""
        cfg = self.cfg
        fi = fc = fh = 0
        per_key = 2 * (cfg.d_qk + cfg.d_v) * cfg.heads
        for t in range(self.cached, self.cached + self.chunk):
            lim = t + 1 - cfg.n_win
            nv = max(0, -(-lim // cfg.m_csa))
            nv_h = max(0, -(-lim // cfg.m_hca))
            n_w = min(cfg.n_win, t + 1)
            fi += nv * cfg.heads_idx * cfg.d_idx * 2
            fc += (n_w + min(cfg.k, nv)) * per_key
            fh += (n_w + nv_h) * per_key
        return {"index": fi, "csa_attend": fc, "hca_attend": fh, "total": fi + fc + fh}


def main(argv=None) -> int:
    """Run `passes` prefill passes of one chunk (the benchmark's shapes: 64 heads, d = 128, indexer 4 x 64,
    top-512) and check the status word; used to profile one block of the prefill on its own."""
    import argparse
    ap = argparse.ArgumentParser(description=main.__doc__)
    ap.add_argument("--cached", type=int, default=65536)
    ap.add_argument("--chunk", type=int, default=4096)
    ap.add_argument("--q-block", type=int, default=4096)
    ap.add_argument("--passes", type=int, default=2)
    a = ap.parse_args(argv)
    cfg = synth.Config("prefill_block", 1, a.cached + a.chunk, 64, 128, 128, 4, 64, 512, seed=3)
    model = PrefillModel(cfg, cached=a.cached, chunk=a.chunk, q_block=a.q_block)
    model.fill_synthetic()
    for _ in range(a.passes):
        model.step()
    torch.cuda.synchronize()
    st = model.check_status()
    print("prefill passes: %d, status %s, device memory %.2f GB"
          % (a.passes, B.status_string(st), torch.cuda.max_memory_allocated() / 1e9))
    return 0 if st == B.OK else 1


if __name__ == "__main__":
    raise SystemExit(main())


class VarlenPrefillModel:
    """One prefill pass over several sequences at once, each with its own cached length and chunk length
    (DeepSeek-V4 report digest, section 7 / Figure 6: the state cache carries each sequence's window
    between chunks; 10100.com article, section 6: the compressed cache is extended chunk by chunk).

    Sequence b holds cached[b] tokens (compressed entries plus its last n_win raw rows in the rings) and
    receives chunk[b] new tokens. The chunks are packed one after another: query row r of the pass is
    position cached[b] + i of sequence b. One pass:
      rings  : restored to the cached state (one ring-only append for all sequences)
      fold   : csa_compress_kv / hca_compress_kv of each sequence's chunk (its own tok0 and length)
      blocks of up to q_block query rows, spanning sequences:
               csa_index_score_topk -> csa_attend, hca_attend, with the packed chunk rows and a
               per-sequence chunk descriptor (first row, first position, length) for the window rows
      rings  : the last n_win rows of every chunk (one ring-only append for all sequences).
    cached[b] and chunk[b] are multiples of m' = 128, cached[b] >= n_win, chunk[b] >= n_win.
    """

    def __init__(self, cfg: synth.Config, cached, chunk, device="cuda", q_block: int = 4096):
        cached, chunk = [int(c) for c in cached], [int(c) for c in chunk]
        if len(cached) != len(chunk) or not cached:
            raise ValueError("one cached and one chunk length per sequence")
        for c0, T in zip(cached, chunk):
            if c0 % cfg.m_hca or T % cfg.m_hca or c0 < cfg.n_win or T < cfg.n_win:
                raise ValueError("cached and chunk lengths must be multiples of m' and at least n_win")
        self.cfg, self.device = cfg, device
        self.cached, self.chunk = cached, chunk
        self.n_seqs = Bn = len(cached)
        self.total = sum(chunk)
        self.q_block = min(q_block, self.total)
        self.row0 = [sum(chunk[:b]) for b in range(Bn)]
        ends = [c0 + T for c0, T in zip(cached, chunk)]
        self.max_pos = max(ends) - 1
        P = cfg.page_size
        self.layers = []
        for kind, m in ((B.LAYER_CSA, cfg.m_csa), (B.LAYER_HCA, cfg.m_hca)):
            pages = [-(-(n // m) // P) for n in ends]
            L = B.Layer.allocate(kind, m, cfg.d_qk, cfg.d_v, n_seqs=Bn, n_pages=sum(pages),
                                 max_pages_per_seq=max(pages), page_size=P, n_win=cfg.n_win, d_idx=cfg.d_idx,
                                 device=device)
            perm = synth.page_permutation(sum(pages), cfg.seed, 700 + kind, device)
            o = 0
            for b, npg in enumerate(pages):
                L.set_pages(b, perm[o:o + npg])
                o += npg
            self.layers.append(L)
        self.seq = torch.arange(Bn, dtype=torch.int32, device=device)
        self.q_seq = torch.cat([torch.full((T,), b, dtype=torch.int32) for b, T in enumerate(chunk)]).to(device)
        self.q_pos = torch.cat([torch.arange(c0, c0 + T, dtype=torch.int64)
                                for c0, T in zip(cached, chunk)]).to(device)
        self.chunk_desc = torch.tensor([[self.row0[b], cached[b], chunk[b]] for b in range(Bn)], dtype=torch.int64,
                                       device=device)
        H, k = cfg.heads, cfg.k
        self.idx = torch.zeros(self.total, k, dtype=torch.int32, device=device)
        self.cnt = torch.zeros(self.total, dtype=torch.int32, device=device)
        self.o_csa = torch.zeros(self.total, H, cfg.d_v, dtype=torch.bfloat16, device=device)
        self.o_hca = torch.zeros(self.total, H, cfg.d_v, dtype=torch.bfloat16, device=device)
        csa, hca = self.layers
        qb = self.q_block
        self.ws_index = torch.empty(B.csa_index_ws_bytes(csa, qb, cfg.heads_idx, self.max_pos, k), dtype=torch.uint8,
                                    device=device)
        self.ws_csa = torch.empty(B.cskv_attend_ws_bytes(csa, qb, H, self.max_pos, k), dtype=torch.uint8,
                                  device=device)
        self.ws_hca = torch.empty(B.cskv_attend_ws_bytes(hca, qb, H, self.max_pos), dtype=torch.uint8,
                                  device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.inputs = None
        self._calls = None

    def fill_synthetic(self):
        """Per sequence: cached entries in stored form, the cached tail as raw rows; the packed chunks and
        their queries."""
        cfg, dev = self.cfg, self.device
        s = cfg.seed
        csa, hca = self.layers
        d, di, nw = cfg.d_qk, cfg.d_idx, cfg.n_win
        for b, c0 in enumerate(self.cached):
            csa.write_entries(b, 0, kv=synth.normal((c0 // cfg.m_csa, d), 1.0 / math.sqrt(d),
                                                    synth.generator(s, 100 + b, dev), dev),
                              idx=synth.normal((c0 // cfg.m_csa, di), 1.0, synth.generator(s, 200 + b, dev), dev))
            hca.write_entries(b, 0, kv=synth.normal((c0 // cfg.m_hca, d), 1.0 / math.sqrt(d),
                                                    synth.generator(s, 300 + b, dev), dev))
        inp = {}
        for name, dd, st in (("x", d, 10), ("xi", di, 20), ("x_h", d, 30)):
            tail_x, tail_z = synth.raw_stream(self.n_seqs, nw, dd, s, st, dev)
            x, z = synth.raw_stream(1, self.total, dd, s, st + 2, dev)
            inp["tail_" + name], inp["tail_z" + name[1:]] = tail_x, tail_z
            inp[name], inp["z" + name[1:]] = x[0], z[0]  # packed chunks [total, dd]
        inp["q"] = synth.normal((self.total, cfg.heads, d), 1.0, synth.generator(s, 40, dev), dev)
        inp["q_h"] = synth.normal((self.total, cfg.heads, d), 1.0, synth.generator(s, 41, dev), dev)
        inp["q_idx"] = synth.normal((self.total, cfg.heads_idx, di), 1.0, synth.generator(s, 42, dev), dev)
        inp["w"] = synth.uniform((self.total, cfg.heads_idx), 0.0, 1.0, synth.generator(s, 43, dev), dev)
        self.inputs = inp
        torch.cuda.synchronize()

    def prepare(self):
        L = B.lib()
        cfg, inp, qb, nw = self.cfg, self.inputs, self.q_block, self.cfg.n_win
        csa, hca = self.layers
        sm = 1.0 / math.sqrt(cfg.d_qk)
        keep = [csa.struct, hca.struct]
        lc, lh = ctypes.pointer(keep[0]), ctypes.pointer(keep[1])
        calls = []
        Bn = self.n_seqs
        tail_pos = torch.tensor([c0 - nw for c0 in self.cached], dtype=torch.int64, device=self.device)
        end_pos = torch.tensor([c0 + T - nw for c0, T in zip(self.cached, self.chunk)], dtype=torch.int64,
                               device=self.device)
        # the last n_win rows of every chunk, stacked [n_seqs, n_win, d]
        last = {k_: torch.stack([inp[k_][r + T - nw:r + T] for r, T in zip(self.row0, self.chunk)]).contiguous()
                for k_ in ("x", "z", "xi", "zi", "x_h", "z_h")}
        chunks = []  # per-sequence chunk views [1, T, d] for the folds
        for b, (r, T) in enumerate(zip(self.row0, self.chunk)):
            chunks.append({k_: inp[k_][r:r + T].unsqueeze(0).contiguous()
                           for k_ in ("x", "z", "xi", "zi", "x_h", "z_h")})
        self._keep_tensors = (tail_pos, end_pos, last, chunks)
        calls.append(_Call(L.cskv_cache_append, B.AppendArgs(
            ctypes.sizeof(B.AppendArgs), lc, Bn, nw, B._ptr(self.seq), B._ptr(tail_pos), B._ptr(inp["tail_x"]),
            B._ptr(inp["tail_z"]), B._ptr(inp["tail_xi"]), B._ptr(inp["tail_zi"]), 1, B._ptr(self.status)),
            where="cskv_cache_append"))
        calls.append(_Call(L.cskv_cache_append, B.AppendArgs(
            ctypes.sizeof(B.AppendArgs), lh, Bn, nw, B._ptr(self.seq), B._ptr(tail_pos), B._ptr(inp["tail_x_h"]),
            B._ptr(inp["tail_z_h"]), None, None, 1, B._ptr(self.status)), where="cskv_cache_append"))
        for b in range(Bn):
            c = chunks[b]
            sq = self.seq[b:b + 1]
            calls.append(_Call(L.csa_compress_kv, B.CompressArgs(
                ctypes.sizeof(B.CompressArgs), lc, 1, B._ptr(sq), self.cached[b], self.chunk[b], B._ptr(c["x"]),
                B._ptr(c["z"]), B._ptr(c["xi"]), B._ptr(c["zi"]), B._ptr(self.status)), where="csa_compress_kv"))
            calls.append(_Call(L.hca_compress_kv, B.CompressArgs(
                ctypes.sizeof(B.CompressArgs), lh, 1, B._ptr(sq), self.cached[b], self.chunk[b], B._ptr(c["x_h"]),
                B._ptr(c["z_h"]), None, None, B._ptr(self.status)), where="hca_compress_kv"))
        for q0 in range(0, self.total, qb):
            sl = slice(q0, min(self.total, q0 + qb))
            ia = B._index_args(csa, self.q_seq[sl], self.q_pos[sl], self.max_pos, inp["q_idx"][sl], inp["w"][sl],
                               cfg.k, self.idx[sl], self.cnt[sl], None, None, self.status)
            ia.layer = lc
            calls.append(_Call(L.csa_index_score_topk, ia, self.ws_index, "csa_index_score_topk"))
            aa = B._attend_args(csa, self.q_seq[sl], self.q_pos[sl], self.max_pos, inp["q"][sl], self.idx[sl],
                                self.cnt[sl], cfg.k, sm, self.o_csa[sl], None, inp["x"], 0, self.status,
                                chunk_desc=self.chunk_desc)
            aa.layer = lc
            calls.append(_Call(L.csa_attend, aa, self.ws_csa, "csa_attend"))
            ha = B._attend_args(hca, self.q_seq[sl], self.q_pos[sl], self.max_pos, inp["q_h"][sl], None, None, 0, sm,
                                self.o_hca[sl], None, inp["x_h"], 0, self.status, chunk_desc=self.chunk_desc)
            ha.layer = lh
            calls.append(_Call(L.hca_attend, ha, self.ws_hca, "hca_attend"))
        calls.append(_Call(L.cskv_cache_append, B.AppendArgs(
            ctypes.sizeof(B.AppendArgs), lc, Bn, nw, B._ptr(self.seq), B._ptr(end_pos), B._ptr(last["x"]),
            B._ptr(last["z"]), B._ptr(last["xi"]), B._ptr(last["zi"]), 1, B._ptr(self.status)),
            where="cskv_cache_append"))
        calls.append(_Call(L.cskv_cache_append, B.AppendArgs(
            ctypes.sizeof(B.AppendArgs), lh, Bn, nw, B._ptr(self.seq), B._ptr(end_pos), B._ptr(last["x_h"]),
            B._ptr(last["z_h"]), None, None, 1, B._ptr(self.status)), where="cskv_cache_append"))
        self._keep = keep
        self._calls = calls
        return calls

    def step(self, stream=None):
        if self._calls is None:
            self.prepare()
        st = B._stream(stream)
        for c in self._calls:
            c(st)

    def check_status(self) -> int:
        return B.cskv_get_status(self.status)
