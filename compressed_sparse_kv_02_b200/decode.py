"""One decode step through interleaved CSA and HCA layers, as a fixed sequence
of C-ABI calls (DeepSeek-V4 report digest, section 3: CSA and HCA layers are
interleaved; 10100.com article, section 2.3).

Per layer pair and step, for a batch of sequences whose newest token sits at
position t_b:
  CSA: cskv_cache_append -> csa_index_score_topk -> csa_attend
  HCA: cskv_cache_append -> hca_attend
The entry a step completes covers positions inside the step's own window, so
no query of the step reads it (the visibility rule: an entry is visible once
it lies wholly before the window). Its compression therefore runs off the
critical path, on a second stream:
  CSA: the whole append runs beside the indexer; csa_attend, which reads the
       ring's new row, waits for it;
  HCA: the ring rows are written first (ring_only), the compression
       (emit_only) runs beside hca_attend;
and the step ends when both streams have finished (the next append of a layer
overwrites ring rows that the compression reads). The argument blocks are
marshalled once (`DecodeModel.prepare`); the whole step can also be captured
in a CUDA graph (every call is stream-ordered and allocates nothing, and the
second stream forks from and joins the first through events).
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional

import torch

from . import _binding as B
from . import synth


FORK = "fork"  # the side stream waits for everything issued on the main stream so far
JOIN = "join"  # the main stream waits for everything issued on the side stream so far


class _Call:
    __slots__ = ("fn", "args", "ws", "ws_bytes", "where", "side")

    def __init__(self, fn, args, ws=None, where="", side=False):
        self.fn, self.args, self.where, self.side = fn, args, where, side
        self.ws = None if ws is None else ctypes.c_void_p(ws.data_ptr())
        self.ws_bytes = 0 if ws is None else ws.numel()

    def __call__(self, stream: ctypes.c_void_p):
        if self.ws_bytes:
            rc = self.fn(ctypes.byref(self.args), self.ws, self.ws_bytes, stream)
        else:
            rc = self.fn(ctypes.byref(self.args), stream)
        if rc != B.OK:
            raise B.CskvError(rc, self.where)


_DT = {"bf16": B.BF16, "fp8": B.FP8_E4M3, "fp4": B.FP4_E2M1}


class DecodeModel:
    """n_pairs (CSA, HCA) layer pairs with paged caches for `cfg.batch` sequences.

    ctx_lens: per-sequence stream lengths (the decode token of sequence b sits
    at position ctx_lens[b] - 1); defaults to cfg.ctx for every sequence.
    """

    def __init__(self, cfg: synth.Config, device="cuda", ctx_lens=None, n_pairs: int = 1):
        self.cfg = cfg
        self.device = device
        Bn = cfg.batch
        self.ctx_lens = [cfg.ctx] * Bn if ctx_lens is None else [int(c) for c in ctx_lens]
        self.max_pos = max(self.ctx_lens) - 1
        P = cfg.page_size
        self.layers = []
        for li in range(n_pairs):
            for kind, m in ((B.LAYER_CSA, cfg.m_csa), (B.LAYER_HCA, cfg.m_hca)):
                pages = [-(-(c // m) // P) for c in self.ctx_lens]
                L = B.Layer.allocate(kind, m, cfg.d_qk, cfg.d_v, n_seqs=Bn, n_pages=sum(pages),
                                     max_pages_per_seq=max(pages), page_size=P, n_win=cfg.n_win, d_idx=cfg.d_idx,
                                     kv_dtype=_DT[cfg.kv_dtype], idx_dtype=_DT[cfg.idx_dtype], device=device)
                perm = synth.page_permutation(sum(pages), cfg.seed, 500 + 2 * li + kind, device)
                o = 0
                for b, npg in enumerate(pages):
                    L.set_pages(b, perm[o:o + npg])
                    o += npg
                self.layers.append(L)
        self.seq = torch.arange(Bn, dtype=torch.int32, device=device)
        self.pos = torch.tensor([c - 1 for c in self.ctx_lens], dtype=torch.int64, device=device)
        H, k = cfg.heads, cfg.k
        self.out = {}
        for li in range(n_pairs):
            self.out[li] = dict(
                idx=torch.zeros(Bn, k, dtype=torch.int32, device=device),
                cnt=torch.zeros(Bn, dtype=torch.int32, device=device),
                o_csa=torch.zeros(Bn, H, cfg.d_v, dtype=torch.bfloat16, device=device),
                lse_csa=torch.zeros(Bn, H, dtype=torch.float32, device=device),
                o_hca=torch.zeros(Bn, H, cfg.d_v, dtype=torch.bfloat16, device=device),
                lse_hca=torch.zeros(Bn, H, dtype=torch.float32, device=device),
            )
        csa0, hca0 = self.layers[0], self.layers[1]
        self.ws_index = torch.empty(B.csa_index_ws_bytes(csa0, Bn, cfg.heads_idx, self.max_pos, k),
                                    dtype=torch.uint8, device=device)
        self.ws_csa = torch.empty(B.cskv_attend_ws_bytes(csa0, Bn, H, self.max_pos, k), dtype=torch.uint8,
                                  device=device)
        self.ws_hca = torch.empty(B.cskv_attend_ws_bytes(hca0, Bn, H, self.max_pos), dtype=torch.uint8,
                                  device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.inputs = None
        self._calls = None
        self._ops = None
        self._side = torch.cuda.Stream(device=device) if torch.device(device).type == "cuda" else None

    @property
    def n_pairs(self) -> int:
        return len(self.layers) // 2

    def step_inputs_like(self, device=None, pin=False) -> dict:
        """Empty per-step input tensors (queries and the new token's raw rows) for every layer pair."""
        cfg, Bn = self.cfg, self.cfg.batch
        dev = self.device if device is None else device
        kw = dict(device=dev, pin_memory=pin) if dev == "cpu" else dict(device=dev)
        inp = {}
        idx_q_shape = (Bn, cfg.heads_idx, cfg.d_idx if cfg.idx_dtype == "bf16" else cfg.d_idx // 2)
        for li in range(self.n_pairs):
            inp[li] = dict(
                csa_x=torch.empty(Bn, 1, cfg.d_qk, dtype=torch.bfloat16, **kw),
                csa_z=torch.empty(Bn, 1, cfg.d_qk, dtype=torch.bfloat16, **kw),
                csa_xi=torch.empty(Bn, 1, cfg.d_idx, dtype=torch.bfloat16, **kw),
                csa_zi=torch.empty(Bn, 1, cfg.d_idx, dtype=torch.bfloat16, **kw),
                q_csa=torch.empty(Bn, cfg.heads, cfg.d_qk, dtype=torch.bfloat16, **kw),
                q_idx=torch.empty(idx_q_shape, dtype=torch.bfloat16 if cfg.idx_dtype == "bf16" else torch.uint8,
                                  **kw),
                w=torch.empty(Bn, cfg.heads_idx, dtype=torch.float32, **kw),
                hca_x=torch.empty(Bn, 1, cfg.d_qk, dtype=torch.bfloat16, **kw),
                hca_z=torch.empty(Bn, 1, cfg.d_qk, dtype=torch.bfloat16, **kw),
                q_hca=torch.empty(Bn, cfg.heads, cfg.d_qk, dtype=torch.bfloat16, **kw),
            )
            if cfg.idx_dtype == "fp4":
                inp[li]["q_idx_scale"] = torch.empty(Bn, cfg.heads_idx, cfg.d_idx // 16, dtype=torch.uint8, **kw)
        return inp

    def fill_synthetic(self):
        """Synthesise every layer's cache and ring in stored form, plus the step inputs."""
        cfg = self.cfg
        if cfg.kv_dtype == "fp8" and cfg.idx_dtype == "fp4":
            return self._fill_synthetic_quantised()
        if cfg.kv_dtype != "bf16" or cfg.idx_dtype != "bf16" or len(set(self.ctx_lens)) != 1:
            raise NotImplementedError("fill_synthetic covers uniform-length bf16 and FP8 / FP4 workloads")
        self.inputs = self.step_inputs_like()
        self.planted = {}
        for li in range(self.n_pairs):
            csa, hca = self.layers[2 * li], self.layers[2 * li + 1]
            for kind, L in (("csa", csa), ("hca", hca)):
                st = synth.decode_layer_state(cfg, kind, self.device, stream_base=1000 * li)
                for b in range(cfg.batch):
                    L.write_entries(b, 0, kv=st["entries"][b], idx=st["idx_entries"][b] if kind == "csa" else None)
                L.ring_x.copy_(st["ring_x"])
                L.ring_z.copy_(st["ring_z"])
                inp = self.inputs[li]
                inp[kind + "_x"].copy_(st["new_x"])
                inp[kind + "_z"].copy_(st["new_z"])
                inp["q_" + kind].copy_(st["q"])
                if kind == "csa":
                    L.ring_xi.copy_(st["ring_xi"])
                    L.ring_zi.copy_(st["ring_zi"])
                    inp["csa_xi"].copy_(st["new_xi"])
                    inp["csa_zi"].copy_(st["new_zi"])
                    inp["q_idx"].copy_(st["q_idx"])
                    inp["w"].copy_(st["w"])
                    self.planted[li] = st["planted"]
                del st
        torch.cuda.synchronize()

    def _fill_synthetic_quantised(self):
        """FP8 KV and FP4 indexer caches, per-sequence lengths: one sequence at a time (bounded temporaries)."""
        cfg = self.cfg
        self.inputs = self.step_inputs_like()
        self.planted = {}
        for li in range(self.n_pairs):
            csa, hca = self.layers[2 * li], self.layers[2 * li + 1]
            for kind, L in (("csa", csa), ("hca", hca)):
                for b, n_b in enumerate(self.ctx_lens):
                    st = synth.stored_sequence_state(cfg, kind, b, n_b, self.device, stream_base=1000 * li)
                    if st["kv_codes"].shape[0]:
                        L.write_entries(b, 0, kv=st["kv_codes"], kv_scale=st["kv_scale"],
                                        idx=st.get("idx_codes"), idx_scale=st.get("idx_scales"))
                    L.ring_x[b].copy_(st["ring_x"])
                    L.ring_z[b].copy_(st["ring_z"])
                    if kind == "csa":
                        L.ring_xi[b].copy_(st["ring_xi"])
                        L.ring_zi[b].copy_(st["ring_zi"])
                    del st
            x = synth.stored_step_inputs(cfg, self.device, stream_base=1000 * li)
            for k_, v in x.items():
                self.inputs[li][k_].copy_(v.view(self.inputs[li][k_].shape))
            self.planted[li] = [torch.empty(0, dtype=torch.int64) for _ in range(cfg.batch)]
        torch.cuda.synchronize()

    def prepare(self, inputs: Optional[dict] = None):
        """Marshal every call of a step once; `inputs` (device tensors) defaults to self.inputs.

        Returns the step's ops for `run`: the calls in issue order (a call's `side` says which stream
        it goes to) with FORK / JOIN markers between them."""
        inp = self.inputs if inputs is None else inputs
        L = B.lib()
        cfg = self.cfg
        calls = []
        ops = []
        sm = 1.0 / math.sqrt(cfg.d_qk)
        self._keep = []
        for li in range(self.n_pairs):
            csa, hca = self.layers[2 * li], self.layers[2 * li + 1]
            x, o = inp[li], self.out[li]
            for layer, kind in ((csa, "csa"), (hca, "hca")):
                s = layer.struct
                self._keep.append(s)
                lp = ctypes.pointer(s)
                is_csa = kind == "csa"
                def append_args(ring_only, emit_only):
                    return B.AppendArgs(ctypes.sizeof(B.AppendArgs), lp, cfg.batch, 1, B._ptr(self.seq),
                                        B._ptr(self.pos), B._ptr(x[kind + "_x"]), B._ptr(x[kind + "_z"]),
                                        B._ptr(x["csa_xi"]) if is_csa else None,
                                        B._ptr(x["csa_zi"]) if is_csa else None,
                                        ring_only, B._ptr(self.status), emit_only)

                n0 = len(calls)
                if is_csa:
                    ia = B._index_args(layer, self.seq, self.pos, self.max_pos, x["q_idx"], x["w"], cfg.k, o["idx"],
                                       o["cnt"], None, x.get("q_idx_scale"), self.status)
                    aa = B._attend_args(layer, self.seq, self.pos, self.max_pos, x["q_csa"], o["idx"], o["cnt"],
                                        cfg.k, sm, o["o_csa"], o["lse_csa"], None, 0, self.status)
                    calls += [_Call(L.cskv_cache_append, append_args(0, 0), where="cskv_cache_append", side=True),
                              _Call(L.csa_index_score_topk, ia, self.ws_index, "csa_index_score_topk"),
                              _Call(L.csa_attend, aa, self.ws_csa, "csa_attend")]
                    ops += [FORK, calls[n0], calls[n0 + 1], JOIN, calls[n0 + 2]]
                else:
                    aa = B._attend_args(layer, self.seq, self.pos, self.max_pos, x["q_hca"], None, None, 0, sm,
                                        o["o_hca"], o["lse_hca"], None, 0, self.status)
                    calls += [_Call(L.cskv_cache_append, append_args(1, 0), where="cskv_cache_append_ring"),
                              _Call(L.cskv_cache_append, append_args(0, 1), where="cskv_cache_append_emit", side=True),
                              _Call(L.hca_attend, aa, self.ws_hca, "hca_attend")]
                    ops += [calls[n0], FORK, calls[n0 + 1], calls[n0 + 2]]
                for c in calls[n0:]:
                    self._keep.append(c.args)
        ops.append(JOIN)
        self._calls = calls
        self._ops = ops
        return ops

    def run(self, ops, stream=None, before=None, after=None):
        """Issue `ops` (from `prepare`) on `stream` (default: torch's current stream) and the side stream;
        before / after (optional) are called as f(i, call, stream) around the i-th call."""
        main = torch.cuda.current_stream() if stream is None else stream
        side = self._side
        i = 0
        for op in ops:
            if op is FORK:
                e = torch.cuda.Event()
                e.record(main)
                side.wait_event(e)
            elif op is JOIN:
                e = torch.cuda.Event()
                e.record(side)
                main.wait_event(e)
            else:
                s = side if op.side else main
                if before is not None:
                    before(i, op, s)
                op(B._stream(s))
                if after is not None:
                    after(i, op, s)
                i += 1

    def step(self, stream=None):
        """Run one decode step (all layer pairs) on `stream` (default: torch's current stream)."""
        if self._ops is None:
            self.prepare()
        self.run(self._ops, stream)

    def check_status(self) -> int:
        return B.cskv_get_status(self.status)
