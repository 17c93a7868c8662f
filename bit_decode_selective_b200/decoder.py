"""A Llama-shaped decode step built from the refined kernels.

Every step of the computation runs in the CUDA library (include/sf.h); this
module only owns the buffers (allocated with PyTorch), the streams and events,
and the order of the calls.  The call order implements the schedule of
"StrataFlux -- Selective precision streaming -- What does it mean?":
  which-tiles-count paragraph -- every projection refines the k channels with
    the largest |x| per 1,024-channel chunk; attention refines the
    highest-scoring tokens per KV head;
  the-map-app-also-loads-tiles paragraph -- refinement rows live in host RAM;
    fetch lead (1 layer) selects a projection's channels from the previous
    layer's activation and starts the row transfer on a staging stream while the
    layers in between compute; fetch lag (1 layer) applies the residual-writing
    projections' (o, down) corrections at the start of the next layer.  With
    the rows staged a layer ahead, o's projection computes its correction in
    the same launch and writes it to a separate buffer that the next layer's
    residual add picks up (so the MLP input does not see it); down's lagged
    correction enters the residual stream at the same point as down's own
    output (nothing reads the residual in between), so down refines in place.
Readings as in the oracle (oracle/decoder.py): layer 0 selects from its own
activations; q/k/v and gate/up correct in place; the new token is appended at
position T and attention runs over T + 1 tokens.

step() only enqueues work on the current stream (plus the two staging
streams), so it can be captured in a CUDA graph and replayed.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import abi
from .abi import check
from .ops import KVCache, QuantWeights, _p


@dataclass
class DecoderConfig:
    n_layers: int = 32
    hidden: int = 4096
    inter: int = 14336
    h_q: int = 32
    h_kv: int = 8
    d: int = 128
    vocab: int = 128256
    w_bits: int = 2
    w_refine: int = 2
    group: int = 128
    chunk: int = 1024
    kch: int = 32
    kv_bits: int = 2
    kv_refine: int = 2
    k_tok: int = 512
    lead: int = 1
    lag: int = 1
    host_refine: bool = True  # refinement rows in pinned host memory, staged per layer
    # refinement rows kept on the device across steps, per (layer, projection,
    # batch row): capacity = cache_rows x the projection's selected channels (0: no cache)
    cache_rows: float = 0.0
    skip_missing: bool = False  # with the cache: a missing row leaves its channel at base precision this step
    eps: float = 1e-5
    theta: float = 500000.0

    def shapes(self):
        """(name, n, k) of the four fused projections of a layer."""
        qkv = (self.h_q + 2 * self.h_kv) * self.d
        return (("qkv", qkv, self.hidden), ("o", self.hidden, self.h_q * self.d),
                ("gate_up", 2 * self.inter, self.hidden), ("down", self.hidden, self.inter))


PROJ = ("qkv", "o", "gate_up", "down")


def _s(stream):
    return ctypes.c_void_p(stream.cuda_stream)


class Decoder:
    def __init__(self, cfg: DecoderConfig, batch: int, t: int, device="cuda"):
        self.cfg, self.B, self.T = cfg, batch, t
        self.dev = torch.device(device)
        dev = self.dev
        self.t_max = (t + 1 + 15) // 16 * 16
        self.layers = []
        self.host_rows = []   # per layer: name -> pinned [k][n*r/8] uint8
        f32 = lambda *s: torch.zeros(*s, dtype=torch.float32, device=dev)
        f16 = lambda *s: torch.zeros(*s, dtype=torch.float16, device=dev)
        i32 = lambda *s: torch.zeros(*s, dtype=torch.int32, device=dev)
        shp = {n: (nn, kk) for n, nn, kk in cfg.shapes()}
        self.shp = shp
        self.n_sel = {n: (shp[n][1] // cfg.chunk) * cfg.kch for n in PROJ}
        self.row_bytes = {n: shp[n][0] * cfg.w_refine // 8 for n in PROJ}
        B = batch
        # activations
        self.h = f32(B, cfg.hidden)
        self.x_attn = [f16(B, cfg.hidden) for _ in range(2)]
        self.qkv_out = f32(B, shp["qkv"][0])
        self.q = f16(B, cfg.h_q, cfg.d)
        self.x_o = [f16(B, cfg.h_q * cfg.d) for _ in range(2)]
        self.o_out = f32(B, cfg.hidden)
        self.x_mlp = [f16(B, cfg.hidden) for _ in range(2)]
        self.gu_out = f32(B, 2 * cfg.inter)
        self.x_down = [f16(B, cfg.inter) for _ in range(2)]
        self.down_out = f32(B, cfg.hidden)
        self.x_final = f16(B, cfg.hidden)
        self.logits = f32(B, cfg.vocab)
        self.tok_sel = i32(B, cfg.h_kv, cfg.k_tok)
        # selections (two slots: this layer / next layer) and staged rows
        self.sel = {n: [i32(B, self.n_sel[n]) for _ in range(2)] for n in PROJ}
        if cfg.kch and cfg.host_refine:
            self.slots = {n: [torch.empty(B * self.n_sel[n] * self.row_bytes[n], dtype=torch.uint8, device=dev)
                              for _ in range(2)] for n in PROJ}
        else:
            self.slots = None
        # with the row cache: the selection each GEMV uses (channels whose rows
        # did not arrive are marked -1 - c), per projection and slot
        self.use_cache = bool(cfg.kch and cfg.host_refine and cfg.cache_rows > 0)
        self.sel_eff = ({n: [i32(B, self.n_sel[n]) for _ in range(2)] for n in PROJ} if self.use_cache else None)
        self.caches = []  # per layer: name -> (ctypes array of B sf_row_cache, tensors kept alive)
        # the GEMV's workspace (its size query returns 0 today; sized for the widest input)
        kmax = max(kk for _, _, kk in cfg.shapes())
        wq = abi.sf_wq(128, kmax, cfg.w_bits, cfg.w_refine, cfg.group, None, None, None)
        self.gemv_ws = torch.empty(max(abi.sf_gemv_workspace_bytes(ctypes.byref(wq), B, cfg.chunk, cfg.kch), 16),
                                   dtype=torch.uint8, device=dev)
        # staging queues: selections and row transfers of qkv and gate_up on one,
        # of o and down on the other, so that transfers of different projections overlap
        self.side = torch.cuda.Stream(device=dev)
        self.side2 = torch.cuda.Stream(device=dev)
        self.stage_stream = {"qkv": self.side, "gate_up": self.side, "o": self.side2, "down": self.side2}
        self.ev_sel = {n: [torch.cuda.Event() for _ in range(2)] for n in PROJ}
        self.ev_stage = {n: [torch.cuda.Event() for _ in range(2)] for n in PROJ}
        for evs in (self.ev_sel, self.ev_stage):  # create the events now: the library records them by handle
            for pair in evs.values():
                for ev in pair:
                    ev.record(torch.cuda.current_stream(dev))
        # fetch lag: layer l's o correction, written by its projection and added
        # by the next layer's residual add
        self.delta = f32(B, cfg.hidden)
        self.lm_head = None
        self.ws = None
        # when a list: every selection a projection or the attention uses is
        # copied into it (on the step's stream), for checks against the oracle
        self.trace = None

    # ---- model state -----------------------------------------------------

    def load_layer(self, weights: dict, k_cache: torch.Tensor, v_cache: torch.Tensor):
        """weights: name -> fp32 [n][k] on the device; k/v_cache fp16
        [B][h_kv][T][d] on the device (the T cached tokens)."""
        cfg = self.cfg
        L = {}
        host = {}
        for n in PROJ:
            w = weights[n]
            qw = QuantWeights.pack(w.contiguous(), cfg.w_bits, cfg.w_refine, cfg.group)
            if cfg.host_refine:
                rows = torch.empty(qw.refine.numel(), dtype=torch.uint8, pin_memory=True)
                rows.copy_(qw.refine)
                host[n] = rows
                qw.refine = None
                qw.desc.refine = None
            L[n] = qw
        if self.use_cache:
            self.caches.append({n: self._make_caches(n) for n in PROJ})
        kv = KVCache(self.B, cfg.h_kv, self.t_max, cfg.kv_bits, cfg.kv_refine, cfg.d, device=self.dev)
        kv.pack_tokens(k_cache.contiguous(), v_cache.contiguous(), 0)
        L["kv"] = kv
        self.layers.append(L)
        self.host_rows.append(host)
        torch.cuda.synchronize(self.dev)

    def _make_caches(self, name):
        """One empty row cache per batch row for one projection of one layer."""
        n_ch = self.shp[name][1]
        cap = max(self.n_sel[name], int(round(self.cfg.cache_rows * self.n_sel[name])))
        i32 = lambda n: torch.empty(n, dtype=torch.int32, device=self.dev)
        arr = (abi.sf_row_cache * self.B)()
        keep = []
        for b in range(self.B):
            t = dict(slot_of=i32(n_ch), channel_of=i32(cap), stamp=i32(cap), state=i32(4),
                     work=i32(self.n_sel[name]),
                     rows=torch.empty(cap * self.row_bytes[name], dtype=torch.uint8, device=self.dev))
            keep.append(t)
            arr[b] = abi.sf_row_cache(cap, n_ch, self.row_bytes[name], t["slot_of"].data_ptr(),
                                      t["channel_of"].data_ptr(), t["stamp"].data_ptr(), t["state"].data_ptr(),
                                      t["work"].data_ptr(), self.n_sel[name], t["rows"].data_ptr())
            check(abi.sf_row_cache_reset(ctypes.byref(arr[b]), _s(torch.cuda.current_stream(self.dev))),
                  "sf_row_cache_reset")
        return arr, keep

    def cache_stats(self):
        """{projection: (hits, misses)} summed over the layers' and batch rows'
        row caches since they were made (empty without caches)."""
        out = {}
        for L in self.caches:
            for name, (arr, keep) in L.items():
                h, m = out.get(name, (0, 0))
                for t in keep:
                    st = t["state"].cpu()
                    h += int(st[2]) & 0xFFFFFFFF
                    m += int(st[3]) & 0xFFFFFFFF
                out[name] = (h, m)
        return out

    def set_rows_resident(self, resident: bool):
        """Keep the refinement rows on the device (True: every projection reads
        its selected rows from its own refinement buffer and nothing crosses the
        host link; the selections still run a layer ahead on the staging
        streams) or stage them from pinned host memory again (False).  Only for
        a decoder built with host_refine and run without the row cache."""
        assert self.cfg.host_refine and self.cfg.kch and not self.use_cache
        if resident and self.slots is not None:
            self._host_slots = self.slots
            self.slots = None
            for L, host in zip(self.layers, self.host_rows):
                for n in PROJ:
                    qw = L[n]
                    if getattr(qw, "_dev_refine", None) is None:
                        qw._dev_refine = host[n].to(self.dev)
                    qw.refine = qw._dev_refine
                    qw.desc.refine = qw.refine.data_ptr()
            torch.cuda.synchronize(self.dev)
        elif not resident and self.slots is None:
            self.slots = self._host_slots
            for L in self.layers:
                for n in PROJ:
                    L[n].refine = None
                    L[n].desc.refine = None

    def set_lm_head(self, lm_fp16: torch.Tensor):
        self.lm_head = lm_fp16.contiguous()
        kv = self.layers[0]["kv"]
        need = kv.attend_workspace(self.T + 1, self.cfg.h_q, self.cfg.k_tok, False)
        self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=self.dev)

    # ---- the step ----------------------------------------------------------

    def _select(self, name, x, slot, stream):
        cfg = self.cfg
        check(abi.sf_select_channels(_p(x), self.B, self.shp[name][1], cfg.chunk, cfg.kch,
                                     _p(self.sel[name][slot]), _s(stream)), "sf_select_channels")

    def _stage(self, layer, name, slot, done):
        """Copy layer `layer`'s rows of the selection in `slot` into staging
        slot `slot` on the projection's staging stream (after the selection);
        `done` is recorded once the projection may use them."""
        side = self.stage_stream[name]
        if self.use_cache:
            arr, _ = self.caches[layer][name]
            check(abi.sf_stage_refinements_cached(_p(self.host_rows[layer][name]), self.row_bytes[name],
                                                  self.shp[name][1], _p(self.sel[name][slot]), self.n_sel[name],
                                                  self.B, arr, int(self.cfg.skip_missing), _p(self.slots[name][slot]),
                                                  _p(self.sel_eff[name][slot]), _s(side),
                                                  ctypes.c_void_p(done.cuda_event)),
                  "sf_stage_refinements_cached")
            return
        check(abi.sf_stage_refinements(_p(self.host_rows[layer][name]), self.row_bytes[name],
                                       self.shp[name][1], _p(self.sel[name][slot]), self.B * self.n_sel[name],
                                       _p(self.slots[name][slot]), None, _s(side), None),
              "sf_stage_refinements")
        done.record(side)

    def _side_select_stage(self, layer, name, x, slot, main):
        """Selection from x and the row transfer, both on the projection's
        staging stream; the event ev_stage[name][slot] marks both done."""
        side = self.stage_stream[name]
        ev = self.ev_sel[name][slot]
        ev.record(main)
        side.wait_event(ev)
        self._select(name, x, slot, side)
        if self.slots is not None:
            self._stage(layer, name, slot, self.ev_stage[name][slot])
        else:
            self.ev_stage[name][slot].record(side)

    def _ready(self, name, slot, main):
        """Wait (on the main stream) for the selection and rows in `slot`."""
        main.wait_event(self.ev_stage[name][slot])
        return self.slots[name][slot] if self.slots is not None else None

    def _proj(self, layer, name, x, y, slot, main, y_corr=None):
        """y = W~ x for layer `layer` with the selection in `slot`; with y_corr,
        y gets the base product and y_corr the correction (fetch lag)."""
        cfg = self.cfg
        qw = self.layers[layer][name]
        if cfg.kch == 0:
            check(abi.sf_gemv_refined(ctypes.byref(qw.desc), _p(x), self.B, cfg.chunk, 0, None, None, None,
                                      _p(y), _p(self.gemv_ws), self.gemv_ws.numel(), _s(main)), "sf_gemv_refined")
            return
        rows = self._ready(name, slot, main)
        sel = self.sel_eff[name][slot] if self.use_cache else self.sel[name][slot]
        if self.trace is not None:
            self.trace.append((("w", layer, name), sel.clone()))
        if y_corr is not None:
            check(abi.sf_gemv_refined_split(ctypes.byref(qw.desc), _p(x), self.B, cfg.chunk, cfg.kch,
                                            _p(sel), _p(rows), _p(y), _p(y_corr), _s(main)),
                  "sf_gemv_refined_split")
            return
        check(abi.sf_gemv_refined(ctypes.byref(qw.desc), _p(x), self.B, cfg.chunk, cfg.kch,
                                  _p(sel), None, _p(rows), _p(y), _p(self.gemv_ws),
                                  self.gemv_ws.numel(), _s(main)),
              "sf_gemv_refined")

    def _prepare(self, layer, name, x, main):
        """Without lead (or at layer 0) the projection selects from its own
        input: selection and transfer now, the projection waits for them."""
        cfg = self.cfg
        if cfg.kch == 0:
            return
        if not cfg.lead or layer == 0:
            self._side_select_stage(layer, name, x, layer % 2, main)

    def _lead(self, layer, name, x, main):
        """Fetch lead: select (layer + 1)'s channels from this activation and
        start their transfer on the projection's staging stream."""
        cfg = self.cfg
        if cfg.kch == 0 or not cfg.lead or layer + 1 >= cfg.n_layers:
            return
        self._side_select_stage(layer + 1, name, x, (layer + 1) % 2, main)

    def step(self, hidden: torch.Tensor):
        """Enqueue one decode step: hidden fp16 [B][hidden] -> self.logits."""
        cfg = self.cfg
        main = torch.cuda.current_stream(self.dev)
        self.side.wait_stream(main)
        self.side2.wait_stream(main)
        B, T = self.B, self.T
        check(abi.sf_widen_f16(_p(hidden), B * cfg.hidden, _p(self.h), _s(main)), "sf_widen_f16")
        add = None
        lagging = cfg.kch > 0 and bool(cfg.lag)
        delta = None  # the previous layer's lagged o correction
        for l in range(cfg.n_layers):
            slot = l % 2
            L = self.layers[l]
            x_attn, x_o, x_mlp, x_down = self.x_attn[slot], self.x_o[slot], self.x_mlp[slot], self.x_down[slot]
            check(abi.sf_rmsnorm_residual(_p(self.h), _p(add), _p(delta), B, cfg.hidden, cfg.eps, _p(x_attn),
                                          _s(main)), "sf_rmsnorm_residual")
            # attention block
            self._prepare(l, "qkv", x_attn, main)
            self._lead(l, "qkv", x_attn, main)
            self._proj(l, "qkv", x_attn, self.qkv_out, slot, main)
            kv = L["kv"]
            # rotary embedding of q and k and the new token's append, in one launch
            check(abi.sf_kv_append_rope(ctypes.byref(kv.desc), _p(self.qkv_out), cfg.h_q, T, cfg.theta, T,
                                        _p(self.q), _s(main)), "sf_kv_append_rope")
            # attention over T + 1 tokens; its fp16 output is o's input
            check(abi.sf_kv_attend_selective_f16(ctypes.byref(kv.desc), T + 1, _p(self.q), cfg.h_q, cfg.k_tok,
                                                 _p(self.tok_sel), None, _p(x_o), _p(self.ws), self.ws.numel(),
                                                 _s(main)), "sf_kv_attend_selective_f16")
            if self.trace is not None:
                self.trace.append((("tok", l), self.tok_sel.clone()))
            self._prepare(l, "o", x_o, main)
            self._lead(l, "o", x_o, main)
            self._proj(l, "o", x_o, self.o_out, slot, main, y_corr=self.delta if lagging else None)
            check(abi.sf_rmsnorm_residual(_p(self.h), _p(self.o_out), None, B, cfg.hidden, cfg.eps,
                                          _p(x_mlp), _s(main)), "sf_rmsnorm_residual")
            # MLP block
            self._prepare(l, "gate_up", x_mlp, main)
            self._lead(l, "gate_up", x_mlp, main)
            self._proj(l, "gate_up", x_mlp, self.gu_out, slot, main)
            check(abi.sf_silu_mul(_p(self.gu_out), B, cfg.inter, _p(x_down), _s(main)), "sf_silu_mul")
            self._prepare(l, "down", x_down, main)
            self._lead(l, "down", x_down, main)
            self._proj(l, "down", x_down, self.down_out, slot, main)  # its lagged correction lands with it
            add = self.down_out
            delta = self.delta if lagging else None
        check(abi.sf_rmsnorm_residual(_p(self.h), _p(add), _p(delta), B, cfg.hidden, cfg.eps, _p(self.x_final),
                                      _s(main)), "sf_rmsnorm_residual")
        check(abi.sf_gemv_f16(_p(self.lm_head), _p(self.x_final), B, cfg.vocab, cfg.hidden, _p(self.logits),
                              _s(main)), "sf_gemv_f16")
        main.wait_stream(self.side)
        main.wait_stream(self.side2)
        return self.logits
