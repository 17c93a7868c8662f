"""Torch-facing helpers over the C ABI: they allocate caller-owned buffers with
PyTorch (device memory and streams are all PyTorch is used for) and pass raw
pointers to the CUDA library.  No arithmetic of the method happens here."""
from __future__ import annotations

import ctypes

import torch

from . import abi
from .abi import check


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _f16(t: torch.Tensor) -> torch.Tensor:
    assert t.dtype in (torch.float16, torch.int16, torch.uint16), t.dtype
    assert t.is_cuda and t.is_contiguous()
    return t


class QuantWeights:
    """A nested-quantised weight matrix W[n][k] (format: include/sf.h, sf_wq)."""

    def __init__(self, n: int, k: int, b: int, r: int, group: int = 128, device="cuda",
                 with_refine: bool = True):
        sizes = [ctypes.c_size_t() for _ in range(3)]
        check(abi.sf_wq_bytes(n, k, b, r, group, *[ctypes.byref(s) for s in sizes]), "sf_wq_bytes")
        self.n, self.k, self.b, self.r, self.group = n, k, b, r, group
        self.base = torch.empty(sizes[0].value, dtype=torch.uint8, device=device)
        self.refine = torch.empty(sizes[1].value, dtype=torch.uint8, device=device) if with_refine else None
        self.sz = torch.empty(sizes[2].value // 2, dtype=torch.int16, device=device)
        self.desc = abi.sf_wq(n, k, b, r, group, self.base.data_ptr(),
                              self.refine.data_ptr() if with_refine else None, self.sz.data_ptr())

    @classmethod
    def pack(cls, w: torch.Tensor, b: int, r: int, group: int = 128) -> "QuantWeights":
        assert w.dtype == torch.float32 and w.is_cuda and w.is_contiguous() and w.dim() == 2
        q = cls(w.shape[0], w.shape[1], b, r, group, device=w.device)
        check(abi.sf_pack_nested(_p(w), ctypes.byref(q.desc), _stream()), "sf_pack_nested")
        return q

    def fit_refinements(self, w: torch.Tensor, x_cal: torch.Tensor, chunk: int = 1024, kch: int = 32,
                        alpha: float = 0.01, want_delta: bool = False, stream=None):
        """Refit the refinement codes on calibration activations x_cal [n_cal][k]
        (sf_fit_refinements); w is the fp32 matrix this one was packed from.
        Returns the fitted corrections [n][k] fp64 when want_delta."""
        assert w.dtype == torch.float32 and w.is_contiguous() and tuple(w.shape) == (self.n, self.k)
        x_cal = _f16(x_cal)
        n_cal = x_cal.shape[0]
        nbytes = abi.sf_fit_refinements_workspace_bytes(self.n, self.k, n_cal, chunk, kch)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=w.device)
        delta = torch.empty((self.n, self.k), dtype=torch.float64, device=w.device) if want_delta else None
        check(abi.sf_fit_refinements(_p(w), ctypes.byref(self.desc), _p(x_cal), n_cal, chunk, kch, alpha, _p(delta),
                                     _p(ws), nbytes, _stream(stream)), "sf_fit_refinements")
        return delta

    def refine_rows(self) -> torch.Tensor:
        """The refinement buffer viewed as [k][n*r/8] rows (one per input channel)."""
        return self.refine.view(self.k, self.n * self.r // 8)

    def unpack(self):
        qb = torch.empty((self.n, self.k), dtype=torch.uint8, device=self.base.device)
        rho = torch.empty_like(qb) if self.refine is not None else None
        check(abi.sf_unpack_codes(ctypes.byref(self.desc), _p(qb), _p(rho), _stream()), "sf_unpack_codes")
        return qb, rho

    def gemv(self, x: torch.Tensor, chunk: int = 1024, kch: int = 32, sel_in=None,
             refine_rows=None, y=None, sel_out=None, ws=None, stream=None):
        """y = W~ x (sf_gemv_refined).  Returns (y [batch][n] fp32, selection)."""
        x = _f16(x if x.dim() == 2 else x.view(1, -1))
        batch = x.shape[0]
        if y is None:
            y = torch.empty((batch, self.n), dtype=torch.float32, device=x.device)
        if kch > 0 and sel_in is None and sel_out is None:
            sel_out = torch.empty((batch, self.k // chunk, kch), dtype=torch.int32, device=x.device)
        if ws is None:
            need = abi.sf_gemv_workspace_bytes(ctypes.byref(self.desc), batch, chunk, kch)
            ws = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
        check(abi.sf_gemv_refined(ctypes.byref(self.desc), _p(x), batch, chunk, kch, _p(sel_in),
                                  _p(sel_out), _p(refine_rows), _p(y), _p(ws), ws.numel(), _stream(stream)),
              "sf_gemv_refined")
        return y, (sel_in if sel_in is not None else sel_out)

    def correction(self, x: torch.Tensor, sel, y, chunk: int = 1024, kch: int = 32,
                   refine_rows=None, stream=None):
        """y += (W~ - W^) x over the selected channels (sf_gemv_correction)."""
        x = _f16(x if x.dim() == 2 else x.view(1, -1))
        check(abi.sf_gemv_correction(ctypes.byref(self.desc), _p(x), x.shape[0], chunk, kch, _p(sel),
                                     _p(refine_rows), _p(y), _stream(stream)),
              "sf_gemv_correction")
        return y


    def gemv_split(self, x: torch.Tensor, sel, chunk: int = 1024, kch: int = 32, refine_rows=None,
                   y_base=None, y_corr=None, stream=None):
        """Base product and correction to separate outputs (sf_gemv_refined_split).
        Returns (y_base, y_corr), each [batch][n] fp32."""
        x = _f16(x if x.dim() == 2 else x.view(1, -1))
        batch = x.shape[0]
        if y_base is None:
            y_base = torch.empty((batch, self.n), dtype=torch.float32, device=x.device)
        if y_corr is None:
            y_corr = torch.empty((batch, self.n), dtype=torch.float32, device=x.device)
        check(abi.sf_gemv_refined_split(ctypes.byref(self.desc), _p(x), batch, chunk, kch, _p(sel),
                                        _p(refine_rows), _p(y_base), _p(y_corr), _stream(stream)),
              "sf_gemv_refined_split")
        return y_base, y_corr


def select_channels(x: torch.Tensor, chunk: int = 1024, kch: int = 32, sel=None, stream=None):
    x = _f16(x if x.dim() == 2 else x.view(1, -1))
    batch, k = x.shape
    if sel is None:
        sel = torch.empty((batch, k // chunk, kch), dtype=torch.int32, device=x.device)
    check(abi.sf_select_channels(_p(x), batch, k, chunk, kch, _p(sel), _stream(stream)),
          "sf_select_channels")
    return sel


class KVCache:
    """`batch` nested-quantised KV caches (format: include/sf.h, sf_kv)."""

    def __init__(self, batch: int, h_kv: int, t_max: int, b: int = 2, r: int = 2, d: int = 128,
                 group: int = 32, device="cuda"):
        sizes = [ctypes.c_size_t() for _ in range(3)]
        check(abi.sf_kv_bytes(batch, h_kv, d, t_max, b, r, group, *[ctypes.byref(s) for s in sizes]),
              "sf_kv_bytes")
        mk = lambda nbytes: torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.batch, self.h_kv, self.t_max, self.b, self.r, self.d, self.group = batch, h_kv, t_max, b, r, d, group
        self.kb, self.kr, self.vb, self.vr = mk(sizes[0].value), mk(sizes[1].value), mk(sizes[0].value), mk(sizes[1].value)
        self.ksz = torch.zeros(sizes[2].value // 2, dtype=torch.int16, device=device)
        self.vsz = torch.zeros(sizes[2].value // 2, dtype=torch.int16, device=device)
        self.desc = abi.sf_kv(batch, h_kv, d, t_max, b, r, group, self.kb.data_ptr(), self.kr.data_ptr(),
                              self.vb.data_ptr(), self.vr.data_ptr(), self.ksz.data_ptr(), self.vsz.data_ptr())

    def pack_tokens(self, k, v, t0: int, stream=None):
        """k, v: [batch][h_kv][nt][d] fp16 (either may be None)."""
        nt = (k if k is not None else v).shape[2]
        check(abi.sf_kv_pack_tokens(ctypes.byref(self.desc), _p(k), _p(v), t0, nt, _stream(stream)),
              "sf_kv_pack_tokens")

    def unpack(self, which: int, t: int):
        dev = self.kb.device
        qb = torch.empty((self.batch, self.h_kv, t, self.d), dtype=torch.uint8, device=dev)
        rho = torch.empty_like(qb)
        check(abi.sf_kv_unpack_codes(ctypes.byref(self.desc), which, t, _p(qb), _p(rho), _stream()),
              "sf_kv_unpack_codes")
        return qb, rho

    def score_select_workspace(self, t: int, h_q: int, k_tok: int, logits_given: bool) -> int:
        return abi.sf_kv_score_select_workspace_bytes(ctypes.byref(self.desc), t, h_q, k_tok,
                                                      int(logits_given))

    def score_select(self, q: torch.Tensor, t: int, k_tok: int, logits=None, scores=None,
                     want_logits: bool = True, want_scores: bool = False, sel=None, ws=None,
                     stream=None):
        q = _f16(q)
        h_q = q.shape[1]
        dev = q.device
        if logits is None and want_logits:
            logits = torch.empty((self.batch, h_q, t), dtype=torch.float32, device=dev)
        if scores is None and want_scores:
            scores = torch.empty((self.batch, self.h_kv, t), dtype=torch.float32, device=dev)
        if sel is None:
            sel = torch.empty((self.batch, self.h_kv, k_tok), dtype=torch.int32, device=dev)
        need = self.score_select_workspace(t, h_q, k_tok, logits is not None)
        if ws is None:
            ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        check(abi.sf_kv_score_select(ctypes.byref(self.desc), t, _p(q), h_q, k_tok, _p(sel), _p(logits),
                                     _p(scores), _p(ws), ws.numel(), _stream(stream)),
              "sf_kv_score_select")
        return sel, logits, scores

    def logits_fma(self, q: torch.Tensor, t: int, logits=None, ws=None, stream=None):
        """The base logits on the CUDA cores (sf_kv_logits_fma): [batch][h_q][t] fp32."""
        q = _f16(q)
        h_q = q.shape[1]
        if logits is None:
            logits = torch.empty((self.batch, h_q, t), dtype=torch.float32, device=q.device)
        need = abi.sf_kv_logits_fma_workspace_bytes(ctypes.byref(self.desc), t, h_q)
        if ws is None:
            ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        check(abi.sf_kv_logits_fma(ctypes.byref(self.desc), t, _p(q), h_q, _p(logits), _p(ws), ws.numel(),
                                   _stream(stream)), "sf_kv_logits_fma")
        return logits

    def attn_workspace(self, t: int, h_q: int, k_tok: int, n_splits: int = 0) -> int:
        return abi.sf_kv_attn_workspace_bytes(ctypes.byref(self.desc), t, h_q, k_tok, n_splits)

    def attn_refined(self, q: torch.Tensor, t: int, sel, k_tok: int, n_splits: int = 0, out=None,
                     ws=None, stream=None):
        q = _f16(q)
        h_q = q.shape[1]
        if out is None:
            out = torch.empty((self.batch, h_q, self.d), dtype=torch.float32, device=q.device)
        need = self.attn_workspace(t, h_q, k_tok, n_splits)
        if ws is None:
            ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        check(abi.sf_kv_attn_refined(ctypes.byref(self.desc), t, _p(q), h_q, _p(sel), k_tok, n_splits,
                                     _p(out), _p(ws), ws.numel(), _stream(stream)),
              "sf_kv_attn_refined")
        return out

    def attend_workspace(self, t: int, h_q: int, k_tok: int, logits_given: bool) -> int:
        return abi.sf_kv_attend_selective_workspace_bytes(ctypes.byref(self.desc), t, h_q, k_tok,
                                                          int(logits_given))

    def attend_selective(self, q: torch.Tensor, t: int, k_tok: int, sel=None, logits=None,
                         out=None, ws=None, stream=None):
        """Score, select and attend in one call.  Returns (out, sel)."""
        q = _f16(q)
        h_q = q.shape[1]
        dev = q.device
        if out is None:
            out = torch.empty((self.batch, h_q, self.d), dtype=torch.float32, device=dev)
        if sel is None:
            sel = torch.empty((self.batch, self.h_kv, k_tok), dtype=torch.int32, device=dev)
        need = self.attend_workspace(t, h_q, k_tok, logits is not None)
        if ws is None:
            ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        check(abi.sf_kv_attend_selective(ctypes.byref(self.desc), t, _p(q), h_q, k_tok, _p(sel),
                                         _p(logits), _p(out), _p(ws), ws.numel(), _stream(stream)),
              "sf_kv_attend_selective")
        return out, sel
