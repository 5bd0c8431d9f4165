"""thinned_softmax_attention_b200 -- Thinformer and Thinformer Express attention on B200 (sm_100a).

A thin Python binding over the C ABI declared in ``include/thin_attn.h``: it
only marshals arguments (device pointers of torch tensors, the current CUDA
stream).  Every step of the computation runs in the CUDA library
``libthin_attn.so``; if that library is missing the binding raises instead of
falling back to anything else.

Layouts follow the Thinformer README ("Getting Started"):
    query (B, T, H, E), key (B, S, H, E), value (B, S, H, D)  ->  attn_output (B, T, H, D)
with ``causal=True`` meaning Thinformer Express prefill (S = T).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Dict, Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libthin_attn.so")

FP32, BF16 = 0, 1
_STATUS = {0: "OK", 1: "EINVAL", 2: "ENOMEM", 3: "ECUDA", 4: "ETIMEOUT", 5: "EUNSUPPORTED"}


class ThinAttnError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"thin_attn {_STATUS.get(status, status)}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("B", ctypes.c_int), ("T", ctypes.c_int), ("S", ctypes.c_int),
                ("H", ctypes.c_int), ("E", ctypes.c_int), ("D", ctypes.c_int), ("scale", ctypes.c_float),
                ("n_exact", ctypes.c_int), ("batch", ctypes.c_int), ("device", ctypes.c_int),
                ("b0", ctypes.c_int), ("h0", ctypes.c_int), ("H_total", ctypes.c_int), ("qk_fp8", ctypes.c_int),
                ("q_begin", ctypes.c_int), ("q_end", ctypes.c_int), ("thin_split", ctypes.c_int)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("levels", ctypes.c_int), ("leaf", ctypes.c_int), ("subsampled", ctypes.c_int),
                ("coreset_rows", ctypes.c_int), ("n_batches", ctypes.c_int), ("n_nodes", ctypes.c_int),
                ("n_halvings", ctypes.c_int), ("kernel_launches", ctypes.c_int), ("trace_words", ctypes.c_uint64),
                ("coreset_idx_elems", ctypes.c_uint64), ("workspace_bytes", ctypes.c_uint64), ("attn_rows", ctypes.c_int)]


class TraceEntry(ctypes.Structure):
    _fields_ = [("bh", ctypes.c_uint32), ("round_id", ctypes.c_uint32), ("pair0", ctypes.c_uint32),
                ("n_pairs", ctypes.c_uint32), ("word_offset", ctypes.c_uint64)]


_lib = None
EXPORTS = ("thin_attn_version", "thin_attn_last_error", "thin_attn_create", "thin_attn_destroy",
           "thin_attn_plan", "thin_attn_reserve", "thin_attn_trace_layout", "thin_attn_forward",
           "thin_attn_forward_host", "thin_attn_check", "thin_attn_profile", "thin_attn_profile_read",
           "thin_attn_profile_steps",
           "thin_attn_cache_create", "thin_attn_cache_destroy", "thin_attn_cache_length", "thin_attn_cache_decode",
           "thin_attn_cache_nodes", "thin_attn_cache_check", "thin_attn_sched_layout", "thin_attn_cache_decode_n",
           "thin_attn_forward_phase", "thin_attn_nodes_layout", "thin_attn_nodes_export", "thin_attn_nodes_import")


def lib() -> ctypes.CDLL:
    """Load libthin_attn.so (built in-tree by ``python -m thinned_softmax_attention_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m thinned_softmax_attention_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64
    L.thin_attn_version.restype = ctypes.c_char_p
    L.thin_attn_last_error.restype = ctypes.c_char_p
    L.thin_attn_create.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(Config)]
    L.thin_attn_destroy.argtypes = [vp]
    L.thin_attn_plan.argtypes = [vp, i, i, ctypes.POINTER(PlanInfo)]
    L.thin_attn_reserve.argtypes = [vp, i, i]
    L.thin_attn_trace_layout.argtypes = [vp, i, i, ctypes.POINTER(TraceEntry), ctypes.c_size_t,
                                         ctypes.POINTER(ctypes.c_size_t)]
    L.thin_attn_forward.argtypes = [vp, vp, vp, vp, vp, i, i, u64, vp, vp, vp, vp]
    L.thin_attn_forward_host.argtypes = [vp, vp, vp, vp, vp, i, i, u64, vp, vp]
    L.thin_attn_check.argtypes = [vp, vp]
    L.thin_attn_cache_create.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(Config), i, u64]
    L.thin_attn_cache_destroy.argtypes = [vp]
    L.thin_attn_cache_length.argtypes = [vp, ctypes.POINTER(ctypes.c_int64)]
    L.thin_attn_cache_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp]
    L.thin_attn_cache_decode_n.argtypes = [vp, vp, vp, vp, vp, vp, i, vp]
    L.thin_attn_cache_nodes.argtypes = [vp, vp, vp]
    L.thin_attn_cache_check.argtypes = [vp, vp]
    sz = ctypes.c_size_t
    L.thin_attn_sched_layout.argtypes = [vp, i, i, vp, vp, vp, sz, sz, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.thin_attn_profile.argtypes = [vp, i]
    L.thin_attn_profile_read.argtypes = [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]
    ip = ctypes.POINTER(ctypes.c_int)
    L.thin_attn_profile_steps.argtypes = [vp, i, ctypes.POINTER(ctypes.c_double), ip, ip, ip, ip]
    for f in EXPORTS[2:]:
        getattr(L, f).restype = ctypes.c_int
    _lib = L
    return L


def _check(status: int):
    if status != 0:
        raise ThinAttnError(status, lib().thin_attn_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class ThinAttention:
    """One problem shape on one device: Thinformer (non-causal) and Thinformer Express (causal).

    ``forward(q, k, v, causal, g, seed)`` returns a dict: ``out`` (B,T,H,D) and, on request,
    ``lse`` (B,H,T) fp32, the log-sum-exp ln sum_j w_j e^{s q.k_j} (``return_lse=True``),
    ``coreset`` int32 token indices (``return_coreset=True``: (B,H,|C|), or (B,H,n_nodes,c) when
    causal) and ``trace``, one bit per halving decision (``return_trace=True``).  The dense
    attention weights are never formed; the layer call ``thinformer_attention`` returns
    ``(attn_output, None)``.

    ``qk_fp8=True``: QK^T in e4m3 with one scale per (b,h) for q and for k (E = 128, bf16); the
    thinning keeps the bf16 keys.

    ``shard=(b0, h0, H_total)``: the tensors hold batch rows [b0, b0 + B) and heads
    [h0, h0 + H) of a larger problem with H_total heads (one handle per GPU of a batch- or
    head-parallel run); the random decisions, and so every output, equal the whole
    problem's for those (b,h).

    ``q_range=(q_begin, q_end)``: attend only query rows [q_begin, q_end) (multiples of 128; the
    end may be T) of every (b,h); the thinning runs over all keys, so those rows equal the whole
    run's and the other rows of ``out`` and ``lse`` are left as they were (sequence-parallel
    shards of one long sequence, one per GPU, with no communication).

    ``thin_split=True`` (Express, with ``q_range``): the handle thins only the batches whose last
    token lies in its range; a forward is ``forward_phase(..., phase=1)``, an exchange of the batch
    coresets (``nodes_export`` on every rank, an all-gather, ``nodes_import`` of the others'), then
    ``forward_phase(..., phase=2)`` (see ``exchange_batch_coresets``).
    """

    def __init__(self, B: int, T: int, S: int, H: int, E: int, D: int, dtype: torch.dtype,
                 scale: Optional[float] = None, n_exact: int = 0, batch: int = 0, device: int = 0,
                 shard: Tuple[int, int, int] = (0, 0, 0), qk_fp8: bool = False,
                 q_range: Tuple[int, int] = (0, 0), thin_split: bool = False):
        self.cfg = Config(FP32 if dtype == torch.float32 else BF16, B, T, S, H, E, D,
                          0.0 if scale is None else float(scale), n_exact, batch, device, *shard, int(qk_fp8),
                          *q_range, int(thin_split))
        self.dtype = dtype
        self.device = torch.device("cuda", device)
        self._h = ctypes.c_void_p()
        _check(lib().thin_attn_create(ctypes.byref(self._h), ctypes.byref(self.cfg)))

    def close(self):
        if self._h:
            lib().thin_attn_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def plan(self, causal: bool, g: int) -> Dict[str, int]:
        info = PlanInfo()
        _check(lib().thin_attn_plan(self._h, int(causal), g, ctypes.byref(info)))
        return {f: getattr(info, f) for f, _ in PlanInfo._fields_}

    def sched_layout(self, causal: bool, g: int):
        """Work items of the persistent halving launch: (trace entry of each item in queue order,
        list of predecessor item indices per item); empty when every step runs on its own."""
        ni, npr = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().thin_attn_sched_layout(self._h, int(causal), g, None, None, None, 0, 0, ctypes.byref(ni),
                                            ctypes.byref(npr)))
        ent = (ctypes.c_int32 * max(1, ni.value))()
        off = (ctypes.c_int32 * (ni.value + 1))()
        prd = (ctypes.c_int32 * max(1, npr.value))()
        _check(lib().thin_attn_sched_layout(self._h, int(causal), g, ent, off, prd, ni.value, npr.value,
                                            ctypes.byref(ni), ctypes.byref(npr)))
        return list(ent[:ni.value]), [list(prd[off[i]:off[i + 1]]) for i in range(ni.value)]

    def reserve(self, causal: bool, g: int):
        _check(lib().thin_attn_reserve(self._h, int(causal), g))

    def trace_layout(self, causal: bool, g: int):
        n = ctypes.c_size_t()
        _check(lib().thin_attn_trace_layout(self._h, int(causal), g, None, 0, ctypes.byref(n)))
        arr = (TraceEntry * max(1, n.value))()
        _check(lib().thin_attn_trace_layout(self._h, int(causal), g, arr, n.value, ctypes.byref(n)))
        return [(e.bh, e.round_id, e.pair0, e.n_pairs, e.word_offset) for e in arr[:n.value]]

    def forward(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False, g: int = 2,
                seed: int = 0, return_lse: bool = False, return_coreset: bool = False,
                return_trace: bool = False, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
        """``out`` and ``lse`` (B,H,T fp32) may be the caller's buffers (a query-row shard writes only its
        rows of them); ``lse`` given implies ``return_lse``."""
        c = self.cfg
        L = c.T if causal else c.S
        for name, t, shape in (("q", q, (c.B, c.T, c.H, c.E)), ("k", k, (c.B, L, c.H, c.E)),
                               ("v", v, (c.B, L, c.H, c.D))):
            if tuple(t.shape) != shape or t.dtype != self.dtype or not t.is_contiguous() or t.device != self.device:
                raise ValueError(f"{name}: expected contiguous {self.dtype} {shape} on {self.device}, "
                                 f"got {t.dtype} {tuple(t.shape)} on {t.device}")
        if out is None:
            out = torch.empty(c.B, c.T, c.H, c.D, dtype=self.dtype, device=self.device)
        info = self.plan(causal, g)
        if lse is not None:
            if tuple(lse.shape) != (c.B, c.H, c.T) or lse.dtype != torch.float32 or not lse.is_contiguous():
                raise ValueError(f"lse: expected contiguous float32 {(c.B, c.H, c.T)}, got {lse.dtype} {tuple(lse.shape)}")
            return_lse = True
        elif return_lse:
            lse = torch.empty(c.B, c.H, c.T, dtype=torch.float32, device=self.device)
        cidx = (torch.empty(max(1, info["coreset_idx_elems"]), dtype=torch.int32, device=self.device)
                if return_coreset else None)
        trace = (torch.zeros(max(1, info["trace_words"]), dtype=torch.int32, device=self.device)
                 if return_trace else None)
        stream = torch.cuda.current_stream(self.device).cuda_stream
        _check(lib().thin_attn_forward(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(out), int(causal), g,
                                       ctypes.c_uint64(seed & (2 ** 64 - 1)), _ptr(lse), _ptr(cidx), _ptr(trace),
                                       ctypes.c_void_p(stream)))
        res = {"out": out}
        if return_lse:
            res["lse"] = lse
        if return_coreset:
            n = info["coreset_idx_elems"]
            if causal:
                res["coreset"] = cidx[:n].view(c.B, c.H, info["n_nodes"], info["coreset_rows"])
            else:
                res["coreset"] = cidx[:n].view(c.B, c.H, info["coreset_rows"])
        if return_trace:
            res["trace"] = trace
        return res

    def forward_phase(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, phase: int, g: int = 2, seed: int = 0,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      return_coreset: bool = False, return_trace: bool = False):
        """One phase of a thin_split handle's Express forward: 1 thins the owned batches, 2 runs the
        merges and the attention of the query-row range (after the batch coresets are exchanged)."""
        c = self.cfg
        for name, t, shape in (("q", q, (c.B, c.T, c.H, c.E)), ("k", k, (c.B, c.T, c.H, c.E)),
                               ("v", v, (c.B, c.T, c.H, c.D))):
            if tuple(t.shape) != shape or t.dtype != self.dtype or not t.is_contiguous() or t.device != self.device:
                raise ValueError(f"{name}: expected contiguous {self.dtype} {shape} on {self.device}")
        if out is None:
            out = torch.empty(c.B, c.T, c.H, c.D, dtype=self.dtype, device=self.device)
        info = self.plan(True, g)
        cidx = (torch.empty(max(1, info["coreset_idx_elems"]), dtype=torch.int32, device=self.device)
                if return_coreset else None)
        trace = (torch.zeros(max(1, info["trace_words"]), dtype=torch.int32, device=self.device)
                 if return_trace else None)
        stream = torch.cuda.current_stream(self.device).cuda_stream
        _check(lib().thin_attn_forward_phase(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(out), 1, g,
                                             ctypes.c_uint64(seed & (2 ** 64 - 1)), _ptr(lse), _ptr(cidx), _ptr(trace),
                                             int(phase), ctypes.c_void_p(stream)))
        res = {"out": out}
        if lse is not None:
            res["lse"] = lse
        if return_coreset:
            n = info["coreset_idx_elems"]
            res["coreset"] = cidx[:n].view(c.B, c.H, info["n_nodes"], info["coreset_rows"])
        if return_trace:
            res["trace"] = trace
        return res

    def nodes_layout(self, g: int = 2):
        """(own_begin, own_end, n_batches, bytes_per_batch) of the Express batch coresets."""
        k0, k1, nb, bpb = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_uint64()
        _check(lib().thin_attn_nodes_layout(self._h, 1, g, ctypes.byref(k0), ctypes.byref(k1), ctypes.byref(nb),
                                            ctypes.byref(bpb)))
        return k0.value, k1.value, nb.value, bpb.value

    def nodes_export(self, dst: torch.Tensor, g: int = 2):
        """The owned batches' coreset blocks into ``dst`` (uint8 on this device)."""
        k0, k1, _, bpb = self.nodes_layout(g)
        if dst.device != self.device or dst.dtype != torch.uint8 or dst.numel() < (k1 - k0) * bpb:
            raise ValueError("dst: uint8 on the handle's device, (own_end - own_begin) * bytes_per_batch bytes")
        stream = torch.cuda.current_stream(self.device).cuda_stream
        _check(lib().thin_attn_nodes_export(self._h, 1, g, _ptr(dst), ctypes.c_void_p(stream)))

    def nodes_import(self, src: torch.Tensor, batch_begin: int, batch_end: int, g: int = 2):
        """Write batches [batch_begin, batch_end)'s coreset blocks from ``src`` into this handle."""
        _, _, _, bpb = self.nodes_layout(g)
        if src.device != self.device or src.dtype != torch.uint8 or src.numel() < (batch_end - batch_begin) * bpb:
            raise ValueError("src: uint8 on the handle's device, one block per batch")
        stream = torch.cuda.current_stream(self.device).cuda_stream
        _check(lib().thin_attn_nodes_import(self._h, 1, g, _ptr(src), int(batch_begin), int(batch_end),
                                            ctypes.c_void_p(stream)))

    def forward_host(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                     causal: bool = False, g: int = 2, seed: int = 0, lse: Optional[torch.Tensor] = None):
        """Host tensors in, host tensors out (copies included); synchronises the current stream."""
        for t in (q, k, v, out):
            if t.device.type != "cpu" or not t.is_contiguous():
                raise ValueError("forward_host takes contiguous CPU tensors")
        stream = torch.cuda.current_stream(self.device).cuda_stream
        _check(lib().thin_attn_forward_host(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(out), int(causal), g,
                                            ctypes.c_uint64(seed & (2 ** 64 - 1)), _ptr(lse),
                                            ctypes.c_void_p(stream)))
        return out

    def profile(self, enable: bool = True):
        """Record per-phase CUDA events on every forward (thinning, merges, attention)."""
        _check(lib().thin_attn_profile(self._h, int(enable)))

    def profile_read(self):
        """Summed phase times (ms) of the forwards recorded since the last read, and their count."""
        ms = (ctypes.c_double * 4)()
        calls = ctypes.c_int()
        _check(lib().thin_attn_profile_read(self._h, ms, ctypes.byref(calls)))
        return {"thin_ms": ms[0], "merge_ms": ms[1], "attn_ms": ms[2], "total_ms": ms[3], "calls": calls.value}

    def profile_steps(self):
        """Summed device time (ms) of every halving step of the forwards recorded since the last
        call, in launch order, with each step's instances and points per instance."""
        cap = 64
        ms = (ctypes.c_double * cap)()
        ni, npt = (ctypes.c_int * cap)(), (ctypes.c_int * cap)()
        ns, calls = ctypes.c_int(), ctypes.c_int()
        _check(lib().thin_attn_profile_steps(self._h, cap, ms, ni, npt, ctypes.byref(ns), ctypes.byref(calls)))
        return {"calls": calls.value,
                "steps": [{"ms": ms[j], "n_inst": ni[j], "n": npt[j]} for j in range(min(ns.value, cap))]}

    def check(self):
        stream = torch.cuda.current_stream(self.device).cuda_stream
        _check(lib().thin_attn_check(self._h, ctypes.c_void_p(stream)))


class ThinAttentionCache:
    """Express decode cache: one token per (b,h) and call, attended like query t of the prefill.

    ``decode(q, k, v)`` takes (B,1,H,E), (B,1,H,E), (B,1,H,D) device tensors and returns the
    (B,1,H,D) attention output of the new token; completed batches are thinned and merged on the
    fly.  ``capacity`` bounds the number of tokens.
    """

    def __init__(self, B: int, H: int, E: int, D: int, dtype: torch.dtype, capacity: int, n_exact: int, batch: int,
                 g: int = 2, seed: int = 0, scale: Optional[float] = None, device: int = 0,
                 shard: Tuple[int, int, int] = (0, 0, 0)):
        self.cfg = Config(FP32 if dtype == torch.float32 else BF16, B, capacity, capacity, H, E, D,
                          0.0 if scale is None else float(scale), n_exact, batch, device, *shard)
        self.dtype, self.device = dtype, torch.device("cuda", device)
        self._h = ctypes.c_void_p()
        _check(lib().thin_attn_cache_create(ctypes.byref(self._h), ctypes.byref(self.cfg), g,
                                            ctypes.c_uint64(seed & (2 ** 64 - 1))))
        plan = ThinAttention(B, capacity, capacity, H, E, D, dtype, scale, n_exact, batch, device).plan(True, g)
        self.n_nodes, self.node_rows = plan["n_nodes"], plan["coreset_rows"]
        self._shapes = None

    def close(self):
        if self._h:
            lib().thin_attn_cache_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __len__(self):
        t = ctypes.c_int64()
        _check(lib().thin_attn_cache_length(self._h, ctypes.byref(t)))
        return t.value

    def decode(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None) -> torch.Tensor:
        c = self.cfg
        if self._shapes is None:
            self._shapes = ((c.B, 1, c.H, c.E), (c.B, 1, c.H, c.E), (c.B, 1, c.H, c.D))
            self._decode_fn = lib().thin_attn_cache_decode
        for name, t, shape in zip("qkv", (q, k, v), self._shapes):
            if t.shape != shape or t.dtype != self.dtype or not t.is_contiguous() or t.device != self.device:
                raise ValueError(f"{name}: expected contiguous {self.dtype} {shape} on {self.device}")
        if out is None:
            out = torch.empty(c.B, 1, c.H, c.D, dtype=self.dtype, device=self.device)
        stream = torch.cuda.current_stream(self.device).cuda_stream
        _check(self._decode_fn(self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               None if lse is None else lse.data_ptr(), stream))
        return out

    def decode_n(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None) -> torch.Tensor:
        """n consecutive tokens in one call: (B,n,H,E), (B,n,H,E), (B,n,H,D) -> (B,n,H,D); the same
        results as n calls of decode, without a host round trip per token.  ``lse``: (B,H,n) fp32."""
        c = self.cfg
        n = q.shape[1]
        for name, t, shape in (("q", q, (c.B, n, c.H, c.E)), ("k", k, (c.B, n, c.H, c.E)), ("v", v, (c.B, n, c.H, c.D))):
            if tuple(t.shape) != shape or t.dtype != self.dtype or not t.is_contiguous() or t.device != self.device:
                raise ValueError(f"{name}: expected contiguous {self.dtype} {shape} on {self.device}")
        if out is None:
            out = torch.empty(c.B, n, c.H, c.D, dtype=self.dtype, device=self.device)
        stream = torch.cuda.current_stream(self.device).cuda_stream
        _check(lib().thin_attn_cache_decode_n(self._h, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                              None if lse is None else lse.data_ptr(), n, stream))
        return out

    def nodes(self) -> torch.Tensor:
        """(B,H,n_nodes,c) token indices of every coreset slot (-1 while empty), the node order of
        ThinAttention.forward(causal=True, return_coreset=True)."""
        c = self.cfg
        n = c.B * c.H * self.n_nodes * self.node_rows
        rows = torch.full((max(1, n),), -1, dtype=torch.int32, device=self.device)
        stream = torch.cuda.current_stream(self.device).cuda_stream
        _check(lib().thin_attn_cache_nodes(self._h, _ptr(rows), ctypes.c_void_p(stream)))
        return rows[:n].view(c.B, c.H, self.n_nodes, self.node_rows)

    def check(self):
        stream = torch.cuda.current_stream(self.device).cuda_stream
        _check(lib().thin_attn_cache_check(self._h, ctypes.c_void_p(stream)))


def decode_trace(words, layout) -> Dict[Tuple[int, int], np.ndarray]:
    """Decision bits of every halving, keyed by (b*H+h, round id), over the Philox pair index."""
    w = np.asarray(words.cpu().numpy() if isinstance(words, torch.Tensor) else words).view(np.uint32)
    acc: Dict[Tuple[int, int], Dict[int, np.ndarray]] = {}
    for bh, rid, pair0, m, off in layout:
        nw = (m + 31) // 32
        bits = np.unpackbits(w[off:off + nw].astype("<u4").view(np.uint8), bitorder="little")[:m].astype(bool)
        acc.setdefault((bh, rid), {})[pair0] = bits
    return {key: np.concatenate([parts[p0] for p0 in sorted(parts)]) for key, parts in acc.items()}


_cache: Dict[tuple, ThinAttention] = {}


def thinformer_attention(query: torch.Tensor, key: torch.Tensor, value: torch.Tensor, causal: bool = False,
                         g: int = 2, seed: int = 0, n_exact: int = 1024, batch: int = 1024,
                         scale: Optional[float] = None):
    """Drop-in attention layer call: ``attn_output, attn_output_weights = thinformer_attention(q, k, v)``.

    ``attn_output_weights`` is always None (the dense weights are never formed).
    """
    B, T, H, E = query.shape
    S, D = key.shape[1], value.shape[3]
    dev = query.device.index or 0
    k_ = (B, T, S, H, E, D, query.dtype, scale, n_exact if causal else 0, batch if causal else 0, dev)
    if k_ not in _cache:
        _cache[k_] = ThinAttention(B, T, S, H, E, D, query.dtype, scale, n_exact if causal else 0,
                                   batch if causal else 0, dev)
    return _cache[k_].forward(query, key, value, causal=causal, g=g, seed=seed)["out"], None


class ThinformerAttention:
    """The README's layer: ``layer = ThinformerAttention(); out, weights = layer(query, key, value)``
    (query (B,T,H,E), key (B,S,H,E), value (B,S,H,D)) or ``layer(query, key, value, causal=True)``
    (S = T, Thinformer Express with an exact phase of ``n_exact`` tokens and thin batches of
    ``batch``).  ``weights`` is always None: the dense attention weights are never formed.  Every
    call with the same shapes reuses one handle (and its workspace) per device.
    """

    def __init__(self, g: int = 2, seed: int = 0, n_exact: int = 1024, batch: int = 1024,
                 scale: Optional[float] = None):
        self.g, self.seed, self.n_exact, self.batch, self.scale = g, seed, n_exact, batch, scale

    def __call__(self, query: torch.Tensor, key: torch.Tensor, value: torch.Tensor, causal: bool = False):
        return thinformer_attention(query, key, value, causal=causal, g=self.g, seed=self.seed,
                                    n_exact=self.n_exact, batch=self.batch, scale=self.scale)


__all__ = ["ThinAttention", "ThinAttentionCache", "ThinAttnError", "ThinformerAttention", "thinformer_attention",
           "decode_trace", "exchange_batch_coresets", "lib", "LIB_PATH", "EXPORTS"]


def exchange_batch_coresets(h: "ThinAttention", g: int = 2, dist=None):
    """Between phase 1 and phase 2 of thin_split handles: every rank's owned batch coresets reach
    every other rank.  With ``dist`` (torch.distributed, one handle per rank): one all-gather of the
    padded blocks over the process group.  ``h`` may also be a list of handles on this device (ranks
    emulated in one process), whose blocks are copied directly."""
    if isinstance(h, (list, tuple)):
        lays = [x.nodes_layout(g) for x in h]
        bufs = []
        for x, (k0, k1, _, bpb) in zip(h, lays):
            buf = torch.empty(max(1, (k1 - k0) * bpb), dtype=torch.uint8, device=x.device)
            if k1 > k0:
                x.nodes_export(buf, g)
            bufs.append(buf)
        for i, x in enumerate(h):
            for j, (k0, k1, _, bpb) in enumerate(lays):
                if j != i and k1 > k0:
                    x.nodes_import(bufs[j].to(x.device), k0, k1, g)
        return
    k0, k1, nb, bpb = h.nodes_layout(g)
    world = dist.get_world_size()
    rng = torch.tensor([k0, k1], dtype=torch.int64, device=h.device)
    ranges = [torch.empty_like(rng) for _ in range(world)]
    dist.all_gather(ranges, rng)
    ranges = [tuple(int(x) for x in r.tolist()) for r in ranges]
    kmax = max(b - a for a, b in ranges)
    if kmax == 0:
        return
    send = torch.zeros(kmax * bpb, dtype=torch.uint8, device=h.device)
    if k1 > k0:
        h.nodes_export(send, g)
    recv = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(recv, send)
    me = dist.get_rank()
    for r, (a, b) in enumerate(ranges):
        if r != me and b > a:
            h.nodes_import(recv[r], a, b, g)
