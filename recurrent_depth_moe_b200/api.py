"""Python entry points over librdt with torch tensors as device memory.

Each function checks tensor placement, dtype and contiguity, allocates outputs and
the workspace with torch (the library itself allocates nothing), and calls the
C ABI of the same name on the current CUDA stream.  There is no CPU or eager
fallback: without a CUDA device or without librdt.so every call raises.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from . import _native as N

_DT = {"fp32": (0, torch.float32), "bf16": (1, torch.bfloat16)}


def _require_cuda():
    if not torch.cuda.is_available():
        raise RuntimeError("recurrent_depth_moe_b200 needs a CUDA device (B200, sm_100a); no CPU path exists")
    return N.load()


def config_struct(cfg) -> N.rdt_config:
    """rdt_config from any object carrying the MythosConfig-style fields."""
    mla = cfg.attn_type == "mla"
    c = N.rdt_config()
    c.dim, c.n_heads = cfg.dim, cfg.n_heads
    c.n_kv_heads = cfg.n_kv_heads
    c.attn_type = 1 if mla else 0
    c.kv_lora_rank, c.q_lora_rank = cfg.kv_lora_rank, cfg.q_lora_rank
    c.qk_rope_head_dim, c.qk_nope_head_dim, c.v_head_dim = cfg.qk_rope_head_dim, cfg.qk_nope_head_dim, cfg.v_head_dim
    c.n_experts, c.n_shared_experts = cfg.n_experts, cfg.n_shared_experts
    c.top_k, c.expert_dim = cfg.n_experts_per_tok, cfg.expert_dim
    c.lora_rank, c.max_loop_iters, c.loop_dim = cfg.lora_rank, cfg.max_loop_iters, cfg.loop_dim
    c.rope_theta, c.loop_theta, c.norm_eps = cfg.rope_theta, cfg.loop_theta, cfg.norm_eps
    c.dtype = _DT[cfg.dtype][0]
    return c


def dense_config_struct(cfg, hidden: Optional[int] = None) -> N.rdt_config:
    """Config of a prelude/coda block: no routed experts, one dense SwiGLU of width 4*dim/3
    (or `hidden`, the padded width the weights are laid out with)."""
    c = config_struct(cfg)
    c.n_experts, c.top_k, c.n_shared_experts = 0, 0, 1
    c.expert_dim = hidden if hidden is not None else cfg.dim * 4 // 3
    return c


DENSE_ALIGN = 128


def dense_padded(weights: dict) -> tuple:
    """A prelude/coda block's dense FFN with its hidden width F rounded up to a multiple of
    128: zero rows appended to the gate and the up half of w13 [1, 2F, D] and zero columns
    to w2 [1, D, F].  A zero gate and up row gives silu(0) * 0 = 0 and a zero column of w2
    adds nothing, so the block computes the same function; the padded width fits the
    tensor-core GEMM's SwiGLU tile (128 gate + 128 up columns) and its rows are 16-byte
    aligned for the TMA maps (4 dim / 3 seldom is either).  Done once
    when a block is bound.  Returns (weights, padded width)."""
    w13, w2 = weights["w13"], weights["w2"]
    F = w2.shape[-1]
    Fp = -(-F // DENSE_ALIGN) * DENSE_ALIGN
    if Fp == F:
        return weights, F
    n13 = torch.zeros(w13.shape[0], 2 * Fp, w13.shape[2], dtype=w13.dtype, device=w13.device)
    n13[:, :F] = w13[:, :F]
    n13[:, Fp:Fp + F] = w13[:, F:]
    n2 = torch.zeros(w2.shape[0], w2.shape[1], Fp, dtype=w2.dtype, device=w2.device)
    n2[..., :F] = w2
    return {**weights, "w13": n13, "w2": n2}, Fp


class Weights:
    """Holds the tensors (keeps them alive) and the rdt_weights struct of their pointers."""

    def __init__(self, w: dict, model_dtype: torch.dtype):
        self.tensors = {}
        self.struct = N.rdt_weights()
        for name in N.WEIGHT_FIELDS:
            t = w.get(name)
            if t is None:
                continue
            if not t.is_cuda:
                raise ValueError(f"weight {name} must be a CUDA tensor")
            if not t.is_contiguous():
                raise ValueError(f"weight {name} must be contiguous")
            want = torch.float32 if name in _F32_FIELDS else model_dtype
            if t.dtype != want:
                raise ValueError(f"weight {name} must be {want}, got {t.dtype}")
            self.tensors[name] = t
            setattr(self.struct, name, t.data_ptr())


_F32_FIELDS = {"rec_norm_w", "attn_norm_w", "ffn_norm_w", "q_norm_w", "kv_norm_w", "router_bias", "lora_scale",
               "log_A", "log_dt", "inj_B", "halt_w", "halt_b"}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _check_act(t: torch.Tensor, name: str, dtype, shape):
    if not t.is_cuda or not t.is_contiguous() or t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                         f"{t.device} {t.dtype} {tuple(t.shape)} contiguous={t.is_contiguous()}")


def workspace_size(cfg_struct: N.rdt_config, batch: int, seq: int, max_keys: int) -> int:
    lib = N.load()
    return int(lib.rdt_workspace_size(ctypes.byref(cfg_struct), batch, seq, max_keys))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """Workspace as a torch uint8 buffer (torch's allocator returns >= 512-byte aligned blocks)."""
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device or "cuda")
    assert ws.data_ptr() % 256 == 0
    return ws


@dataclass
class KVCache:
    """One attention cache per recurrent loop.
    GQA: k, v [n_loops, batch, Hkv, t_max, hd] (post-RoPE keys, values).
    MLA: k = c_kv [n_loops, batch, t_max, kv_lora_rank] (before its RMSNorm),
         v = k_rope [n_loops, batch, t_max, qk_rope_head_dim] (rotated, shared by all heads)."""
    k: torch.Tensor
    v: torch.Tensor

    @property
    def t_max(self) -> int:
        return self.k.shape[3] if self.k.dim() == 5 else self.k.shape[2]

    def struct(self) -> N.rdt_kv_cache:
        if self.k.dim() not in (4, 5) or self.k.shape[:2] != self.v.shape[:2]:
            raise ValueError("cache tensors must be [n_loops, batch, ...] with matching leading dims")
        if not (self.k.is_contiguous() and self.v.is_contiguous()):
            raise ValueError("cache tensors must be contiguous")
        s = N.rdt_kv_cache()
        s.k, s.v = self.k.data_ptr(), self.v.data_ptr()
        s.n_loops, s.batch, s.t_max = self.k.shape[0], self.k.shape[1], self.t_max
        return s


@dataclass
class Trace:
    row0: int
    n_rows: int
    h_in: Optional[torch.Tensor] = None
    f: Optional[torch.Tensor] = None
    biased_logits: Optional[torch.Tensor] = None
    p: Optional[torch.Tensor] = None

    @staticmethod
    def alloc(cfg, n_loops: int, row0: int, n_rows: int) -> "Trace":
        z = lambda *s: torch.zeros(*s, dtype=torch.float32, device="cuda")
        return Trace(row0, n_rows, z(n_loops, n_rows, cfg.dim), z(n_loops, n_rows, cfg.dim),
                     z(n_loops, n_rows, cfg.n_experts), z(n_loops, n_rows))

    def struct(self) -> N.rdt_trace:
        s = N.rdt_trace()
        s.row0, s.n_rows = self.row0, self.n_rows
        s.h_in, s.f, s.biased_logits, s.p = _ptr(self.h_in), _ptr(self.f), _ptr(self.biased_logits), _ptr(self.p)
        return s


class RecurrentBlock:
    """The looped Recurrent Block bound to one set of device weights."""

    def __init__(self, cfg, weights: dict):
        _require_cuda()
        self.cfg = cfg
        self.cs = config_struct(cfg)
        self.dtype = _DT[cfg.dtype][1]
        self.w = Weights(weights, self.dtype)
        self._ws = None

    def workspace(self, batch: int, seq: int, max_keys: int) -> torch.Tensor:
        need = workspace_size(self.cs, batch, seq, max_keys)
        if need == 0:
            raise N.RdtError("rdt_workspace_size", N.RDT_ERR_INVALID_ARG)
        if self._ws is None or self._ws.numel() < need:
            self._ws = alloc_workspace(need)
        return self._ws

    def forward(self, h0: torch.Tensor, e: torch.Tensor, batch: int, seq: int, n_loops: int,
                act_threshold: float = 0.0, start_pos: int = 0, halt_logit_offset: Optional[torch.Tensor] = None,
                cache: Optional[KVCache] = None, trace: Optional[Trace] = None, flags: int = 0,
                out: Optional[tuple] = None, workspace: Optional[torch.Tensor] = None):
        """rdt_recurrent_forward.  Returns (h_out [N, D] fp32, halt_weights [L, N] fp32,
        expert_ids [L, N, k] int32)."""
        lib = N.load()
        cfg = self.cfg
        Nr = batch * seq
        _check_act(h0, "h0", torch.float32, (Nr, cfg.dim))
        _check_act(e, "e", self.dtype, (Nr, cfg.dim))
        if halt_logit_offset is not None:
            _check_act(halt_logit_offset, "halt_logit_offset", torch.float32, (Nr,))
        if out is None:
            out = (torch.empty(Nr, cfg.dim, dtype=torch.float32, device=h0.device),
                   torch.empty(n_loops, Nr, dtype=torch.float32, device=h0.device),
                   torch.empty(n_loops, Nr, cfg.n_experts_per_tok, dtype=torch.int32, device=h0.device))
        max_keys = start_pos + seq if cache is None else max(start_pos + seq, cache.t_max)
        ws = workspace if workspace is not None else self.workspace(batch, seq, max_keys)
        cs = cache.struct() if cache is not None else None
        ts = trace.struct() if trace is not None else None
        rc = lib.rdt_recurrent_forward(ctypes.byref(self.cs), ctypes.byref(self.w.struct), h0.data_ptr(),
                                       e.data_ptr(), batch, seq, start_pos, n_loops, float(act_threshold),
                                       _ptr(halt_logit_offset), out[0].data_ptr(), out[1].data_ptr(),
                                       out[2].data_ptr(), ctypes.byref(cs) if cs is not None else None,
                                       ctypes.byref(ts) if ts is not None else None, flags, ws.data_ptr(),
                                       ws.numel(), _stream())
        N.check("rdt_recurrent_forward", rc)
        return out

    def decode_step(self, h0: torch.Tensor, e: torch.Tensor, cache_len: torch.Tensor, cache: KVCache,
                    n_loops: int, act_threshold: float = 0.0, out: Optional[tuple] = None,
                    workspace: Optional[torch.Tensor] = None, trace: Optional[Trace] = None,
                    halt_logit_offset: Optional[torch.Tensor] = None):
        """rdt_recurrent_decode_step: one new token per sequence at position cache_len[b]
        (rdt_recurrent_decode_step_ex when a trace or halting-logit offsets are given)."""
        lib = N.load()
        cfg = self.cfg
        B = h0.shape[0]
        _check_act(h0, "h0", torch.float32, (B, cfg.dim))
        _check_act(e, "e", self.dtype, (B, cfg.dim))
        _check_act(cache_len, "cache_len", torch.int32, (B,))
        if out is None:
            out = (torch.empty(B, cfg.dim, dtype=torch.float32, device=h0.device),
                   torch.empty(n_loops, B, dtype=torch.float32, device=h0.device),
                   torch.empty(n_loops, B, cfg.n_experts_per_tok, dtype=torch.int32, device=h0.device))
        ws = workspace if workspace is not None else self.workspace(B, 1, cache.t_max)
        cs = cache.struct()
        if trace is not None or halt_logit_offset is not None:
            if halt_logit_offset is not None:
                _check_act(halt_logit_offset, "halt_logit_offset", torch.float32, (B,))
            ts = trace.struct() if trace is not None else None
            rc = lib.rdt_recurrent_decode_step_ex(ctypes.byref(self.cs), ctypes.byref(self.w.struct),
                                                  h0.data_ptr(), e.data_ptr(), B, cache_len.data_ptr(), n_loops,
                                                  float(act_threshold), _ptr(halt_logit_offset), out[0].data_ptr(),
                                                  out[1].data_ptr(), out[2].data_ptr(), ctypes.byref(cs),
                                                  ctypes.byref(ts) if ts is not None else None,
                                                  ws.data_ptr(), ws.numel(), _stream())
            N.check("rdt_recurrent_decode_step_ex", rc)
            return out
        rc = lib.rdt_recurrent_decode_step(ctypes.byref(self.cs), ctypes.byref(self.w.struct), h0.data_ptr(),
                                           e.data_ptr(), B, cache_len.data_ptr(), n_loops, float(act_threshold),
                                           out[0].data_ptr(), out[1].data_ptr(), out[2].data_ptr(),
                                           ctypes.byref(cs), ws.data_ptr(), ws.numel(), _stream())
        N.check("rdt_recurrent_decode_step", rc)
        return out

    def read_status(self):
        lib = N.load()
        return lib.rdt_read_device_status(self._ws.data_ptr(), _stream()) if self._ws is not None else N.RDT_OK


class DecodeGraph:
    """RecurrentBlock.decode_step replayed from a CUDA graph, for a serving loop that steps
    the same sequences against the same caches.  Every address the captured launches use
    is fixed: the step's h0 / e are copied into `h_in` / `e_in` before each replay, the
    outputs land in `out`, and the cache length advances inside the graph (cache_len += 1
    after the step, as an eager loop would do).  The first call runs eagerly (it also
    performs the kernels' one-time attribute setup), the second captures the step once and
    replays it, every later call replays.  Calls made while the library's profiler records
    run eagerly, since its CUDA events are recorded at launch time."""

    def __init__(self, blk: "RecurrentBlock", batch: int, cache: KVCache, cache_len: torch.Tensor, n_loops: int,
                 act_threshold: float = 0.0, workspace: Optional[torch.Tensor] = None, out: Optional[tuple] = None,
                 halt_logit_offset: bool = False):
        cfg = blk.cfg
        self.blk, self.B, self.cache, self.cache_len = blk, batch, cache, cache_len
        self.L, self.thr = n_loops, act_threshold
        self.ws = workspace if workspace is not None else blk.workspace(batch, 1, cache.t_max)
        self.out = out if out is not None else (
            torch.empty(batch, cfg.dim, dtype=torch.float32, device="cuda"),
            torch.empty(n_loops, batch, dtype=torch.float32, device="cuda"),
            torch.empty(n_loops, batch, cfg.n_experts_per_tok, dtype=torch.int32, device="cuda"))
        self.h_in = torch.empty(batch, cfg.dim, dtype=torch.float32, device="cuda")
        self.e_in = torch.empty(batch, cfg.dim, dtype=blk.dtype, device="cuda")
        # per-step halting-logit offsets (copied in before each replay), when the step takes them
        self.off_in = torch.zeros(batch, dtype=torch.float32, device="cuda") if halt_logit_offset else None
        self._graph = None
        self._eager = 0
        self.graph_launches = 0      # library kernels in one replay

    def _body(self, h0, e, off=None):
        self.blk.decode_step(h0, e, self.cache_len, self.cache, self.L, self.thr, out=self.out, workspace=self.ws,
                             halt_logit_offset=off)
        self.cache_len.add_(1)

    def step(self, h0: torch.Tensor, e: torch.Tensor, halt_logit_offset: Optional[torch.Tensor] = None) -> tuple:
        """One decode step of every sequence; returns (h_out, halt weights, expert ids)."""
        if (halt_logit_offset is None) != (self.off_in is None):
            raise ValueError("halt_logit_offset must be given exactly when the graph was built for it")
        if N.profiling() or self._eager == 0:
            self._body(h0, e, halt_logit_offset)
            self._eager += 1
            return self.out
        self.h_in.copy_(h0)
        self.e_in.copy_(e)
        if self.off_in is not None:
            self.off_in.copy_(halt_logit_offset)
        if self._graph is None:
            g = torch.cuda.CUDAGraph()
            n0 = N.launch_count()
            # thread-local capture: other threads of the process (a collective library's
            # watchdog, for one) keep calling CUDA while this thread captures
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                self._body(self.h_in, self.e_in, self.off_in)
            self.graph_launches = N.launch_count() - n0
            self._graph = g
        self._graph.replay()
        return self.out


class DepthBatch:
    """Continuous depth-wise batching of decode steps (rdt_depth_batch_*): `batch` sequences
    each decode n_tokens tokens in order, one slot per sequence; every tick runs the shared
    block once over all slots, each slot's token at its own loop, and a token that halts
    leaves its slot to the sequence's next token (after its remaining loops' keys / values
    are written from its frozen state).  Results equal n_tokens successive decode_step calls
    per sequence.  h0 [B, S, D] fp32, e [B, S, D] model dtype, cache_len [B] int32 (position
    of token 0), halt_logit_offset [B, S] fp32 or None.  Outputs: h_out [B, S, D],
    halt_weights [B, S, L], expert_ids [B, S, L, k]."""

    def __init__(self, blk: "RecurrentBlock", h0: torch.Tensor, e: torch.Tensor, cache_len: torch.Tensor,
                 cache: KVCache, n_loops: int, act_threshold: float = 0.0,
                 halt_logit_offset: Optional[torch.Tensor] = None, out: Optional[tuple] = None,
                 workspace: Optional[torch.Tensor] = None):
        lib = N.load()
        cfg = blk.cfg
        B, S = h0.shape[0], h0.shape[1]
        _check_act(h0, "h0", torch.float32, (B, S, cfg.dim))
        _check_act(e, "e", blk.dtype, (B, S, cfg.dim))
        _check_act(cache_len, "cache_len", torch.int32, (B,))
        if halt_logit_offset is not None:
            _check_act(halt_logit_offset, "halt_logit_offset", torch.float32, (B, S))
        self.blk, self.B, self.S, self.L = blk, B, S, n_loops
        self.inputs = (h0, e, cache_len, halt_logit_offset)     # kept alive: the struct holds their addresses
        self.out = out if out is not None else (
            torch.empty(B, S, cfg.dim, dtype=torch.float32, device=h0.device),
            torch.empty(B, S, n_loops, dtype=torch.float32, device=h0.device),
            torch.empty(B, S, n_loops, cfg.n_experts_per_tok, dtype=torch.int32, device=h0.device))
        need = int(lib.rdt_depth_batch_workspace_size(ctypes.byref(blk.cs), B, n_loops, cache.t_max))
        if need == 0:
            raise N.RdtError("rdt_depth_batch_workspace_size", N.RDT_ERR_INVALID_ARG)
        self.ws = workspace if workspace is not None and workspace.numel() >= need else alloc_workspace(need)
        self.cache, self._cs = cache, cache.struct()
        db = N.rdt_depth_batch()
        db.cfg, db.w = ctypes.pointer(blk.cs), ctypes.pointer(blk.w.struct)
        db.h0, db.e, db.halt_logit_offset, db.cache_len = (h0.data_ptr(), e.data_ptr(), _ptr(halt_logit_offset),
                                                           cache_len.data_ptr())
        db.batch, db.n_tokens, db.n_loops, db.act_threshold = B, S, n_loops, float(act_threshold)
        db.h_out, db.halt_weights, db.expert_ids = (o.data_ptr() for o in self.out)
        db.cache = ctypes.pointer(self._cs)
        db.ws, db.ws_bytes = self.ws.data_ptr(), self.ws.numel()
        self.db = db
        self._graph = None
        self._graph_ticks = 0
        self.graph_launches = 0
        self.ticks = 0

    def begin(self):
        N.check("rdt_depth_batch_begin", N.load().rdt_depth_batch_begin(ctypes.byref(self.db), _stream()))
        self.ticks = 0

    def tick(self, n: int = 1):
        N.check("rdt_depth_batch_tick", N.load().rdt_depth_batch_tick(ctypes.byref(self.db), n, _stream()))
        self.ticks += n

    def pending(self) -> int:
        v = int(N.load().rdt_depth_batch_pending(ctypes.byref(self.db), _stream()))
        if v < 0:
            raise N.RdtError("rdt_depth_batch_pending", N.RDT_ERR_CUDA)
        return v

    def run(self, check_every: int = 8, cuda_graph: bool = False) -> tuple:
        """All tokens: begin, then ticks in chunks of check_every until none is pending.
        With cuda_graph the first chunk runs eagerly (kernel set-up) and later chunks replay a
        CUDA graph of check_every ticks captured once."""
        if not cuda_graph or N.profiling():
            N.check("rdt_depth_batch_run", N.load().rdt_depth_batch_run(ctypes.byref(self.db), check_every,
                                                                         _stream()))
            return self.out
        self.begin()
        max_ticks = self.S * self.L
        self.tick(min(check_every, max_ticks))
        while self.ticks < max_ticks and self.pending() > 0:
            if self._graph is None or self._graph_ticks != check_every:
                g = torch.cuda.CUDAGraph()
                n0 = N.launch_count()
                with torch.cuda.graph(g, capture_error_mode="thread_local"):
                    N.check("rdt_depth_batch_tick", N.load().rdt_depth_batch_tick(ctypes.byref(self.db),
                                                                                   check_every, _stream()))
                self.graph_launches = N.launch_count() - n0
                self._graph, self._graph_ticks = g, check_every
            self._graph.replay()
            self.ticks += check_every
        return self.out

    def read_status(self) -> int:
        return N.load().rdt_read_device_status(self.ws.data_ptr(), _stream())


class Block:
    """One pre-norm prelude/coda block (dense SwiGLU FFN) or MoE block bound to its weights."""

    def __init__(self, cfg, weights: dict, dense: bool = True):
        _require_cuda()
        self.cfg = cfg
        if dense:
            weights, hidden = dense_padded(weights)
            self.cs = dense_config_struct(cfg, hidden)
        else:
            self.cs = config_struct(cfg)
        self.w = Weights(weights, _DT[cfg.dtype][1])

    def workspace(self, batch: int, seq: int, max_keys: int) -> torch.Tensor:
        return alloc_workspace(workspace_size(self.cs, batch, seq, max_keys))

    def forward(self, x: torch.Tensor, batch: int, seq: int, start_pos: int = 0, cache: Optional[KVCache] = None,
                cache_len: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
        """rdt_block_forward_cached: prefill at start_pos (cache_len None) or one decode
        step at positions cache_len[b] (seq 1); cache None = no cache."""
        lib = N.load()
        _check_act(x, "x", torch.float32, (batch * seq, self.cfg.dim))
        if cache_len is not None:
            _check_act(cache_len, "cache_len", torch.int32, (batch,))
        out = torch.empty_like(x) if out is None else out
        max_keys = start_pos + seq if cache is None else max(start_pos + seq, cache.t_max)
        ws = workspace if workspace is not None else self.workspace(batch, seq, max_keys)
        cs = cache.struct() if cache is not None else None
        rc = lib.rdt_block_forward_cached(ctypes.byref(self.cs), ctypes.byref(self.w.struct), x.data_ptr(),
                                          out.data_ptr(), batch, seq, start_pos,
                                          None if cache_len is None else cache_len.data_ptr(),
                                          None if cs is None else ctypes.byref(cs), ws.data_ptr(), ws.numel(),
                                          _stream())
        N.check("rdt_block_forward_cached", rc)
        return out


def block_forward(cfg, weights: dict, x: torch.Tensor, batch: int, seq: int, start_pos: int = 0,
                  dense: bool = True) -> torch.Tensor:
    """rdt_block_forward: one pre-norm prelude/coda block (dense SwiGLU FFN) or a MoE block."""
    lib = _require_cuda()
    if dense:
        weights, hidden = dense_padded(weights)
        cs = dense_config_struct(cfg, hidden)
    else:
        cs = config_struct(cfg)
    w = Weights(weights, _DT[cfg.dtype][1])
    _check_act(x, "x", torch.float32, (batch * seq, cfg.dim))
    out = torch.empty_like(x)
    ws = alloc_workspace(workspace_size(cs, batch, seq, start_pos + seq))
    rc = lib.rdt_block_forward(ctypes.byref(cs), ctypes.byref(w.struct), x.data_ptr(), out.data_ptr(), batch, seq,
                               start_pos, ws.data_ptr(), ws.numel(), _stream())
    N.check("rdt_block_forward", rc)
    return out


def to_model_dtype(cfg, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """rdt_to_model_dtype: the prelude output as the recurrent block's injected input e."""
    lib = _require_cuda()
    if not x.is_cuda or not x.is_contiguous() or x.dtype != torch.float32:
        raise ValueError("x: expected a contiguous CUDA float32 tensor")
    out = torch.empty(x.shape, dtype=_DT[cfg.dtype][1], device=x.device) if out is None else out
    rc = lib.rdt_to_model_dtype(ctypes.byref(config_struct(cfg)), x.data_ptr(), out.data_ptr(), x.numel(), _stream())
    N.check("rdt_to_model_dtype", rc)
    return out


def greedy_tokens(logits: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """rdt_greedy_tokens: argmax per row of fp32 logits [n, V], ties to the lowest index."""
    lib = _require_cuda()
    _check_act(logits, "logits", torch.float32, tuple(logits.shape))
    n, V = logits.shape
    out = torch.empty(n, dtype=torch.int32, device=logits.device) if out is None else out
    rc = lib.rdt_greedy_tokens(logits.data_ptr(), n, V, out.data_ptr(), 1, _stream())
    N.check("rdt_greedy_tokens", rc)
    return out


def embed(cfg, table: torch.Tensor, ids: torch.Tensor) -> torch.Tensor:
    lib = _require_cuda()
    cs = config_struct(cfg)
    ids32 = ids.reshape(-1).to(device="cuda", dtype=torch.int32).contiguous()
    out = torch.empty(ids32.numel(), cfg.dim, dtype=torch.float32, device="cuda")
    rc = lib.rdt_embed(ctypes.byref(cs), table.data_ptr(), table.shape[0], ids32.data_ptr(), ids32.numel(),
                       out.data_ptr(), _stream())
    N.check("rdt_embed", rc)
    return out


def head(cfg, x: torch.Tensor, norm_w: torch.Tensor, head_w: torch.Tensor, last_of: int = 0,
         out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """rdt_head / rdt_head_rows: logits of every row of x [n, D], or with last_of = T of
    the last row of each T-row sequence (x [B * T, D] -> logits [B, V])."""
    lib = _require_cuda()
    cs = config_struct(cfg)
    if not x.is_cuda or not x.is_contiguous() or x.dtype != torch.float32 or x.shape[-1] != cfg.dim:
        raise ValueError("x: expected a contiguous CUDA float32 [n, dim] tensor")
    n = x.shape[0] // last_of if last_of else x.shape[0]
    V = head_w.shape[0]
    out = torch.empty(n, V, dtype=torch.float32, device="cuda") if out is None else out
    ws = workspace if workspace is not None else alloc_workspace(workspace_size(cs, 1, n, n))
    if last_of:
        ptr = x.data_ptr() + (last_of - 1) * cfg.dim * 4
        rc = lib.rdt_head_rows(ctypes.byref(cs), ptr, last_of * cfg.dim, n, norm_w.data_ptr(), head_w.data_ptr(), V,
                               out.data_ptr(), ws.data_ptr(), ws.numel(), _stream())
    else:
        rc = lib.rdt_head(ctypes.byref(cs), x.data_ptr(), n, norm_w.data_ptr(), head_w.data_ptr(), V,
                          out.data_ptr(), ws.data_ptr(), ws.numel(), _stream())
    N.check("rdt_head", rc)
    return out


def model_forward(cfg, MW: dict, ids: torch.Tensor, n_loops: int, act_threshold: float):
    """OpenMythos.forward composed from the library's entry points (embedding, prelude
    blocks, the recurrent block, coda blocks, head).  Returns (logits [B, T, V],
    (h_out, halt_weights, expert_ids))."""
    B, T = ids.shape
    x = embed(cfg, MW["embed"], ids)
    for W in MW["prelude"]:
        x = block_forward(cfg, W, x, B, T)
    e = to_model_dtype(cfg, x)
    rb = RecurrentBlock(cfg, MW["recurrent"])
    rec = rb.forward(x, e, B, T, n_loops, act_threshold)
    x = rec[0]
    for W in MW["coda"]:
        x = block_forward(cfg, W, x, B, T)
    logits = head(cfg, x, MW["norm_w"], MW["head"])
    return logits.reshape(B, T, -1), rec


def _layer_cache(cfg, n_loops: int, batch: int, t_max: int) -> KVCache:
    """Zeroed per-loop (or, with n_loops 1, per-layer) cache in the layout of rdt_kv_cache."""
    dt = _DT[cfg.dtype][1]
    if cfg.attn_type == "gqa":
        z = torch.zeros(n_loops, batch, cfg.n_kv_heads, t_max, cfg.head_dim, dtype=dt, device="cuda")
        return KVCache(z, torch.zeros_like(z))
    return KVCache(torch.zeros(n_loops, batch, t_max, cfg.kv_lora_rank, dtype=dt, device="cuda"),
                   torch.zeros(n_loops, batch, t_max, cfg.qk_rope_head_dim, dtype=dt, device="cuda"))


class Generator:
    """OpenMythos.generate on the library's entry points ("OpenMythos 분석", RoPE &
    generation cache): step 0 runs the whole prompt at start_pos 0 and fills one cache per
    prelude / coda layer and per recurrent loop; every later step runs the last token
    alone at position prompt_len + step - 1 against those caches.  The next token is the
    greedy choice (rdt_greedy_tokens).  All buffers are allocated once per generator, so
    the decode steps allocate nothing.

    With cuda_graph (the default) the decode step's launches (about 20 per loop plus the
    prelude, coda, head and greedy choice) are captured once into a CUDA graph on the
    second decode call and replayed from then on.  Everything a step reads is at a fixed
    address: the previous token is copied into `cur_tok` and the cache length set before
    the replay, and the new token copied out of `cur_tok` after it.  The first decode call
    runs eagerly (it also performs the kernels' one-time attribute setup), and so does every
    call made while the library's profiler is recording."""

    def __init__(self, cfg, MW: dict, batch: int, prompt_len: int, max_new_tokens: int, n_loops: int,
                 act_threshold: float = 0.0, cuda_graph: bool = True, trace: bool = False):
        _require_cuda()
        self.cfg, self.MW = cfg, MW
        self.B, self.T0, self.new, self.L, self.thr = batch, prompt_len, max_new_tokens, n_loops, act_threshold
        self.t_max = prompt_len + max_new_tokens
        B, D, T0 = batch, cfg.dim, prompt_len
        self.pre = [Block(cfg, W) for W in MW["prelude"]]
        self.coda = [Block(cfg, W) for W in MW["coda"]]
        self.rb = RecurrentBlock(cfg, MW["recurrent"])
        self.pre_cache = [_layer_cache(cfg, 1, B, self.t_max) for _ in self.pre]
        self.coda_cache = [_layer_cache(cfg, 1, B, self.t_max) for _ in self.coda]
        self.rec_cache = _layer_cache(cfg, n_loops, B, self.t_max)
        sizes = [workspace_size(b.cs, B, s, self.t_max) for b in self.pre + self.coda for s in (T0, 1)]
        self.ws_block = alloc_workspace(max(sizes + [256]))
        self.ws_rec_prefill = self.rb.workspace(B, T0, self.t_max)
        self.ws_rec_decode = self.rb.workspace(B, 1, self.t_max)
        cs = config_struct(cfg)
        self.ws_head = alloc_workspace(workspace_size(cs, 1, B, B))
        V = MW["head"].shape[0]
        dt = _DT[cfg.dtype][1]
        self.xa = torch.empty(B * T0, D, dtype=torch.float32, device="cuda")
        self.xb = torch.empty_like(self.xa)
        self.e = torch.empty(B * T0, D, dtype=dt, device="cuda")
        self.rec_out = (torch.empty(B * T0, D, dtype=torch.float32, device="cuda"),
                        torch.empty(n_loops, B * T0, dtype=torch.float32, device="cuda"),
                        torch.empty(n_loops, B * T0, cfg.n_experts_per_tok, dtype=torch.int32, device="cuda"))
        self.logits = torch.empty(B, V, dtype=torch.float32, device="cuda")
        self.tokens = torch.empty(max_new_tokens, B, dtype=torch.int32, device="cuda")
        self.dec_out = (torch.empty(B, D, dtype=torch.float32, device="cuda"),
                        torch.empty(n_loops, B, dtype=torch.float32, device="cuda"),
                        torch.empty(n_loops, B, cfg.n_experts_per_tok, dtype=torch.int32, device="cuda"))
        self.cache_len = torch.empty(B, dtype=torch.int32, device="cuda")
        self.cur_tok = torch.empty(B, dtype=torch.int32, device="cuda")
        self.cuda_graph = cuda_graph
        # optional per-loop trace of the recurrent block (tests): every prompt row of the
        # prefill, every sequence's row of the latest decode step
        self.trace_prefill = Trace.alloc(cfg, n_loops, 0, B * T0) if trace else None
        self.trace_decode = Trace.alloc(cfg, n_loops, 0, B) if trace else None
        self._graph = None
        self._eager_decodes = 0
        self.graph_launches = 0      # library kernels in one replay of the captured step

    def _run_blocks(self, blocks, caches, x, y, seq, start_pos, cache_len):
        for blk, c in zip(blocks, caches):
            blk.forward(x, self.B, seq, start_pos, cache=c, cache_len=cache_len, out=y, workspace=self.ws_block)
            x, y = y, x
        return x, y

    def prefill(self, prompt_ids: torch.Tensor) -> torch.Tensor:
        """Step 0: the prompt [B, T0] (int32, CUDA); returns the first new token [B]."""
        B, T0, D = self.B, self.T0, self.cfg.dim
        lib = N.load()
        ids = prompt_ids.reshape(-1)
        if not ids.is_cuda or ids.dtype != torch.int32 or ids.numel() != B * T0 or not ids.is_contiguous():
            raise ValueError("prompt_ids: expected a contiguous CUDA int32 [batch, prompt_len] tensor")
        x, y = self.xa, self.xb
        rc = lib.rdt_embed(ctypes.byref(config_struct(self.cfg)), self.MW["embed"].data_ptr(),
                           self.MW["embed"].shape[0], ids.data_ptr(), B * T0, x.data_ptr(), _stream())
        N.check("rdt_embed", rc)
        x, y = self._run_blocks(self.pre, self.pre_cache, x, y, T0, 0, None)
        to_model_dtype(self.cfg, x, out=self.e)
        self.rb.forward(x, self.e, B, T0, self.L, self.thr, start_pos=0, cache=self.rec_cache, out=self.rec_out,
                        workspace=self.ws_rec_prefill, trace=self.trace_prefill)
        x, y = self._run_blocks(self.coda, self.coda_cache, self.rec_out[0], y, T0, 0, None)
        head(self.cfg, x, self.MW["norm_w"], self.MW["head"], last_of=T0, out=self.logits, workspace=self.ws_head)
        greedy_tokens(self.logits, out=self.tokens[0])
        return self.tokens[0]

    def _decode_body(self, tok_in: torch.Tensor, tok_out: torch.Tensor):
        """One decode step from the tokens in tok_in [B] to the greedy tokens in tok_out [B],
        with the cache length already in self.cache_len."""
        B = self.B
        lib = N.load()
        x, y = self.xa[:B], self.xb[:B]
        rc = lib.rdt_embed(ctypes.byref(config_struct(self.cfg)), self.MW["embed"].data_ptr(),
                           self.MW["embed"].shape[0], tok_in.data_ptr(), B, x.data_ptr(), _stream())
        N.check("rdt_embed", rc)
        x, y = self._run_blocks(self.pre, self.pre_cache, x, y, 1, 0, self.cache_len)
        e = self.e[:B]
        to_model_dtype(self.cfg, x, out=e)
        out = self.dec_out
        self.rb.decode_step(x, e, self.cache_len, self.rec_cache, self.L, self.thr, out=out,
                            workspace=self.ws_rec_decode, trace=self.trace_decode)
        x, y = self._run_blocks(self.coda, self.coda_cache, out[0], y, 1, 0, self.cache_len)
        head(self.cfg, x, self.MW["norm_w"], self.MW["head"], out=self.logits, workspace=self.ws_head)
        greedy_tokens(self.logits, out=tok_out)

    def decode(self, step: int) -> torch.Tensor:
        """Step `step` >= 1: the token of step - 1 at position prompt_len + step - 1."""
        self.cache_len.fill_(self.T0 + step - 1)
        if not self.cuda_graph or N.profiling() or self._eager_decodes == 0:
            self._decode_body(self.tokens[step - 1], self.tokens[step])
            self._eager_decodes += 1
            return self.tokens[step]
        self.cur_tok.copy_(self.tokens[step - 1])
        if self._graph is None:
            g = torch.cuda.CUDAGraph()
            n0 = N.launch_count()
            # thread-local capture: other threads of the process (a collective library's
            # watchdog, for one) keep calling CUDA while this thread captures
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                self._decode_body(self.cur_tok, self.cur_tok)
            self.graph_launches = N.launch_count() - n0
            self._graph = g
        self._graph.replay()
        self.tokens[step].copy_(self.cur_tok)
        return self.tokens[step]

    def run(self, prompt_ids: torch.Tensor) -> torch.Tensor:
        """Prompt [B, T0] -> the generated tokens [B, max_new_tokens] (int32, CUDA)."""
        self.prefill(prompt_ids)
        for step in range(1, self.new):
            self.decode(step)
        return self.tokens.t()


def generate(cfg, MW: dict, prompt_ids: torch.Tensor, max_new_tokens: int, n_loops: int,
             act_threshold: float = 0.0) -> torch.Tensor:
    """Greedy generation: returns [B, T0 + max_new_tokens] token ids (int32, CUDA)."""
    B, T0 = prompt_ids.shape
    ids = prompt_ids.to(device="cuda", dtype=torch.int32).contiguous()
    gen = Generator(cfg, MW, B, T0, max_new_tokens, n_loops, act_threshold)
    new = gen.run(ids)
    return torch.cat([ids, new], dim=1)
