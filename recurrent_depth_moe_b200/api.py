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


def dense_config_struct(cfg) -> N.rdt_config:
    """Config of a prelude/coda block: no routed experts, one dense SwiGLU of width 4*dim/3."""
    c = config_struct(cfg)
    c.n_experts, c.top_k, c.n_shared_experts, c.expert_dim = 0, 0, 1, cfg.dim * 4 // 3
    return c


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
                    workspace: Optional[torch.Tensor] = None):
        """rdt_recurrent_decode_step: one new token per sequence at position cache_len[b]."""
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
        rc = lib.rdt_recurrent_decode_step(ctypes.byref(self.cs), ctypes.byref(self.w.struct), h0.data_ptr(),
                                           e.data_ptr(), B, cache_len.data_ptr(), n_loops, float(act_threshold),
                                           out[0].data_ptr(), out[1].data_ptr(), out[2].data_ptr(),
                                           ctypes.byref(cs), ws.data_ptr(), ws.numel(), _stream())
        N.check("rdt_recurrent_decode_step", rc)
        return out

    def read_status(self):
        lib = N.load()
        return lib.rdt_read_device_status(self._ws.data_ptr(), _stream()) if self._ws is not None else N.RDT_OK


def block_forward(cfg, weights: dict, x: torch.Tensor, batch: int, seq: int, start_pos: int = 0,
                  dense: bool = True) -> torch.Tensor:
    """rdt_block_forward: one pre-norm prelude/coda block (dense SwiGLU FFN) or a MoE block."""
    lib = _require_cuda()
    cs = dense_config_struct(cfg) if dense else config_struct(cfg)
    w = Weights(weights, _DT[cfg.dtype][1])
    _check_act(x, "x", torch.float32, (batch * seq, cfg.dim))
    out = torch.empty_like(x)
    ws = alloc_workspace(workspace_size(cs, batch, seq, start_pos + seq))
    rc = lib.rdt_block_forward(ctypes.byref(cs), ctypes.byref(w.struct), x.data_ptr(), out.data_ptr(), batch, seq,
                               start_pos, ws.data_ptr(), ws.numel(), _stream())
    N.check("rdt_block_forward", rc)
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


def head(cfg, x: torch.Tensor, norm_w: torch.Tensor, head_w: torch.Tensor) -> torch.Tensor:
    lib = _require_cuda()
    cs = config_struct(cfg)
    n = x.shape[0]
    out = torch.empty(n, head_w.shape[0], dtype=torch.float32, device="cuda")
    ws = alloc_workspace(workspace_size(cs, 1, n, n))
    rc = lib.rdt_head(ctypes.byref(cs), x.data_ptr(), n, norm_w.data_ptr(), head_w.data_ptr(), head_w.shape[0],
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
    e = x.to(_DT[cfg.dtype][1]).contiguous()
    rb = RecurrentBlock(cfg, MW["recurrent"])
    rec = rb.forward(x.contiguous(), e, B, T, n_loops, act_threshold)
    x = rec[0]
    for W in MW["coda"]:
        x = block_forward(cfg, W, x, B, T)
    logits = head(cfg, x, MW["norm_w"], MW["head"])
    return logits.reshape(B, T, -1), rec
