"""ctypes binding of libdflash.so (see include/dflash.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity and passed as raw pointers; every step of the hot path runs in the
library's CUDA kernels.  PyTorch provides device memory and streams.  There
is no fallback: if the library is missing, importing the binding fails.
"""

from __future__ import annotations

import ctypes
import os
import re
from typing import Dict, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdflash.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "dflash.h")
HEADERS = [HEADER, os.path.join(os.path.dirname(_HERE), "include", "dflash_debug.h")]

OK, EINVAL, EUNSUPPORTED, ECUDA, ENOMEM, EWORKSPACE, ESCRATCH = 0, -1, -2, -3, -4, -5, -6
DEV_CTX_CAP, DEV_OUT_CAP, DEV_TOKEN_RANGE, DEV_TIMEOUT, DEV_ROWS, DEV_PAGE, DEV_RANGE = (
    1, 2, 4, 8, 16, 32, 64)
F32, BF16, F16 = 0, 1, 2
TIMING_CLASSES = ("gemm", "attention", "row", "verify", "lm_head")


class DFlashError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call} failed: {status} ({status_str(status)})")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "dtype", "H_t", "n_tap", "n_layers", "d", "n_q", "n_kv", "head_dim", "inter", "vocab",
        "mask_id", "max_pos")] + [("eps", ctypes.c_float), ("rope_base", ctypes.c_double)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("g_in", "Wq", "Wk", "Wv", "Wo", "g_post", "Wg", "Wu", "Wd")]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("emb", "W_fc", "g_ctx", "g_final", "W_lm")] + [
        ("layers", ctypes.POINTER(LayerWeights))]


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        # DFLASH_LIB names another build of the same library (e.g. one built out
        # of tree); there is no fallback when the file is missing
        path = os.environ.get("DFLASH_LIB") or LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with "
                "`python -m block_diffusion_speculative_gemm_b200.build`")
        L = ctypes.CDLL(path)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.dflash_model_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Weights),
                                          ctypes.POINTER(vp)]
        L.dflash_model_destroy.argtypes = [vp]
        L.dflash_workspace_size.argtypes = [vp, i32, i32, i32]
        L.dflash_workspace_size.restype = sz
        L.dflash_verify_workspace_size.argtypes = [i32, i32, i32]
        L.dflash_verify_workspace_size.restype = sz
        L.dflash_workspace_init.argtypes = [vp, sz, vp]
        L.dflash_inject_kv.argtypes = [vp, ctypes.POINTER(vp), vp, vp, i32, i32, vp, vp, i32, vp,
                                       sz, vp]
        L.dflash_draft_block.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp,
                                         sz, vp]
        L.dflash_model_create_shard.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Weights),
                                                i32, i32, ctypes.POINTER(vp)]
        L.dflash_draft_rows.argtypes = [i32, i32, i32, i32]
        L.dflash_draft_begin.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, sz, vp]
        L.dflash_draft_forward_shard.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp,
                                                 sz, vp]
        L.dflash_draft_commit_shards.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, sz, vp]
        L.dflash_draft_end.argtypes = [vp, i32, i32, i32, vp, vp, vp, sz, vp]
        L.dflash_verify_shard.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, sz, vp]
        L.dflash_verify_merge.argtypes = [vp, i32, vp, i32, i32, i32, vp, vp, i32, vp, vp, vp, vp,
                                          sz, vp]
        L.dflash_inject_kv_paged.argtypes = [vp, ctypes.POINTER(vp), vp, vp, i32, i32, vp, vp,
                                             i32, i32, vp, i32, vp, sz, vp]
        L.dflash_draft_block_paged.argtypes = [vp, vp, vp, vp, vp, i32, i32, vp, i32, i32, i32,
                                               i32, vp, vp, vp, vp, sz, vp]
        L.dflash_draft_block_sampled.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                                 ctypes.c_float, ctypes.c_uint64,
                                                 ctypes.c_uint64, vp, vp, vp, i32, vp, sz, vp]
        L.dflash_verify.argtypes = [vp, i32, vp, i32, i32, i32, vp, vp, i32, vp, vp, vp, vp, sz,
                                    vp]
        L.dflash_get_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int32)]
        L.dflash_verify_noalloc.argtypes = [vp, i32, vp, i32, i32, i32, vp, vp, i32, vp, vp, vp,
                                            vp, vp]
        u64 = ctypes.c_uint64
        L.dflash_verify_sampled_workspace_size.argtypes = [i32, i32, i32]
        L.dflash_verify_sampled_workspace_size.restype = sz
        L.dflash_verify_sampled.argtypes = [vp, vp, i32, vp, i32, i32, i32, ctypes.c_float, u64,
                                            u64, vp, vp, i32, vp, vp, vp, vp, sz, vp]
        L.dflash_status_str.argtypes = [i32]
        L.dflash_status_str.restype = ctypes.c_char_p
        L.dflash_timing_enable.argtypes = [i32]
        L.dflash_timing_read.argtypes = [ctypes.POINTER(ctypes.c_double),
                                         ctypes.POINTER(ctypes.c_int64), i32]
        L.dflash_debug_gemm.argtypes = [vp, i32, i32, vp, i32, i32, i32, vp,
                                        ctypes.POINTER(ctypes.c_int), vp, vp]
        L.dflash_debug_lmhead.argtypes = [vp, i32, i32, vp, i32, i32, vp, vp, vp, vp]
        L.dflash_debug_gemm_tiled.argtypes = [vp, i32, i32, vp, i32, i32, i32, vp,
                                              ctypes.POINTER(ctypes.c_int), vp, vp]
        L.dflash_debug_tiled_bytes.argtypes = [i32, i32]
        L.dflash_debug_tiled_bytes.restype = sz
        L.dflash_debug_tile_weights.argtypes = [vp, vp, i32, i32, vp]
        L.dflash_debug_lmhead_tiled.argtypes = [vp, i32, i32, vp, i32, i32, vp, vp, vp, vp]
        L.dflash_debug_gemm_mode.argtypes = [i32]
        L.dflash_debug_gemm_schedule.argtypes = [i32]
        L.dflash_debug_attn_schedule.argtypes = [i32]
        L.dflash_debug_gemm_streamk_ws_bytes.argtypes = [i32]
        L.dflash_debug_gemm_streamk_ws_bytes.restype = sz
        L.dflash_debug_gemm_streamk.argtypes = [vp, i32, i32, vp, i32, i32, vp, vp, sz, vp]
        L.dflash_debug_attn_chunk.argtypes = [i32]
        L.dflash_debug_attn_plan.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp,
                                             ctypes.c_longlong, vp]
        L.dflash_debug_attn_slots.argtypes = [i32, i32, i32]
        L.dflash_debug_pick_splits.argtypes = [i32, i32, i32]
        L.dflash_debug_wait_timeout.argtypes = [vp, vp]
        L.dflash_debug_split_weight.argtypes = [ctypes.c_float]
        L.dflash_debug_sample_math.argtypes = [vp, vp, i32, vp, vp, vp]
        _lib = L
    return _lib


def header_symbols() -> list:
    """Function names declared in the headers under include/."""
    txt = ""
    for h in HEADERS:
        with open(h) as f:
            txt += f.read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(dflash_\w+)\s*\(", txt,
                                 flags=re.M)))


def status_str(status: int) -> str:
    return lib().dflash_status_str(int(status)).decode()


def _check(call: str, st: int):
    if st != OK:
        raise DFlashError(call, st)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(stream.cuda_stream))


def _need(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


_TORCH_DT = {F32: torch.float32, BF16: torch.bfloat16}


class Model:
    """A draft model prepacked on the current CUDA device.

    ``shape`` is any object with attributes dtype ("f32"/"bf16"), H_t, n_tap,
    L, d, nq, nkv, hd, I, V, mask_id, eps, rope_base.  ``weights`` is a dict
    of CUDA tensors laid out as in include/dflash.h (keys emb, W_fc, g_ctx,
    g_final, W_lm, layers[l] with g_in, Wq, Wk, Wv, Wo, g_post, Wg, Wu, Wd).
    """

    def __init__(self, shape, weights: Dict, max_pos: int, vocab_range=None):
        self.shape = shape
        self.dtype = BF16 if shape.dtype == "bf16" else F32
        self.tdtype = _TORCH_DT[self.dtype]
        # K/V cache element type: fp16 for bf16 models (see include/dflash.h), fp32 for fp32
        self.cache_dtype = torch.float16 if self.dtype == BF16 else torch.float32
        cfg = Config(dtype=self.dtype, H_t=shape.H_t, n_tap=shape.n_tap, n_layers=shape.L,
                     d=shape.d, n_q=shape.nq, n_kv=shape.nkv, head_dim=shape.hd, inter=shape.I,
                     vocab=shape.V, mask_id=shape.mask_id, max_pos=int(max_pos),
                     eps=float(shape.eps), rope_base=float(shape.rope_base))
        keep = []

        def p(t, name):
            _need(t, name, self.tdtype)
            keep.append(t)
            return t.data_ptr()

        layers = (LayerWeights * shape.L)()
        for l, lw in enumerate(weights["layers"]):
            for k in LayerWeights._fields_:
                setattr(layers[l], k[0], p(lw[k[0]], f"layers[{l}].{k[0]}"))
        w = Weights(emb=p(weights["emb"], "emb"), W_fc=p(weights["W_fc"], "W_fc"),
                    g_ctx=p(weights["g_ctx"], "g_ctx"), g_final=p(weights["g_final"], "g_final"),
                    W_lm=p(weights["W_lm"], "W_lm"), layers=layers)
        handle = ctypes.c_void_p()
        if vocab_range is None:
            _check("dflash_model_create", lib().dflash_model_create(
                ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(handle)))
            self.vocab_range = (0, shape.V)
        else:
            lo, hi = (int(v) for v in vocab_range)
            _check("dflash_model_create_shard", lib().dflash_model_create_shard(
                ctypes.byref(cfg), ctypes.byref(w), lo, hi, ctypes.byref(handle)))
            self.vocab_range = (lo, hi)
        self.handle = handle
        self.max_pos = int(max_pos)

    def close(self):
        if getattr(self, "handle", None):
            lib().dflash_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_size(self, max_batch: int, B: int, max_inject_rows: int) -> int:
        return int(lib().dflash_workspace_size(self.handle, max_batch, B, max_inject_rows))

    def workspace(self, max_batch: int, B: int, max_inject_rows: int, device=None) -> torch.Tensor:
        return new_workspace(self.workspace_size(max_batch, B, max_inject_rows), device)


def new_workspace(nbytes: int, device=None, stream=None) -> torch.Tensor:
    """A zero-filled, 256-byte aligned device workspace of ``nbytes`` bytes."""
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")
    assert ws.data_ptr() % 256 == 0
    _check("dflash_workspace_init", lib().dflash_workspace_init(_ptr(ws), ws.numel(),
                                                                _stream(stream)))
    return ws


def verify_workspace_size(batch: int, B: int, V: int) -> int:
    return int(lib().dflash_verify_workspace_size(batch, B, V))


def inject_kv(model: Model, taps: Sequence[torch.Tensor], cu_rows: torch.Tensor,
              start_pos: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              ws: torch.Tensor, stream=None):
    s = model.shape
    batch = start_pos.numel()
    n_rows = taps[0].shape[0]
    if len(taps) != s.n_tap:
        raise ValueError(f"expected {s.n_tap} taps")
    for i, t in enumerate(taps):
        _need(t, f"taps[{i}]", model.tdtype, (n_rows, s.H_t))
    _need(cu_rows, "cu_rows", torch.int32, (batch + 1,))
    _need(start_pos, "start_pos", torch.int32)
    _need(k_cache, "k_cache", model.cache_dtype)
    _need(v_cache, "v_cache", model.cache_dtype, k_cache.shape)
    if k_cache.dim() != 5 or tuple(k_cache.shape[:3]) != (s.L, batch, s.nkv) or k_cache.shape[4] != s.hd:
        raise ValueError("k_cache must be [L, batch, n_kv, cap, head_dim]")
    _need(ws, "ws", torch.uint8)
    arr = (ctypes.c_void_p * s.n_tap)(*[t.data_ptr() for t in taps])
    _check("dflash_inject_kv", lib().dflash_inject_kv(
        model.handle, arr, _ptr(cu_rows), _ptr(start_pos), batch, n_rows, _ptr(k_cache),
        _ptr(v_cache), k_cache.shape[3], _ptr(ws), ws.numel(), _stream(stream)))


def draft_block(model: Model, anchor: torch.Tensor, ctx_len: torch.Tensor, k_cache: torch.Tensor,
                v_cache: torch.Tensor, B: int, n_steps: int, draft_tokens: torch.Tensor,
                ws: torch.Tensor, commit_step: Optional[torch.Tensor] = None,
                logits_dbg: Optional[torch.Tensor] = None, stream=None):
    s = model.shape
    batch = anchor.numel()
    _need(anchor, "anchor", torch.int32)
    _need(ctx_len, "ctx_len", torch.int32, (batch,))
    _need(k_cache, "k_cache", model.cache_dtype)
    _need(v_cache, "v_cache", model.cache_dtype, k_cache.shape)
    if k_cache.dim() != 5 or tuple(k_cache.shape[:3]) != (s.L, batch, s.nkv) or k_cache.shape[4] != s.hd:
        raise ValueError("k_cache must be [L, batch, n_kv, cap, head_dim]")
    _need(draft_tokens, "draft_tokens", torch.int32, (batch, B))
    if commit_step is not None:
        _need(commit_step, "commit_step", torch.int32, (batch, B))
    if logits_dbg is not None:
        _need(logits_dbg, "logits_dbg", torch.float32, (n_steps, batch, B, s.V))
    _need(ws, "ws", torch.uint8)
    _check("dflash_draft_block", lib().dflash_draft_block(
        model.handle, _ptr(anchor), _ptr(ctx_len), _ptr(k_cache), _ptr(v_cache), k_cache.shape[3],
        batch, B, n_steps, _ptr(draft_tokens), _ptr(commit_step), _ptr(logits_dbg), _ptr(ws),
        ws.numel(), _stream(stream)))


def _need_pages(model: Model, k_pool, v_pool, page_table, batch):
    s = model.shape
    _need(k_pool, "k_pool", model.cache_dtype)
    _need(v_pool, "v_pool", model.cache_dtype, k_pool.shape)
    if k_pool.dim() != 5 or k_pool.shape[0] != s.L or k_pool.shape[2] != s.nkv or \
            k_pool.shape[4] != s.hd:
        raise ValueError("k_pool must be [L, n_pages, n_kv, page_size, head_dim]")
    _need(page_table, "page_table", torch.int32)
    if page_table.dim() != 2 or page_table.shape[0] != batch:
        raise ValueError("page_table must be [batch, max_pages]")
    return k_pool.shape[1], k_pool.shape[3], page_table.shape[1]


def inject_kv_paged(model: Model, taps: Sequence[torch.Tensor], cu_rows: torch.Tensor,
                    start_pos: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                    page_table: torch.Tensor, ws: torch.Tensor, stream=None):
    """Injection through a page table into K/V page pools (prefix sharing); see
    dflash_inject_kv_paged in include/dflash.h."""
    s = model.shape
    batch = start_pos.numel()
    n_rows = taps[0].shape[0]
    if len(taps) != s.n_tap:
        raise ValueError(f"expected {s.n_tap} taps")
    for i, t in enumerate(taps):
        _need(t, f"taps[{i}]", model.tdtype, (n_rows, s.H_t))
    _need(cu_rows, "cu_rows", torch.int32, (batch + 1,))
    _need(start_pos, "start_pos", torch.int32)
    n_pages, page, max_pages = _need_pages(model, k_pool, v_pool, page_table, batch)
    _need(ws, "ws", torch.uint8)
    arr = (ctypes.c_void_p * s.n_tap)(*[t.data_ptr() for t in taps])
    _check("dflash_inject_kv_paged", lib().dflash_inject_kv_paged(
        model.handle, arr, _ptr(cu_rows), _ptr(start_pos), batch, n_rows, _ptr(k_pool),
        _ptr(v_pool), n_pages, page, _ptr(page_table), max_pages, _ptr(ws), ws.numel(),
        _stream(stream)))


def draft_block_paged(model: Model, anchor: torch.Tensor, ctx_len: torch.Tensor,
                      k_pool: torch.Tensor, v_pool: torch.Tensor, page_table: torch.Tensor, B: int,
                      n_steps: int, draft_tokens: torch.Tensor, ws: torch.Tensor,
                      commit_step: Optional[torch.Tensor] = None,
                      logits_dbg: Optional[torch.Tensor] = None, stream=None):
    """Greedy drafting over paged K/V; see dflash_draft_block_paged in include/dflash.h."""
    s = model.shape
    batch = anchor.numel()
    _need(anchor, "anchor", torch.int32)
    _need(ctx_len, "ctx_len", torch.int32, (batch,))
    n_pages, page, max_pages = _need_pages(model, k_pool, v_pool, page_table, batch)
    _need(draft_tokens, "draft_tokens", torch.int32, (batch, B))
    if commit_step is not None:
        _need(commit_step, "commit_step", torch.int32, (batch, B))
    if logits_dbg is not None:
        _need(logits_dbg, "logits_dbg", torch.float32, (n_steps, batch, B, s.V))
    _need(ws, "ws", torch.uint8)
    _check("dflash_draft_block_paged", lib().dflash_draft_block_paged(
        model.handle, _ptr(anchor), _ptr(ctx_len), _ptr(k_pool), _ptr(v_pool), n_pages, page,
        _ptr(page_table), max_pages, batch, B, n_steps, _ptr(draft_tokens), _ptr(commit_step),
        _ptr(logits_dbg), _ptr(ws), ws.numel(), _stream(stream)))


def draft_block_sampled(model: Model, anchor: torch.Tensor, ctx_len: torch.Tensor,
                        k_cache: torch.Tensor, v_cache: torch.Tensor, B: int, n_steps: int,
                        temperature: float, seed: int, offset: int, draft_tokens: torch.Tensor,
                        draft_logits: torch.Tensor, ws: torch.Tensor,
                        commit_step: Optional[torch.Tensor] = None, stream=None):
    """Sampled (temperature) drafting; ``draft_logits`` (float32 or bfloat16
    [batch, B, V]) receives each position's committing-step logits, the q rows of
    sampled verify.  See dflash_draft_block_sampled in include/dflash.h."""
    s = model.shape
    batch = anchor.numel()
    _need(anchor, "anchor", torch.int32)
    _need(ctx_len, "ctx_len", torch.int32, (batch,))
    _need(k_cache, "k_cache", model.cache_dtype)
    _need(v_cache, "v_cache", model.cache_dtype, k_cache.shape)
    if k_cache.dim() != 5 or tuple(k_cache.shape[:3]) != (s.L, batch, s.nkv) or k_cache.shape[4] != s.hd:
        raise ValueError("k_cache must be [L, batch, n_kv, cap, head_dim]")
    _need(draft_tokens, "draft_tokens", torch.int32, (batch, B))
    if commit_step is not None:
        _need(commit_step, "commit_step", torch.int32, (batch, B))
    dt = {torch.bfloat16: BF16, torch.float32: F32}.get(draft_logits.dtype)
    if dt is None:
        raise TypeError("draft_logits must be bfloat16 or float32")
    _need(draft_logits, "draft_logits", None, (batch, B, s.V))
    _need(ws, "ws", torch.uint8)
    _check("dflash_draft_block_sampled", lib().dflash_draft_block_sampled(
        model.handle, _ptr(anchor), _ptr(ctx_len), _ptr(k_cache), _ptr(v_cache), k_cache.shape[3],
        batch, B, n_steps, float(temperature), int(seed) & (2**64 - 1), int(offset) & (2**64 - 1),
        _ptr(draft_tokens), _ptr(commit_step), _ptr(draft_logits), dt, _ptr(ws), ws.numel(),
        _stream(stream)))


def draft_rows(batch: int, B: int, n_steps: int, step: int) -> int:
    """Masked rows of the batch at a denoising step (the rows of its shard records)."""
    n = int(lib().dflash_draft_rows(batch, B, n_steps, step))
    if n < 0:
        raise DFlashError("dflash_draft_rows", n)
    return n


def _need_kv(model: Model, k_cache, v_cache, batch):
    s = model.shape
    _need(k_cache, "k_cache", model.cache_dtype)
    _need(v_cache, "v_cache", model.cache_dtype, k_cache.shape)
    if k_cache.dim() != 5 or tuple(k_cache.shape[:3]) != (s.L, batch, s.nkv) or k_cache.shape[4] != s.hd:
        raise ValueError("k_cache must be [L, batch, n_kv, cap, head_dim]")


def draft_begin(model: Model, anchor: torch.Tensor, ctx_len: torch.Tensor, cache_cap: int, B: int,
                n_steps: int, ws: torch.Tensor, stream=None):
    batch = anchor.numel()
    _need(anchor, "anchor", torch.int32)
    _need(ctx_len, "ctx_len", torch.int32, (batch,))
    _need(ws, "ws", torch.uint8)
    _check("dflash_draft_begin", lib().dflash_draft_begin(
        model.handle, _ptr(anchor), _ptr(ctx_len), int(cache_cap), batch, B, n_steps, _ptr(ws),
        ws.numel(), _stream(stream)))


def draft_forward_shard(model: Model, ctx_len: torch.Tensor, k_cache: torch.Tensor,
                        v_cache: torch.Tensor, B: int, n_steps: int, step: int,
                        shard_stats: torch.Tensor, ws: torch.Tensor, stream=None):
    """One step's forward; shard_stats (float32 [rows, 4]) receives this shard's
    (max, id bits, sumexp, 0) record of every masked row."""
    batch = ctx_len.numel()
    _need(ctx_len, "ctx_len", torch.int32, (batch,))
    _need_kv(model, k_cache, v_cache, batch)
    _need(shard_stats, "shard_stats", torch.float32, (draft_rows(batch, B, n_steps, step), 4))
    _need(ws, "ws", torch.uint8)
    _check("dflash_draft_forward_shard", lib().dflash_draft_forward_shard(
        model.handle, _ptr(ctx_len), _ptr(k_cache), _ptr(v_cache), k_cache.shape[3], batch, B,
        n_steps, step, _ptr(shard_stats), _ptr(ws), ws.numel(), _stream(stream)))


def draft_commit_shards(model: Model, gathered: torch.Tensor, batch: int, B: int, n_steps: int,
                        step: int, ws: torch.Tensor, stream=None):
    """Merges every shard's records (float32 [world, rows, 4], shards in vocabulary
    order) and commits the step."""
    rows = draft_rows(batch, B, n_steps, step)
    _need(gathered, "gathered", torch.float32)
    if gathered.dim() != 3 or tuple(gathered.shape[1:]) != (rows, 4):
        raise ValueError(f"gathered must be [world, {rows}, 4]")
    _need(ws, "ws", torch.uint8)
    _check("dflash_draft_commit_shards", lib().dflash_draft_commit_shards(
        model.handle, _ptr(gathered), gathered.shape[0], batch, B, n_steps, step, _ptr(ws),
        ws.numel(), _stream(stream)))


def draft_end(model: Model, B: int, n_steps: int, draft_tokens: torch.Tensor, ws: torch.Tensor,
              commit_step: Optional[torch.Tensor] = None, stream=None):
    batch = draft_tokens.shape[0]
    _need(draft_tokens, "draft_tokens", torch.int32, (batch, B))
    if commit_step is not None:
        _need(commit_step, "commit_step", torch.int32, (batch, B))
    _need(ws, "ws", torch.uint8)
    _check("dflash_draft_end", lib().dflash_draft_end(
        model.handle, batch, B, n_steps, _ptr(draft_tokens), _ptr(commit_step), _ptr(ws),
        ws.numel(), _stream(stream)))


def verify_shard(logits_shard: torch.Tensor, vocab_offset: int, row_argmax: torch.Tensor,
                 ws: torch.Tensor, stream=None):
    """Per row of this rank's target-logit columns [batch, B, Vs]: (largest value,
    global id) into row_argmax (float32 [batch * B, 2], the id as int32 bits)."""
    if logits_shard.dim() != 3:
        raise ValueError("logits_shard must be [batch, B, Vs]")
    batch, B, Vs = logits_shard.shape
    dt = {torch.bfloat16: BF16, torch.float32: F32}.get(logits_shard.dtype)
    if dt is None:
        raise TypeError("logits_shard must be bfloat16 or float32")
    _need(logits_shard, "logits_shard")
    _need(row_argmax, "row_argmax", torch.float32, (batch * B, 2))
    _need(ws, "ws", torch.uint8)
    _check("dflash_verify_shard", lib().dflash_verify_shard(
        _ptr(logits_shard), dt, batch, B, Vs, int(vocab_offset), _ptr(row_argmax), _ptr(ws),
        ws.numel(), _stream(stream)))


def verify_merge(gathered: torch.Tensor, draft_tokens: torch.Tensor, V: int,
                 out_tokens: torch.Tensor, out_len: torch.Tensor, seq_lens: torch.Tensor,
                 accept_len: torch.Tensor, next_anchor: torch.Tensor, ws: torch.Tensor,
                 stream=None):
    """Greedy verify from every shard's row argmaxes (float32 [world, batch * B, 2],
    shards in vocabulary order)."""
    batch, B = draft_tokens.shape
    _need(gathered, "gathered", torch.float32)
    if gathered.dim() != 3 or tuple(gathered.shape[1:]) != (batch * B, 2):
        raise ValueError(f"gathered must be [world, {batch * B}, 2]")
    _need(draft_tokens, "draft_tokens", torch.int32, (batch, B))
    _need(out_tokens, "out_tokens", torch.int32)
    if out_tokens.dim() != 2 or out_tokens.shape[0] != batch:
        raise ValueError("out_tokens must be [batch, out_cap]")
    for n, t in (("out_len", out_len), ("seq_lens", seq_lens), ("accept_len", accept_len),
                 ("next_anchor", next_anchor)):
        _need(t, n, torch.int32, (batch,))
    _need(ws, "ws", torch.uint8)
    _check("dflash_verify_merge", lib().dflash_verify_merge(
        _ptr(gathered), gathered.shape[0], _ptr(draft_tokens), batch, B, int(V), _ptr(out_tokens),
        _ptr(out_len), out_tokens.shape[1], _ptr(seq_lens), _ptr(accept_len), _ptr(next_anchor),
        _ptr(ws), ws.numel(), _stream(stream)))


def verify(target_logits: torch.Tensor, draft_tokens: torch.Tensor, out_tokens: torch.Tensor,
           out_len: torch.Tensor, seq_lens: torch.Tensor, accept_len: torch.Tensor,
           next_anchor: torch.Tensor, ws: torch.Tensor, stream=None):
    if target_logits.dim() != 3:
        raise ValueError("target_logits must be [batch, B, V]")
    batch, B, V = target_logits.shape
    dt = {torch.bfloat16: BF16, torch.float32: F32}.get(target_logits.dtype)
    if dt is None:
        raise TypeError("target_logits must be bfloat16 or float32")
    _need(target_logits, "target_logits")
    _need(draft_tokens, "draft_tokens", torch.int32, (batch, B))
    _need(out_tokens, "out_tokens", torch.int32)
    if out_tokens.dim() != 2 or out_tokens.shape[0] != batch:
        raise ValueError("out_tokens must be [batch, out_cap]")
    for n, t in (("out_len", out_len), ("seq_lens", seq_lens), ("accept_len", accept_len),
                 ("next_anchor", next_anchor)):
        _need(t, n, torch.int32, (batch,))
    _need(ws, "ws", torch.uint8)
    _check("dflash_verify", lib().dflash_verify(
        _ptr(target_logits), dt, _ptr(draft_tokens), batch, B, V, _ptr(out_tokens), _ptr(out_len),
        out_tokens.shape[1], _ptr(seq_lens), _ptr(accept_len), _ptr(next_anchor), _ptr(ws),
        ws.numel(), _stream(stream)))


def verify_noalloc(target_logits: torch.Tensor, draft_tokens: torch.Tensor,
                   out_tokens: torch.Tensor, out_len: torch.Tensor, seq_lens: torch.Tensor,
                   accept_len: torch.Tensor, next_anchor: torch.Tensor,
                   error_bits: Optional[torch.Tensor] = None, stream=None):
    """Greedy verify without a workspace, for callers that cannot allocate device
    memory: the library keeps the scratch in a fixed array of its own.  Same
    results as ``verify``; ``error_bits`` (int32 [1] on the device, optional)
    receives the call's device error bits.  Calls that overlap on the GPU race
    on the shared scratch."""
    if target_logits.dim() != 3:
        raise ValueError("target_logits must be [batch, B, V]")
    batch, B, V = target_logits.shape
    dt = {torch.bfloat16: BF16, torch.float32: F32}.get(target_logits.dtype)
    if dt is None:
        raise TypeError("target_logits must be bfloat16 or float32")
    _need(target_logits, "target_logits")
    _need(draft_tokens, "draft_tokens", torch.int32, (batch, B))
    _need(out_tokens, "out_tokens", torch.int32)
    if out_tokens.dim() != 2 or out_tokens.shape[0] != batch:
        raise ValueError("out_tokens must be [batch, out_cap]")
    for n, t in (("out_len", out_len), ("seq_lens", seq_lens), ("accept_len", accept_len),
                 ("next_anchor", next_anchor)):
        _need(t, n, torch.int32, (batch,))
    if error_bits is not None:
        _need(error_bits, "error_bits", torch.int32, (1,))
    _check("dflash_verify_noalloc", lib().dflash_verify_noalloc(
        _ptr(target_logits), dt, _ptr(draft_tokens), batch, B, V, _ptr(out_tokens), _ptr(out_len),
        out_tokens.shape[1], _ptr(seq_lens), _ptr(accept_len), _ptr(next_anchor),
        _ptr(error_bits), _stream(stream)))


def verify_sampled_workspace_size(batch: int, B: int, V: int) -> int:
    return int(lib().dflash_verify_sampled_workspace_size(batch, B, V))


def verify_sampled(target_logits: torch.Tensor, draft_logits: torch.Tensor,
                   draft_tokens: torch.Tensor, temperature: float, seed: int, offset: int,
                   out_tokens: torch.Tensor, out_len: torch.Tensor, seq_lens: torch.Tensor,
                   accept_len: torch.Tensor, next_anchor: torch.Tensor, ws: torch.Tensor,
                   stream=None):
    """Sampled (temperature) verify: speculative sampling of the drafted block
    against the target, draws from Philox4x64-10 under (seed, offset); see
    dflash_verify_sampled in include/dflash.h."""
    if target_logits.dim() != 3:
        raise ValueError("target_logits must be [batch, B, V]")
    batch, B, V = target_logits.shape
    dt = {torch.bfloat16: BF16, torch.float32: F32}.get(target_logits.dtype)
    if dt is None:
        raise TypeError("target_logits must be bfloat16 or float32")
    _need(target_logits, "target_logits")
    _need(draft_logits, "draft_logits", target_logits.dtype, (batch, B, V))
    _need(draft_tokens, "draft_tokens", torch.int32, (batch, B))
    _need(out_tokens, "out_tokens", torch.int32)
    if out_tokens.dim() != 2 or out_tokens.shape[0] != batch:
        raise ValueError("out_tokens must be [batch, out_cap]")
    for n, t in (("out_len", out_len), ("seq_lens", seq_lens), ("accept_len", accept_len),
                 ("next_anchor", next_anchor)):
        _need(t, n, torch.int32, (batch,))
    _need(ws, "ws", torch.uint8)
    _check("dflash_verify_sampled", lib().dflash_verify_sampled(
        _ptr(target_logits), _ptr(draft_logits), dt, _ptr(draft_tokens), batch, B, V,
        float(temperature), int(seed) & (2**64 - 1), int(offset) & (2**64 - 1), _ptr(out_tokens),
        _ptr(out_len), out_tokens.shape[1], _ptr(seq_lens), _ptr(accept_len), _ptr(next_anchor),
        _ptr(ws), ws.numel(), _stream(stream)))


def get_error(ws: torch.Tensor, stream=None) -> int:
    """Reads and clears the device error word (synchronises the stream)."""
    bits = ctypes.c_int32(0)
    _check("dflash_get_error", lib().dflash_get_error(_ptr(ws), _stream(stream), ctypes.byref(bits)))
    return int(bits.value)


def timing_enable(on: bool = True):
    lib().dflash_timing_enable(1 if on else 0)


def timing_read() -> Dict[str, Dict[str, float]]:
    """Per kernel class: total device ms and launch count since the last read."""
    n = len(TIMING_CLASSES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    _check("dflash_timing_read", lib().dflash_timing_read(ms, cnt, n))
    return {TIMING_CLASSES[i]: {"ms": ms[i], "launches": int(cnt[i])} for i in range(n)}


# ---------------------------------------------------------------- test hooks (dflash_debug.h)

_ELEM = {torch.bfloat16: BF16, torch.float16: F16}


def debug_tile_weights(W: torch.Tensor, stream=None) -> torch.Tensor:
    """The pre-tiled streaming image (uint8) of a 16-bit weight W [N, K]."""
    _need(W, "W")
    N, K = W.shape
    Wt = torch.empty(lib().dflash_debug_tiled_bytes(N, K), dtype=torch.uint8, device=W.device)
    _check("dflash_debug_tile_weights", lib().dflash_debug_tile_weights(
        _ptr(W), _ptr(Wt), N, K, _stream(stream)))
    return Wt


def debug_gemm(W: torch.Tensor, X: torch.Tensor, splits: int, err_ws: torch.Tensor, stream=None,
               tiled: bool = False):
    """fp32 split-K partials [splits_used, M, N] of X @ W^T from the tcgen05 core
    (W and X both bf16 or both fp16); ``tiled`` streams W from its pre-tiled image."""
    _need(W, "W")
    _need(X, "X", W.dtype)
    elem = _ELEM[W.dtype]
    N, K = W.shape
    M = X.shape[0]
    nkb = K // 64
    s_req = max(1, min(splits, nkb))
    per = -(-nkb // s_req)
    s_used = -(-nkb // per)
    out = torch.empty((s_used, M, N), dtype=torch.float32, device=W.device)
    used = ctypes.c_int(0)
    if tiled:
        Wt = debug_tile_weights(W, stream)
        _check("dflash_debug_gemm_tiled", lib().dflash_debug_gemm_tiled(
            _ptr(Wt), N, K, _ptr(X), M, elem, s_req, _ptr(out), ctypes.byref(used),
            _ptr(err_ws), _stream(stream)))
    else:
        _check("dflash_debug_gemm", lib().dflash_debug_gemm(
            _ptr(W), N, K, _ptr(X), M, elem, s_req, _ptr(out), ctypes.byref(used),
            _ptr(err_ws), _stream(stream)))
    assert used.value == s_used
    return out


def debug_lmhead(W: torch.Tensor, X: torch.Tensor, err_ws: torch.Tensor, want_logits=True,
                 stream=None, tiled: bool = False):
    """(stats [M, tiles, 4] as (max, idx, sumexp, 0), logits [M, N] or None);
    ``tiled`` streams W from its pre-tiled image."""
    _need(W, "W")
    _need(X, "X", W.dtype)
    elem = _ELEM[W.dtype]
    N, K = W.shape
    M = X.shape[0]
    tiles = -(-N // 128)
    stats = torch.empty((M, tiles, 4), dtype=torch.float32, device=W.device)
    logits = torch.empty((M, N), dtype=torch.float32, device=W.device) if want_logits else None
    if tiled:
        Wt = debug_tile_weights(W, stream)
        _check("dflash_debug_lmhead_tiled", lib().dflash_debug_lmhead_tiled(
            _ptr(Wt), N, K, _ptr(X), M, elem, _ptr(stats), _ptr(logits), _ptr(err_ws),
            _stream(stream)))
    else:
        _check("dflash_debug_lmhead", lib().dflash_debug_lmhead(
            _ptr(W), N, K, _ptr(X), M, elem, _ptr(stats), _ptr(logits), _ptr(err_ws),
            _stream(stream)))
    return stats, logits


def debug_attn_schedule(sched: int) -> None:
    """Process-wide draft attention schedule: 0 the split-KV grid with its
    chunk planned on the device (default), 1 persistent, 2 the split-KV grid on
    the tcgen05 kernel where it applies (tests and tuning)."""
    _check("dflash_debug_attn_schedule", lib().dflash_debug_attn_schedule(int(sched)))


def debug_sample_math(w: torch.Tensor, d: torch.Tensor):
    """Per-entry sampling arithmetic of the draw kernels (tests): returns
    (g2, l2), the log2-unit Gumbel variate of each Philox word in `w`
    (int64 holding the uint64 bits) and log2(1 - 2^d) for each d < 0."""
    assert w.is_cuda and d.is_cuda and w.dtype == torch.int64 and d.dtype == torch.float32
    assert w.is_contiguous() and d.is_contiguous() and w.numel() == d.numel()
    n = w.numel()
    g2 = torch.empty(n, dtype=torch.float32, device=w.device)
    l2 = torch.empty_like(g2)
    _check("dflash_debug_sample_math",
           lib().dflash_debug_sample_math(_ptr(w), _ptr(d), n, _ptr(g2), _ptr(l2), _stream(None)))
    return g2, l2


def debug_attn_chunk(keys: int) -> None:
    """Process-wide split-KV chunk (keys, multiple of 64) of the draft attention;
    0 restores the library's rule (tests and tuning only)."""
    _check("dflash_debug_attn_chunk", lib().dflash_debug_attn_chunk(int(keys)))


def debug_attn_plan(ctx_len: torch.Tensor, req_valid: torch.Tensor, B: int, n_kv: int, cap: int,
                    chunk_min: int, slots: int):
    """The draft attention planner on these context lengths (device int32
    tensors), on the current stream (tests): returns (chunk, items) with items
    the (request, kv head, chunk index, context length) of each CTA of the
    attention grid, in launch order."""
    n = 4 + 2 * int(ctx_len.numel()) * n_kv * ((cap + chunk_min - 1) // chunk_min)
    out = torch.full((n,), -1, dtype=torch.int32, device=ctx_len.device)
    _check("dflash_debug_attn_plan", lib().dflash_debug_attn_plan(
        ctx_len.data_ptr(), req_valid.data_ptr(), int(ctx_len.numel()), int(B), int(n_kv),
        int(cap), int(chunk_min), int(slots), out.data_ptr(), n,
        torch.cuda.current_stream().cuda_stream))
    h = out.cpu().tolist()
    items = [(h[4 + 2 * i] >> 16, (h[4 + 2 * i] >> 8) & 255, h[4 + 2 * i] & 255, h[5 + 2 * i])
             for i in range(h[1])]
    return h[0], items


def debug_attn_slots(head_dim: int, rows: int, B: int) -> int:
    """Resident CTAs of the draft attention's split-KV grid kernel (tests)."""
    r = lib().dflash_debug_attn_slots(int(head_dim), int(rows), int(B))
    if r < 0:
        raise RuntimeError(f"dflash_debug_attn_slots: {r}")
    return r


def debug_gemm_streamk(W: torch.Tensor, X: torch.Tensor, stream=None):
    """(X @ W^T as float32 [M, N] through the stream-K schedule, the workspace's
    error bits); W and X both bf16 or both fp16."""
    _need(W, "W")
    _need(X, "X", W.dtype)
    N, K = W.shape
    M = X.shape[0]
    Wt = debug_tile_weights(W, stream)
    out = torch.full((M, N), float("nan"), dtype=torch.float32, device=W.device)
    ws = new_workspace(lib().dflash_debug_gemm_streamk_ws_bytes(M), W.device, stream)
    _check("dflash_debug_gemm_streamk", lib().dflash_debug_gemm_streamk(
        _ptr(Wt), N, K, _ptr(X), M, _ELEM[W.dtype], _ptr(out), _ptr(ws), ws.numel(),
        _stream(stream)))
    return out, get_error(ws, stream)


def debug_gemm_schedule(sched: int) -> None:
    """Process-wide schedule of the draft and injection GEMMs: 0 the library's
    default (stream-K LM head, fixed-split projections), 1 fixed K splits
    everywhere, 2 stream-K everywhere (tests and tuning)."""
    _check("dflash_debug_gemm_schedule", lib().dflash_debug_gemm_schedule(int(sched)))


def debug_gemm_mode(mode: int) -> None:
    """Process-wide GEMM launch mode for tiled weights: 0 the library's rule,
    1 single CTAs, 2 CTA pairs (tests only)."""
    _check("dflash_debug_gemm_mode", lib().dflash_debug_gemm_mode(int(mode)))
