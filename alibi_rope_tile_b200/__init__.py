"""B200 (sm_100a) attention core: a thin ctypes binding of ``libattn_rope_tile.so``.

The functions here carry the C ABI's names (``include/attn_rope_tile.h``) and only
marshal arguments: they read shapes, dtypes and data pointers from torch CUDA tensors,
allocate outputs with torch when the caller gives none, pass the current torch stream,
and raise ``AttnError`` on a non-zero status. Every step of the computation runs in the
library's CUDA kernels; there is no fallback of any kind. If the library has not been
built, the first call raises ``RuntimeError`` (build it with
``python -m alibi_rope_tile_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn_rope_tile.so")

ATTN_F32, ATTN_BF16 = 0, 1
STATUS = {0: "ATTN_OK", -1: "ATTN_ERR_ARG", -2: "ATTN_ERR_ALIGN", -3: "ATTN_ERR_UNSUPPORTED",
          -4: "ATTN_ERR_CUDA", -5: "ATTN_ERR_TIMEOUT", -6: "ATTN_ERR_WORKSPACE",
          -7: "ATTN_ERR_DEVICE_ARG"}

_P, _I, _L, _F, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t
_FP = ctypes.POINTER(ctypes.c_float)

# (name, restype, argtypes) of every exported entry point
SIGNATURES = {
    "attn_prefill": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _L, _F, _I, _I, _FP, _I, _P]),
    "attn_prefill_workspace_size": (_S, [_I, _I, _I, _I, _F, _I]),
    "attn_prefill_ws": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _L, _F, _I, _I, _FP, _I, _P, _S,
                             _P]),
    "attn_prefill_host_workspace_size": (_S, [_I, _I, _I, _I, _I, _F, _I]),
    "attn_prefill_host": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _L, _F, _I, _I, _FP, _I, _P, _S,
                               _P]),
    "attn_decode_workspace_size": (_S, [_I, _I, _I, _I, _I]),
    "attn_decode": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _FP, _I, _P, _S,
                         _P]),
    "attn_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _FP, _I,
                                 _P]),
    "attn_kv_append": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "attn_prefill_chunk": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _FP,
                                _I, _P]),
    "attn_kv_write": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_decode_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _FP,
                               _I, _P, _S, _P]),
    "attn_kv_write_paged": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "attn_decode_latent_workspace_size": (_S, [_I, _I, _I, _I, _I]),
    "attn_block_fused_workspace_size": (_S, [_I, _I, _I, _I, _I, _I]),
    "attn_fold_rmsnorm_gamma": (_I, [_P, _P, _P, _I, _I, _P]),
    "attn_block_fused": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _L, _F, _I, _I,
                              _FP, _F, _I, _P, _S, _P]),
    "attn_decode_latent": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _FP, _I, _P, _S,
                                _P]),
    "attn_block_workspace_size": (_S, [_I, _I, _I, _I, _I, _I, _I]),
    "attn_block": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _L, _F, _I, _I, _FP, _I,
                        _P, _S, _P]),
    "attn_alibi_slopes": (None, [_I, _FP]),
    "attn_sync_status": (_I, [_P]),
    "attn_last_error": (_I, [ctypes.c_char_p, _S]),
    "attn_version": (ctypes.c_char_p, []),
}


class AttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded on first use; raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m alibi_rope_tile_b200.build)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(status: int) -> None:
    if status != 0:
        buf = ctypes.create_string_buffer(512)
        lib().attn_last_error(buf, 512)
        raise AttnError(status, buf.value.decode(errors="replace"))


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return ATTN_F32
    if t.dtype == torch.bfloat16:
        return ATTN_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _dev(t: Optional[torch.Tensor], name: str, dtype=None) -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def _shape(t: Optional[torch.Tensor], shape, name: str) -> None:
    """Raise unless ``t`` (when given) has exactly ``shape``: the library derives every index
    from the sizes it is passed, so a tensor of another shape would be read or written out of
    bounds."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _slopes(slopes, H: int):
    if slopes is None:
        return None
    vals = [float(x) for x in (slopes.tolist() if hasattr(slopes, "tolist") else slopes)]
    if len(vals) != H:
        raise ValueError(f"alibi_slopes needs {H} values, got {len(vals)}")
    return (ctypes.c_float * H)(*vals)


def alibi_slopes(H: int) -> list:
    """The library's ALiBi schedule 2^(-8(h+1)/H) (computed by attn_alibi_slopes)."""
    buf = (ctypes.c_float * H)()
    lib().attn_alibi_slopes(H, buf)
    return list(buf)


def attn_prefill_workspace_size(B: int, T: int, KV: int, hd: int, rope_base: float,
                                dtype=torch.bfloat16) -> int:
    """Bytes of scratch the key rotation pass of attn_prefill uses (0: the keys are turned
    inside the attention kernel)."""
    dt = ATTN_BF16 if dtype == torch.bfloat16 else ATTN_F32
    return int(lib().attn_prefill_workspace_size(B, T, KV, hd, float(rope_base), dt))


def attn_prefill(q, k, v, out=None, lse=None, *, pos0: int = 0, rope_base: float = 0.0,
                 causal: bool = True, window: int = 0, alibi_slopes: Optional[Sequence] = None,
                 workspace=None, turn_keys_first: bool = True, stream=None):
    """q [B,T,H,hd], k/v [B,T,KV,hd] (CUDA, fp32 or bf16) -> out [B,T,H,hd] (and lse [B,H,T]).

    Where a separate key rotation pass applies (bf16, hd 64 or 128, RoPE on) the keys are turned
    once into ``workspace`` (a device byte tensor of attn_prefill_workspace_size bytes;
    allocated here when not given) before the attention kernel; ``turn_keys_first=False``
    turns them inside the attention kernel instead (no workspace)."""
    B, T, H, hd = q.shape
    KV = k.shape[2]
    if k.shape != (B, T, KV, hd) or v.shape != k.shape:
        raise ValueError(f"k and v must be [B,T,KV,hd] matching q {tuple(q.shape)}")
    _shape(out, q.shape, "out")
    _shape(lse, (B, H, T), "lse")
    dt = q.dtype
    if out is None:
        out = torch.empty_like(q)
    ws_ptr, ws_bytes = 0, 0
    if turn_keys_first:
        need = attn_prefill_workspace_size(B, T, KV, hd, rope_base, dt)
        if need > 0:
            if workspace is None:
                workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
            ws_ptr = _dev(workspace, "workspace")
            ws_bytes = workspace.numel() * workspace.element_size()
    st = lib().attn_prefill_ws(_dev(q, "q"), _dev(k, "k", dt), _dev(v, "v", dt), _dev(out, "out", dt),
                               _dev(lse, "lse", torch.float32), B, T, H, KV, hd, int(pos0),
                               float(rope_base), int(bool(causal)), int(window),
                               _slopes(alibi_slopes, H), _dtype(q), ws_ptr, ws_bytes, _stream(stream))
    _check(st)
    return out


def _host(t: Optional[torch.Tensor], name: str, dtype=None) -> int:
    if t is None:
        return 0
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def attn_prefill_host_workspace_size(B: int, T: int, H: int, KV: int, hd: int, rope_base: float,
                                     dtype=torch.bfloat16) -> int:
    dt = ATTN_BF16 if dtype == torch.bfloat16 else ATTN_F32
    return int(lib().attn_prefill_host_workspace_size(B, T, H, KV, hd, float(rope_base), dt))


def attn_prefill_host(q, k, v, out=None, lse=None, *, pos0: int = 0, rope_base: float = 0.0,
                      causal: bool = True, window: int = 0, alibi_slopes: Optional[Sequence] = None,
                      workspace=None, stream=None):
    """attn_prefill on HOST tensors (pinned memory lets the copies overlap the attention):
    q [B,T,H,hd], k/v [B,T,KV,hd] -> out [B,T,H,hd] (and lse [B,H,T]) in host memory, written
    once the stream reaches the end of the call. ``workspace``: a device byte tensor of
    attn_prefill_host_workspace_size bytes (allocated here when not given)."""
    B, T, H, hd = q.shape
    KV = k.shape[2]
    if k.shape != (B, T, KV, hd) or v.shape != k.shape:
        raise ValueError(f"k and v must be [B,T,KV,hd] matching q {tuple(q.shape)}")
    _shape(out, q.shape, "out")
    _shape(lse, (B, H, T), "lse")
    dt = q.dtype
    if out is None:
        out = torch.empty(q.shape, dtype=dt, pin_memory=True)
    need = attn_prefill_host_workspace_size(B, T, H, KV, hd, rope_base, dt)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    st = lib().attn_prefill_host(_host(q, "q"), _host(k, "k", dt), _host(v, "v", dt), _host(out, "out", dt),
                                 _host(lse, "lse", torch.float32), B, T, H, KV, hd, int(pos0),
                                 float(rope_base), int(bool(causal)), int(window), _slopes(alibi_slopes, H),
                                 _dtype(q), _dev(workspace, "workspace"),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)
    return out


def _decode_shapes(q, kcache, vcache, seqlens, qpos, out, lse) -> None:
    B, H, hd = q.shape
    if kcache.dim() != 4 or kcache.shape[0] != B or kcache.shape[3] != hd:
        raise ValueError(f"kcache must be [B={B},Lmax,KV,hd={hd}], got {tuple(kcache.shape)}")
    _shape(vcache, kcache.shape, "vcache")
    _shape(seqlens, (B,), "seqlens")
    _shape(qpos, (B,), "qpos")
    _shape(out, q.shape, "out")
    _shape(lse, (B, H), "lse")


def attn_decode_workspace_size(B: int, H: int, KV: int, hd: int, Lmax: int) -> int:
    return int(lib().attn_decode_workspace_size(B, H, KV, hd, Lmax))


def attn_decode(q, kcache, vcache, seqlens, qpos, out=None, lse=None, workspace=None, *,
                rope_base: float = 0.0, window: int = 0, alibi_slopes=None, stream=None):
    """q [B,H,hd] (not rotated), caches [B,Lmax,KV,hd], seqlens/qpos [B] int32 -> out [B,H,hd]."""
    B, H, hd = q.shape
    _, Lmax, KV, _ = kcache.shape
    _decode_shapes(q, kcache, vcache, seqlens, qpos, out, lse)
    dt = q.dtype
    if out is None:
        out = torch.empty_like(q)
    need = attn_decode_workspace_size(B, H, KV, hd, Lmax)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib().attn_decode(_dev(q, "q"), _dev(kcache, "kcache", dt), _dev(vcache, "vcache", dt),
                           _dev(seqlens, "seqlens", torch.int32), _dev(qpos, "qpos", torch.int32),
                           _dev(out, "out", dt), _dev(lse, "lse", torch.float32), B, H, KV, hd, Lmax,
                           float(rope_base), int(window), _slopes(alibi_slopes, H), _dtype(q),
                           _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                           _stream(stream))
    _check(st)
    return out


def attn_decode_noalloc(q, kcache, vcache, seqlens, qpos, out, lse=None, *,
                        rope_base: float = 0.0, window: int = 0, alibi_slopes=None, stream=None):
    """attn_decode for callers that cannot allocate device memory: the split partials use
    the library's fixed scratch array, so no workspace is passed; ``out`` must be given."""
    B, H, hd = q.shape
    _, Lmax, KV, _ = kcache.shape
    if out is None:
        raise ValueError("attn_decode_noalloc writes into a caller-given out [B,H,hd]")
    _decode_shapes(q, kcache, vcache, seqlens, qpos, out, lse)
    dt = q.dtype
    st = lib().attn_decode_noalloc(_dev(q, "q"), _dev(kcache, "kcache", dt),
                                   _dev(vcache, "vcache", dt), _dev(seqlens, "seqlens", torch.int32),
                                   _dev(qpos, "qpos", torch.int32), _dev(out, "out", dt),
                                   _dev(lse, "lse", torch.float32), B, H, KV, hd, Lmax,
                                   float(rope_base), int(window), _slopes(alibi_slopes, H),
                                   _dtype(q), _stream(stream))
    _check(st)
    return out


def attn_prefill_chunk(q, kcache, vcache, seqlens, qpos0, out=None, lse=None, *,
                       rope_base: float = 0.0, causal: bool = True, window: int = 0,
                       alibi_slopes=None, stream=None):
    """q [B,Tq,H,hd] (not rotated; row i at position qpos0[b]+i) over caches [B,Lmax,KV,hd]
    (keys rotated), slots < seqlens[b] -> out [B,Tq,H,hd] (and lse [B,H,Tq])."""
    B, Tq, H, hd = q.shape
    _, Lmax, KV, _ = kcache.shape
    _shape(kcache, (B, Lmax, KV, hd), "kcache")
    _shape(vcache, kcache.shape, "vcache")
    _shape(seqlens, (B,), "seqlens")
    _shape(qpos0, (B,), "qpos0")
    _shape(out, q.shape, "out")
    _shape(lse, (B, H, Tq), "lse")
    dt = q.dtype
    if out is None:
        out = torch.empty_like(q)
    st = lib().attn_prefill_chunk(_dev(q, "q"), _dev(kcache, "kcache", dt), _dev(vcache, "vcache", dt),
                                  _dev(seqlens, "seqlens", torch.int32), _dev(qpos0, "qpos0", torch.int32),
                                  _dev(out, "out", dt), _dev(lse, "lse", torch.float32), B, Tq, H, KV, hd,
                                  Lmax, float(rope_base), int(bool(causal)), int(window),
                                  _slopes(alibi_slopes, H), _dtype(q), _stream(stream))
    _check(st)
    return out


def attn_kv_write(k_new, v_new, kcache, vcache, pos0, *, rope_base: float = 0.0, stream=None):
    """Write k_new, v_new [B,Tn,KV,hd] into cache slots pos0[b] .. pos0[b]+Tn-1 (keys rotated)."""
    B, Tn, KV, hd = k_new.shape
    Lmax = kcache.shape[1]
    _shape(v_new, k_new.shape, "v_new")
    _shape(kcache, (B, Lmax, KV, hd), "kcache")
    _shape(vcache, kcache.shape, "vcache")
    _shape(pos0, (B,), "pos0")
    dt = k_new.dtype
    st = lib().attn_kv_write(_dev(k_new, "k_new"), _dev(v_new, "v_new", dt), _dev(kcache, "kcache", dt),
                             _dev(vcache, "vcache", dt), _dev(pos0, "pos0", torch.int32), B, Tn, KV, hd,
                             Lmax, float(rope_base), _dtype(k_new), _stream(stream))
    _check(st)


def attn_decode_paged(q, kpages, vpages, block_table, seqlens, qpos, out=None, lse=None,
                      workspace=None, *, rope_base: float = 0.0, window: int = 0, alibi_slopes=None,
                      stream=None):
    """q [B,H,hd] (not rotated) over page pools [num_pages,page_size,KV,hd] through
    block_table [B,max_blocks] int32 -> out [B,H,hd]."""
    B, H, hd = q.shape
    num_pages, page_size, KV, _ = kpages.shape
    max_blocks = block_table.shape[1]
    _shape(kpages, (num_pages, page_size, KV, hd), "kpages")
    _shape(vpages, kpages.shape, "vpages")
    _shape(block_table, (B, max_blocks), "block_table")
    _shape(seqlens, (B,), "seqlens")
    _shape(qpos, (B,), "qpos")
    _shape(out, q.shape, "out")
    _shape(lse, (B, H), "lse")
    dt = q.dtype
    if out is None:
        out = torch.empty_like(q)
    need = attn_decode_workspace_size(B, H, KV, hd, max_blocks * page_size)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib().attn_decode_paged(_dev(q, "q"), _dev(kpages, "kpages", dt), _dev(vpages, "vpages", dt),
                                 _dev(block_table, "block_table", torch.int32),
                                 _dev(seqlens, "seqlens", torch.int32), _dev(qpos, "qpos", torch.int32),
                                 _dev(out, "out", dt), _dev(lse, "lse", torch.float32), B, H, KV, hd,
                                 page_size, num_pages, max_blocks, float(rope_base), int(window),
                                 _slopes(alibi_slopes, H), _dtype(q), _dev(workspace, "workspace"),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)
    return out


def attn_kv_write_paged(k_new, v_new, kpages, vpages, block_table, pos0, *, rope_base: float = 0.0,
                        stream=None):
    """Write k_new, v_new [B,Tn,KV,hd] into the page pools at slots pos0[b] .. pos0[b]+Tn-1."""
    B, Tn, KV, hd = k_new.shape
    num_pages, page_size = kpages.shape[:2]
    max_blocks = block_table.shape[1]
    _shape(v_new, k_new.shape, "v_new")
    _shape(kpages, (num_pages, page_size, KV, hd), "kpages")
    _shape(vpages, kpages.shape, "vpages")
    _shape(block_table, (B, max_blocks), "block_table")
    _shape(pos0, (B,), "pos0")
    dt = k_new.dtype
    st = lib().attn_kv_write_paged(_dev(k_new, "k_new"), _dev(v_new, "v_new", dt),
                                   _dev(kpages, "kpages", dt), _dev(vpages, "vpages", dt),
                                   _dev(block_table, "block_table", torch.int32),
                                   _dev(pos0, "pos0", torch.int32), B, Tn, KV, hd, page_size,
                                   num_pages, max_blocks, float(rope_base), _dtype(k_new),
                                   _stream(stream))
    _check(st)


def attn_decode_latent(q, ccache, W_uk, W_uv, seqlens, qpos, out=None, lse=None, workspace=None, *,
                       window: int = 0, alibi_slopes=None, stream=None):
    """q [B,H,hd] over a latent cache ccache [B,Lmax,dc] with per-head up-projections
    W_uk, W_uv [H,dc,hd] -> out [B,H,hd] (the key up-projection folded into the query)."""
    B, H, hd = q.shape
    _, Lmax, dc = ccache.shape
    _shape(ccache, (B, Lmax, dc), "ccache")
    _shape(W_uk, (H, dc, hd), "W_uk")
    _shape(W_uv, (H, dc, hd), "W_uv")
    _shape(seqlens, (B,), "seqlens")
    _shape(qpos, (B,), "qpos")
    _shape(out, q.shape, "out")
    _shape(lse, (B, H), "lse")
    dt = q.dtype
    if out is None:
        out = torch.empty_like(q)
    need = int(lib().attn_decode_latent_workspace_size(B, H, hd, dc, Lmax))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib().attn_decode_latent(_dev(q, "q"), _dev(ccache, "ccache", dt), _dev(W_uk, "W_uk", dt),
                                  _dev(W_uv, "W_uv", dt), _dev(seqlens, "seqlens", torch.int32),
                                  _dev(qpos, "qpos", torch.int32), _dev(out, "out", dt),
                                  _dev(lse, "lse", torch.float32), B, H, hd, dc, Lmax, int(window),
                                  _slopes(alibi_slopes, H), _dtype(q), _dev(workspace, "workspace"),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)
    return out


def attn_kv_append(k_new, v_new, kcache, vcache, pos, *, rope_base: float = 0.0, stream=None):
    """Write k_new (rotated at pos[b]) and v_new [B,KV,hd] into cache slot pos[b]."""
    B, KV, hd = k_new.shape
    Lmax = kcache.shape[1]
    _shape(v_new, k_new.shape, "v_new")
    _shape(kcache, (B, Lmax, KV, hd), "kcache")
    _shape(vcache, kcache.shape, "vcache")
    _shape(pos, (B,), "pos")
    dt = k_new.dtype
    st = lib().attn_kv_append(_dev(k_new, "k_new"), _dev(v_new, "v_new", dt),
                              _dev(kcache, "kcache", dt), _dev(vcache, "vcache", dt),
                              _dev(pos, "pos", torch.int32), B, KV, hd, Lmax, float(rope_base),
                              _dtype(k_new), _stream(stream))
    _check(st)


def attn_block_workspace_size(B, T, d, H, KV, hd, dtype) -> int:
    code = dtype if isinstance(dtype, int) else (ATTN_F32 if dtype == torch.float32 else ATTN_BF16)
    return int(lib().attn_block_workspace_size(B, T, d, H, KV, hd, code))


def attn_block(x, Wq, Wk, Wv, Wo, out=None, workspace=None, *, H: int, KV: int, pos0: int = 0,
               rope_base: float = 0.0, causal: bool = True, window: int = 0, alibi_slopes=None,
               stream=None):
    """x [B,T,d] -> out [B,T,d] = attention(x Wq, x Wk, x Wv) Wo (weights [in, out])."""
    B, T, d = x.shape
    if H < 1 or KV < 1 or Wq.dim() != 2 or Wq.shape[1] % H:
        raise ValueError(f"Wq must be [d, H*hd] with H={H}, got {tuple(Wq.shape)}")
    hd = Wq.shape[1] // H
    _shape(Wq, (d, H * hd), "Wq")
    _shape(Wk, (d, KV * hd), "Wk")
    _shape(Wv, (d, KV * hd), "Wv")
    _shape(Wo, (H * hd, d), "Wo")
    _shape(out, x.shape, "out")
    dt = x.dtype
    if out is None:
        out = torch.empty_like(x)
    need = attn_block_workspace_size(B, T, d, H, KV, hd, dt)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    st = lib().attn_block(_dev(x, "x"), _dev(Wq, "Wq", dt), _dev(Wk, "Wk", dt), _dev(Wv, "Wv", dt),
                          _dev(Wo, "Wo", dt), _dev(out, "out", dt), B, T, d, H, KV, hd, int(pos0),
                          float(rope_base), int(bool(causal)), int(window), _slopes(alibi_slopes, H),
                          _dtype(x), _dev(workspace, "workspace"),
                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st)
    return out


def attn_block_fused(x, gamma, Wqkv, Wo, out=None, kcache=None, vcache=None, workspace=None, *,
                     H: int, KV: int, pos0: int = 0, rope_base: float = 0.0, causal: bool = True,
                     window: int = 0, alibi_slopes=None, eps: float = 1e-6, stream=None):
    """x [B,T,d] -> x + attention(RMSNorm(x) Wqkv) Wo (Wqkv [d,(H+2KV)hd] = [q|k|v] heads);
    with caches [B,Lmax,KV,hd], the turned keys and the values go to slots pos0 .. pos0+T-1.
    gamma=None: Wqkv already carries gamma (fold_rmsnorm_gamma), so it is not folded again."""
    B, T, d = x.shape
    if H < 1 or KV < 1 or Wqkv.dim() != 2 or Wqkv.shape[1] % (H + 2 * KV):
        raise ValueError(f"Wqkv must be [d, (H+2KV)*hd] with H={H}, KV={KV}, got {tuple(Wqkv.shape)}")
    hd = Wqkv.shape[1] // (H + 2 * KV)
    _shape(Wqkv, (d, (H + 2 * KV) * hd), "Wqkv")
    _shape(Wo, (H * hd, d), "Wo")
    if gamma is not None:
        _shape(gamma, (d,), "gamma")
    _shape(out, x.shape, "out")
    if (kcache is None) != (vcache is None):
        raise ValueError("give both kcache and vcache, or neither")
    if kcache is not None:
        if kcache.dim() != 4:
            raise ValueError(f"kcache must be [B,Lmax,KV,hd], got {tuple(kcache.shape)}")
        _shape(kcache, (B, kcache.shape[1], KV, hd), "kcache")
        _shape(vcache, kcache.shape, "vcache")
    dt = x.dtype
    if out is None:
        out = torch.empty_like(x)
    Lmax = kcache.shape[1] if kcache is not None else 0
    need = int(lib().attn_block_fused_workspace_size(B, T, d, H, KV, hd))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    st = lib().attn_block_fused(_dev(x, "x"), None if gamma is None else _dev(gamma, "gamma", dt),
                                _dev(Wqkv, "Wqkv", dt),
                                _dev(Wo, "Wo", dt), _dev(out, "out", dt), _dev(kcache, "kcache", dt),
                                _dev(vcache, "vcache", dt), Lmax, B, T, d, H, KV, hd, int(pos0),
                                float(rope_base), int(bool(causal)), int(window),
                                _slopes(alibi_slopes, H), float(eps), _dtype(x),
                                _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                _stream(stream))
    _check(st)
    return out


def fold_rmsnorm_gamma(gamma, W, out=None, stream=None):
    """diag(gamma) W for W [d, N] (bf16): weights for attn_block_fused(..., gamma=None, ...)."""
    d, N = W.shape
    _shape(gamma, (d,), "gamma")
    if out is None:
        out = torch.empty_like(W)
    _shape(out, W.shape, "out")
    st = lib().attn_fold_rmsnorm_gamma(_dev(gamma, "gamma", W.dtype), _dev(W, "W", W.dtype),
                                       _dev(out, "out", W.dtype), d, N, _stream(stream))
    _check(st)
    return out


def attn_sync_status(stream=None) -> int:
    """Synchronise and read (then clear) the device error word; raises AttnError if set."""
    st = lib().attn_sync_status(_stream(stream))
    _check(st)
    return st


def attn_version() -> str:
    return lib().attn_version().decode()
