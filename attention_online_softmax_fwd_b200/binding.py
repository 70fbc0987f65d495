"""ctypes binding of libattn_b200.so (the C ABI declared in include/attn_b200.h).

Argument marshalling only: shape/dtype checks, output allocation through
torch, and the call into the library on torch's current CUDA stream. Every
step of the computation runs in the library's kernels. If the library is not
built, every entry point raises :class:`AttnError`; there is no fallback.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libattn_b200.so"

STATUS = {
    0: "ATTN_OK",
    1: "ATTN_ERR_INVALID_ARG",
    2: "ATTN_ERR_UNSUPPORTED",
    3: "ATTN_ERR_CUDA",
    4: "ATTN_ERR_DEVICE_BOUNDS",
    5: "ATTN_ERR_TIMEOUT",
}


class AttnError(RuntimeError):
    def __init__(self, msg, status=None):
        super().__init__(msg)
        self.status = status


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t

SIGNATURES = {
    "attn_status_string": (ctypes.c_char_p, [_I]),
    "attn_abi_version": (_I, []),
    "attn_prefill": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "attn_prefill_blasst": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _F, _P, _P, _P, _P]),
    "attn_prefill_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P]),
    "attn_decode_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "attn_decode_blasst_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "attn_decode_skip_passes": (_I, [_I, _I, _I, _I, _I, _I]),
    "attn_decode_paged": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _I, _P, _P,
                               _P, _SZ, _P, _P, _P, _P]),
    "attn_decode_paged_blasst_heads": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _I, _P,
                                            _P, _P, _SZ, _P, _P, _P, _P]),
    "attn_kv_append": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P]),
    "attn_decode_paged_fp8": (_I, [_P, _P, _P, _F, _F, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P,
                                   _P, _SZ, _P, _P]),
    "attn_decode_paged_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _I, _P, _P,
                                       _P, _P, _P]),
    "attn_read_device_status": (_I, [ctypes.POINTER(_I), _I]),
    "attn_set_library_status": (_I, [_I]),
    "attn_debug_prefill_timeout": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, ctypes.c_ulonglong, _I,
                                        _P, _P]),
}

NOALLOC_SCRATCH_BYTES = 16 << 20   # ATTN_NOALLOC_SCRATCH_BYTES


def lib_path() -> str:
    return os.path.join(HERE, _LIB_NAME)


def load_library():
    """Load the in-tree library (raises AttnError when it is missing)."""
    global _lib
    if _lib is None:
        path = lib_path()
        if not os.path.exists(path):
            raise AttnError(f"{_LIB_NAME} is not built (python -m attention_online_softmax_fwd_b200.build)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(status: int, what: str):
    if status != 0:
        raise AttnError(f"{what} failed: {STATUS.get(status, status)}", status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, ndim, name):
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or t.dim() != ndim:
        raise AttnError(f"{name}: expected a {ndim}-d {dtype} tensor")
    if not t.is_cuda or not t.is_contiguous():
        raise AttnError(f"{name}: expected a contiguous CUDA tensor")


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


def read_device_status(clear: bool = True) -> int:
    """Library-wide device status word (synchronises the device); written only
    while set_library_status(True) is in effect on the device."""
    out = ctypes.c_int(0)
    _check(load_library().attn_read_device_status(ctypes.byref(out), int(clear)), "attn_read_device_status")
    return out.value


def set_library_status(enable: bool) -> None:
    """Switch the library's device status word on the current device on or off."""
    _check(load_library().attn_set_library_status(int(bool(enable))), "attn_set_library_status")


def _counter(t, name):
    """A one-element int64 device tensor used as the library's unsigned 64-bit counter."""
    if t is None:
        return None
    _need(t, torch.int64, 1, name)
    if t.numel() != 1:
        raise AttnError(f"{name}: expected one element")
    return t


# ------------------------------------------------------------------ prefill

def _prefill_args(q, k, v, out, lse, return_lse):
    _need(q, torch.bfloat16, 4, "q")
    _need(k, torch.bfloat16, 4, "k")
    _need(v, torch.bfloat16, 4, "v")
    B, S, Hq, D = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[1] != S or k.shape[3] != D:
        raise AttnError("k/v must be [B, S, Hkv, D] matching q")
    o = torch.empty_like(q) if out is None else out
    _need(o, torch.bfloat16, 4, "out")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, torch.float32, 3, "lse")
    return B, S, Hq, k.shape[2], D, o, lse


def prefill(q, k, v, causal: bool = True, scale: float | None = None, out=None, lse=None,
            return_lse: bool = True, stream=None):
    """Dense prefill attention: q [B,S,Hq,D], k/v [B,S,Hkv,D] bf16 -> (o, lse [B,Hq,S] fp32)."""
    B, S, Hq, Hkv, D, o, lse = _prefill_args(q, k, v, out, lse, return_lse)
    scale = default_scale(D) if scale is None else scale
    st = load_library().attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, S, D,
                                     int(bool(causal)), scale, _stream_handle(stream))
    _check(st, "attn_prefill")
    return o, lse


def prefill_paged(q, k_pages, v_pages, block_table, seq_lens, scale: float | None = None, out=None, lse=None,
                  device_status=None, return_lse: bool = True, stream=None):
    """Chunked prefill over a paged KV cache: q [B,Sq,Hq,D] bf16 are the Sq newest
    tokens of each sequence (their K/V already in the pages); row i of sequence b
    sees its cached keys 0 .. seq_lens[b] - Sq + i. -> (o [B,Sq,Hq,D], lse [B,Hq,Sq])."""
    _need(q, torch.bfloat16, 4, "q")
    _need(k_pages, torch.bfloat16, 4, "k_pages")
    _need(v_pages, torch.bfloat16, 4, "v_pages")
    _need(block_table, torch.int32, 2, "block_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    B, Sq, Hq, D = q.shape
    P, page_size, Hkv, _ = k_pages.shape
    scale = default_scale(D) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    st = load_library().attn_prefill_paged(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), _ptr(o), _ptr(lse), B, Sq, Hq,
        Hkv, D, page_size, block_table.shape[1], P, scale, _ptr(device_status), _stream_handle(stream))
    _check(st, "attn_prefill_paged")
    return o, lse


def kv_append(k_new, v_new, k_pages, v_pages, block_table, start_pos, device_status=None, stream=None):
    """Write new tokens' K/V ([N,T,Hkv,D] bf16) into the page pools in place:
    token t of sequence b goes to position start_pos[b] + t through block_table."""
    _need(k_new, torch.bfloat16, 4, "k_new")
    _need(v_new, torch.bfloat16, 4, "v_new")
    _need(k_pages, torch.bfloat16, 4, "k_pages")
    _need(v_pages, torch.bfloat16, 4, "v_pages")
    _need(block_table, torch.int32, 2, "block_table")
    _need(start_pos, torch.int32, 1, "start_pos")
    N, T, Hkv, D = k_new.shape
    P, page_size, _, _ = k_pages.shape
    st = load_library().attn_kv_append(
        _ptr(k_new), _ptr(v_new), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(start_pos), N, T, Hkv, D,
        page_size, block_table.shape[1], P, _ptr(device_status), _stream_handle(stream))
    _check(st, "attn_kv_append")


def prefill_skip_mask_shape(B, Hq, S):
    return (B, Hq, -(-S // 128), -(-S // 64))


def prefill_blasst(q, k, v, lam: float, causal: bool = True, scale: float | None = None, out=None,
                   lse=None, skip_mask=True, device_status=None, return_lse: bool = True, stream=None,
                   skipped_tiles=None):
    """Prefill with the BLASST tile skip. Returns (o, lse, skip_mask) where
    skip_mask [B, Hq, ceil(S/128), ceil(S/64)] uint8 holds 1 (skipped) / 0 (kept)
    for visited tiles and 2 for tiles never visited. ``skipped_tiles`` (a
    one-element int64 device tensor) receives the count of skipped decisions
    added to its value."""
    B, S, Hq, Hkv, D, o, lse = _prefill_args(q, k, v, out, lse, return_lse)
    scale = default_scale(D) if scale is None else scale
    mask = None
    if skip_mask is True:
        mask = torch.full(prefill_skip_mask_shape(B, Hq, S), 2, dtype=torch.uint8, device=q.device)
    elif isinstance(skip_mask, torch.Tensor):
        mask = skip_mask
    st = load_library().attn_prefill_blasst(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, S, D,
                                            int(bool(causal)), scale, lam, _ptr(mask),
                                            _ptr(_counter(skipped_tiles, "skipped_tiles")), _ptr(device_status),
                                            _stream_handle(stream))
    _check(st, "attn_prefill_blasst")
    return o, lse, mask


# ------------------------------------------------------------------ decode

def decode_workspace_bytes(num_seqs, Hq, D, max_pages, page_size, split_tokens) -> int:
    """Workspace of the dense decode."""
    return int(load_library().attn_decode_workspace_bytes(num_seqs, Hq, D, max_pages, page_size, split_tokens))


def decode_skip_passes(num_seqs, Hq, Hkv, max_pages, page_size, split_tokens) -> int:
    """Passes over K of the tile-skip decode for these sizes (1 or 2; 0 if rejected)."""
    return int(load_library().attn_decode_skip_passes(num_seqs, Hq, Hkv, max_pages, page_size, split_tokens))


def decode_blasst_workspace_bytes(num_seqs, Hq, D, max_pages, page_size, split_tokens) -> int:
    """Workspace of the tile-skip decode (scores, maxima and chunk partials)."""
    return int(load_library().attn_decode_blasst_workspace_bytes(num_seqs, Hq, D, max_pages, page_size,
                                                                 split_tokens))


def decode_skip_mask_shape(num_seqs, Hkv, max_pages, page_size):
    return (num_seqs, Hkv, -(-max_pages * page_size // 64))


def _decode(q, k_pages, v_pages, block_table, seq_lens, lam, scale, split_tokens, out, lse, workspace,
            skip_mask, device_status, return_lse, stream, per_head=False, skipped_tiles=None):
    _need(q, torch.bfloat16, 3, "q")
    _need(k_pages, torch.bfloat16, 4, "k_pages")
    _need(v_pages, torch.bfloat16, 4, "v_pages")
    _need(block_table, torch.int32, 2, "block_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    N, Hq, D = q.shape
    P, page_size, Hkv, Dk = k_pages.shape
    if v_pages.shape != k_pages.shape or Dk != D or block_table.shape[0] != N or seq_lens.shape[0] != N:
        raise AttnError("inconsistent decode shapes")
    max_pages = block_table.shape[1]
    scale = default_scale(D) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    if lse is None and return_lse:
        lse = torch.empty((N, Hq), dtype=torch.float32, device=q.device)
    skip_path = (lam > 0 or (skip_mask is not None and skip_mask is not False) or per_head
                 or skipped_tiles is not None)
    size_fn = decode_blasst_workspace_bytes if skip_path else decode_workspace_bytes
    need = size_fn(N, Hq, D, max_pages, page_size, split_tokens)
    if need == 0:
        raise AttnError("invalid decode configuration", 1)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    mask = None
    if skip_mask is True:
        mask = torch.full(decode_skip_mask_shape(N, Hq if per_head else Hkv, max_pages, page_size), 2,
                          dtype=torch.uint8, device=q.device)
    elif isinstance(skip_mask, torch.Tensor):
        mask = skip_mask
    fn = load_library().attn_decode_paged_blasst_heads if per_head else load_library().attn_decode_paged
    st = fn(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), N, Hq, Hkv, D, page_size,
        max_pages, P, scale, lam, split_tokens, _ptr(o), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(mask), _ptr(_counter(skipped_tiles, "skipped_tiles")),
        _ptr(device_status), _stream_handle(stream))
    _check(st, "attn_decode_paged_blasst_heads" if per_head else "attn_decode_paged")
    return o, lse, mask


def decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale=None, split_tokens: int = 1024,
                 out=None, lse=None, workspace=None, device_status=None, return_lse=True, stream=None):
    """Single-token paged decode (dense). Returns (o [N,Hq,D] bf16, lse [N,Hq] fp32)."""
    o, lse, _ = _decode(q, k_pages, v_pages, block_table, seq_lens, 0.0, scale, split_tokens, out, lse,
                        workspace, None, device_status, return_lse, stream)
    return o, lse


def decode_paged_blasst(q, k_pages, v_pages, block_table, seq_lens, lam: float, scale=None,
                        split_tokens: int = 1024, out=None, lse=None, workspace=None, skip_mask=True,
                        device_status=None, return_lse=True, stream=None, rows_per_unit: str = "group",
                        skipped_tiles=None):
    """Paged decode with the BLASST tile skip. Returns (o, lse, skip_mask).

    rows_per_unit="group": one decision per (sequence, KV head, tile) for the G
    query heads that share the KV head (mask [N, Hkv, tiles]); "head": one per
    query head (mask [N, Hq, tiles]). ``skipped_tiles`` (one-element int64
    device tensor) receives the count of skipped decisions added to it. The
    workspace, when given, must hold decode_blasst_workspace_bytes(...)."""
    if rows_per_unit not in ("group", "head"):
        raise AttnError("rows_per_unit must be 'group' or 'head'")
    return _decode(q, k_pages, v_pages, block_table, seq_lens, lam, scale, split_tokens, out, lse,
                   workspace, skip_mask, device_status, return_lse, stream, per_head=rows_per_unit == "head",
                   skipped_tiles=skipped_tiles)


def decode_paged_fp8(q, k_codes, v_codes, k_scale: float, v_scale: float, block_table, seq_lens, scale=None,
                     split_tokens: int = 1024, out=None, lse=None, workspace=None, device_status=None,
                     return_lse=True, stream=None):
    """Dense paged decode over FP8 E4M3 code pools (uint8 [P, page_size, Hkv, D]) with
    one scale per pool: K = k_scale * e4m3(k_codes), V = v_scale * e4m3(v_codes).
    Returns (o [N,Hq,D] bf16, lse [N,Hq] fp32)."""
    _need(q, torch.bfloat16, 3, "q")
    _need(k_codes, torch.uint8, 4, "k_codes")
    _need(v_codes, torch.uint8, 4, "v_codes")
    _need(block_table, torch.int32, 2, "block_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    N, Hq, D = q.shape
    P, page_size, Hkv, Dk = k_codes.shape
    if v_codes.shape != k_codes.shape or Dk != D or block_table.shape[0] != N or seq_lens.shape[0] != N:
        raise AttnError("inconsistent decode shapes")
    max_pages = block_table.shape[1]
    scale = default_scale(D) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    if lse is None and return_lse:
        lse = torch.empty((N, Hq), dtype=torch.float32, device=q.device)
    need = decode_workspace_bytes(N, Hq, D, max_pages, page_size, split_tokens)
    if need == 0:
        raise AttnError("invalid decode configuration", 1)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = load_library().attn_decode_paged_fp8(
        _ptr(q), _ptr(k_codes), _ptr(v_codes), float(k_scale), float(v_scale), _ptr(block_table),
        _ptr(seq_lens), N, Hq, Hkv, D, page_size, max_pages, P, scale, split_tokens, _ptr(o), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(device_status),
        _stream_handle(stream))
    _check(st, "attn_decode_paged_fp8")
    return o, lse


def decode_paged_noalloc(q, k_pages, v_pages, block_table, seq_lens, scale=None, split_tokens: int = 1024,
                         out=None, lse=None, device_status=None, return_lse=True, stream=None):
    """Dense paged decode through the entry point that allocates nothing: the
    split partials go to the library's fixed 16 MiB device scratch instead of a
    caller workspace (for callers that cannot allocate device memory at decode
    time). Calls on one device share that scratch, so they must not overlap on
    the GPU. Returns (o, lse)."""
    _need(q, torch.bfloat16, 3, "q")
    _need(k_pages, torch.bfloat16, 4, "k_pages")
    _need(v_pages, torch.bfloat16, 4, "v_pages")
    _need(block_table, torch.int32, 2, "block_table")
    _need(seq_lens, torch.int32, 1, "seq_lens")
    N, Hq, D = q.shape
    P, page_size, Hkv, _ = k_pages.shape
    scale = default_scale(D) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    if lse is None and return_lse:
        lse = torch.empty((N, Hq), dtype=torch.float32, device=q.device)
    st = load_library().attn_decode_paged_noalloc(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), N, Hq, Hkv, D, page_size,
        block_table.shape[1], P, scale, 0.0, split_tokens, _ptr(o), _ptr(lse), None, _ptr(device_status),
        _stream_handle(stream))
    _check(st, "attn_decode_paged_noalloc")
    return o, lse


def debug_prefill_timeout(q, k, v, wait_limit_ns: int, withhold_step: int, causal: bool = True,
                          scale: float | None = None, device_status=None, stream=None):
    """TEST ONLY: a dense prefill whose pipeline waits give up after
    ``wait_limit_ns`` and whose producer leaves out ring step ``withhold_step``
    (-1: none). The output is undefined after a timeout; ``device_status`` then
    holds ATTN_ERR_TIMEOUT (5). Returns (o, lse)."""
    B, S, Hq, Hkv, D, o, lse = _prefill_args(q, k, v, None, None, True)
    scale = default_scale(D) if scale is None else scale
    st = load_library().attn_debug_prefill_timeout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, S,
                                                   D, int(bool(causal)), scale, int(wait_limit_ns),
                                                   int(withhold_step), _ptr(device_status), _stream_handle(stream))
    _check(st, "attn_debug_prefill_timeout")
    return o, lse
