"""Python binding of libddt (ctypes).  Argument marshalling only: every step of
the path runs in the library's CUDA kernels.  Tensors are torch CUDA tensors;
calls are asynchronous on torch's current stream.

The library must have been built (``python -m tree_speculative_decoding_05_b200.build``
or ``__graft_entry__.build()``); loading fails loudly otherwise — there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

_LIB = None

DDT_OK, DDT_ERR_INVALID_ARG, DDT_ERR_UNSUPPORTED, DDT_ERR_CUDA, DDT_ERR_INPUT = range(5)
REQ_OK, REQ_BAD_PARENT, REQ_BAD_INDEX, REQ_WALK_LIMIT, REQ_BAD_PREFIX, REQ_BAD_LENGTH, \
    REQ_BAD_LP = range(7)
FAULT_WAIT_TIMEOUT = 1
DDT_F32, DDT_BF16 = 0, 1
NUM_HEADS, D_LATENT, D_ROPE, MAX_Q_LEN = 64, 512, 64, 128

EXPORTED_SYMBOLS = (
    "ddt_tree_build", "ddt_build_mask", "ddt_verify_attn", "ddt_verify_attn_workspace_size",
    "ddt_verify_attn_num_splits", "ddt_tree_accept", "ddt_kv_compact", "ddt_accept_compact",
    "ddt_kv_write_block", "ddt_decode_step", "ddt_verify_attn_split_tail",
    "ddt_selftest_bounded_wait",
    "ddt_verify_attn_split_tail_workspace_size",
    "ddt_status_str",
    "ddt_fault_flags", "ddt_version",
)


class DdtError(RuntimeError):
    pass


class AttnArgs(ctypes.Structure):
    """Mirror of ddt_attn_args (field order and types as in include/ddt.h)."""
    _fields_ = [
        ("B", ctypes.c_int32), ("q_len", ctypes.c_int32), ("num_heads", ctypes.c_int32),
        ("d_latent", ctypes.c_int32), ("d_rope", ctypes.c_int32), ("capacity", ctypes.c_int32),
        ("prefix_lens", ctypes.c_void_p), ("q_lat", ctypes.c_void_p), ("q_rope", ctypes.c_void_p),
        ("c_kv", ctypes.c_void_p), ("k_rope", ctypes.c_void_p),
        ("ckv_batch_stride", ctypes.c_int64), ("ckv_row_stride", ctypes.c_int64),
        ("kr_batch_stride", ctypes.c_int64), ("kr_row_stride", ctypes.c_int64),
        ("mask", ctypes.c_void_p), ("softmax_scale", ctypes.c_float), ("out_dtype", ctypes.c_int32),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("max_prefix", ctypes.c_int32),
        ("num_splits", ctypes.c_int32), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("status", ctypes.c_void_p),
    ]


class DecodeArgs(ctypes.Structure):
    """Mirror of ddt_decode_args."""
    _fields_ = [
        ("attn", AttnArgs), ("depth_levels", ctypes.c_int32), ("topk", ctypes.c_int32),
        ("lp", ctypes.c_void_p), ("tok", ctypes.c_void_p), ("root_token", ctypes.c_void_p),
        ("block_ckv", ctypes.c_void_p), ("block_krope", ctypes.c_void_p),
        ("target_continuation", ctypes.c_void_p), ("parents", ctypes.c_void_p),
        ("node_tokens", ctypes.c_void_p), ("depth", ctypes.c_void_p),
        ("next_token", ctypes.c_void_p), ("next_sibling", ctypes.c_void_p),
        ("n_nodes", ctypes.c_void_p), ("target_tokens", ctypes.c_void_p),
        ("path", ctypes.c_void_p), ("accept_len", ctypes.c_void_p), ("status", ctypes.c_void_p),
    ]


def library_path() -> str:
    return _build.LIB_PATH


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libddt.so (raises if it has not been built)."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or library_path()
    if not os.path.exists(p):
        raise DdtError(f"libddt not built ({p} missing); run "
                       "`python -m tree_speculative_decoding_05_b200.build`")
    lib = ctypes.CDLL(p)
    V, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.ddt_tree_build.argtypes = [V, V, V, i32, i32, i32, i32, V, V, V, V, V, V, V, V, V, V]
    lib.ddt_tree_build.restype = i32
    lib.ddt_build_mask.argtypes = [V, i32, i32, V, V, V, V]
    lib.ddt_build_mask.restype = i32
    lib.ddt_verify_attn.argtypes = [ctypes.POINTER(AttnArgs), V]
    lib.ddt_verify_attn.restype = i32
    lib.ddt_verify_attn_workspace_size.argtypes = [ctypes.POINTER(AttnArgs)]
    lib.ddt_verify_attn_workspace_size.restype = ctypes.c_size_t
    lib.ddt_verify_attn_num_splits.argtypes = [ctypes.POINTER(AttnArgs)]
    lib.ddt_verify_attn_num_splits.restype = i32
    lib.ddt_tree_accept.argtypes = [V, V, V, V, i32, i32, V, V, V, V, V]
    lib.ddt_tree_accept.restype = i32
    lib.ddt_kv_compact.argtypes = [V, V, i64, i64, i64, i64, i32, V, V, V, i32, i32, V, V, V]
    lib.ddt_kv_compact.restype = i32
    lib.ddt_accept_compact.argtypes = [V, V, V, V, i32, i32, V, V, i64, i64, i64, i64, i32, V,
                                       V, V, V, V, V, V, V]
    lib.ddt_accept_compact.restype = i32
    lib.ddt_verify_attn_split_tail.argtypes = [ctypes.POINTER(AttnArgs), V]
    lib.ddt_verify_attn_split_tail.restype = i32
    lib.ddt_verify_attn_split_tail_workspace_size.argtypes = [ctypes.POINTER(AttnArgs)]
    lib.ddt_verify_attn_split_tail_workspace_size.restype = ctypes.c_size_t
    lib.ddt_kv_write_block.argtypes = [V, V, i64, i64, i64, i64, i32, V, V, V, i32, i32, V, V]
    lib.ddt_kv_write_block.restype = i32
    lib.ddt_decode_step.argtypes = [ctypes.POINTER(DecodeArgs), V]
    lib.ddt_decode_step.restype = i32
    lib.ddt_selftest_bounded_wait.argtypes = [ctypes.c_uint32, V, V]
    lib.ddt_selftest_bounded_wait.restype = i32
    lib.ddt_status_str.argtypes = [i32]
    lib.ddt_status_str.restype = ctypes.c_char_p
    lib.ddt_fault_flags.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
    lib.ddt_fault_flags.restype = i32
    lib.ddt_version.restype = ctypes.c_char_p
    if path is None:
        _LIB = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, what: str) -> None:
    if rc != DDT_OK:
        msg = load().ddt_status_str(rc).decode()
        raise DdtError(f"{what}: {msg} (status {rc})")


def _req(t: torch.Tensor, dtype: torch.dtype, name: str, contiguous: bool = True) -> None:
    if not t.is_cuda:
        raise DdtError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise DdtError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise DdtError(f"{name} must be contiguous")


# ---------------------------------------------------------------------------
# Calls
# ---------------------------------------------------------------------------

def tree_build(lp: torch.Tensor, tok: torch.Tensor, root_token: torch.Tensor, q_len: int,
               out: Optional[dict] = None, stream=None) -> dict:
    """Best-first draft tree.  lp float32 [B, D, K], tok int32 [B, D, K], root_token
    int32 [B] -> dict of parents, node_tokens, depth, next_token, next_sibling (int32
    [B, Q]), logw (float32 [B, Q]), mask (uint64-as-int64 [B, Q, W]), n_nodes and
    status (int32 [B]).  Tensors given in `out` are written in place."""
    _req(lp, torch.float32, "lp")
    _req(tok, torch.int32, "tok")
    _req(root_token, torch.int32, "root_token")
    B, D, K = lp.shape
    Q = int(q_len)
    W = (Q + 63) // 64
    dev = lp.device
    o = dict(out or {})
    shapes = {"parents": ((B, Q), torch.int32), "node_tokens": ((B, Q), torch.int32),
              "depth": ((B, Q), torch.int32), "next_token": ((B, Q), torch.int32),
              "next_sibling": ((B, Q), torch.int32), "logw": ((B, Q), torch.float32),
              "mask": ((B, Q, W), torch.int64), "n_nodes": ((B,), torch.int32),
              "status": ((B,), torch.int32)}
    for k, (shape, dtype) in shapes.items():
        if k not in o:
            o[k] = torch.empty(shape, dtype=dtype, device=dev)
    rc = load().ddt_tree_build(_ptr(lp), _ptr(tok), _ptr(root_token), B, D, K, Q,
                               _ptr(o["parents"]), _ptr(o["node_tokens"]), _ptr(o["depth"]),
                               _ptr(o["logw"]), _ptr(o["next_token"]), _ptr(o["next_sibling"]),
                               _ptr(o["mask"]), _ptr(o["n_nodes"]), _ptr(o["status"]),
                               _stream(stream))
    _check(rc, "ddt_tree_build")
    return o


def build_mask(parents: torch.Tensor, mask: Optional[torch.Tensor] = None,
               depth: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
               stream=None):
    """parents int32 [B, Q] -> (mask uint64-as-int64 [B, Q, W], depth int32 [B, Q], status int32 [B])."""
    _req(parents, torch.int32, "parents")
    B, Q = parents.shape
    W = (Q + 63) // 64
    dev = parents.device
    mask = mask if mask is not None else torch.empty((B, Q, W), dtype=torch.int64, device=dev)
    depth = depth if depth is not None else torch.empty((B, Q), dtype=torch.int32, device=dev)
    status = status if status is not None else torch.empty((B,), dtype=torch.int32, device=dev)
    rc = load().ddt_build_mask(_ptr(parents), B, Q, _ptr(mask), _ptr(depth), _ptr(status),
                               _stream(stream))
    _check(rc, "ddt_build_mask")
    return mask, depth, status


def _attn_args(q_lat, q_rope, c_kv, k_rope, prefix_lens, mask, softmax_scale, out, lse,
               max_prefix, num_splits, workspace, status) -> AttnArgs:
    B, Q, H, DL = q_lat.shape
    a = AttnArgs()
    a.B, a.q_len, a.num_heads, a.d_latent, a.d_rope = B, Q, H, DL, q_rope.shape[3]
    a.capacity = c_kv.shape[1]
    a.prefix_lens = prefix_lens.data_ptr()
    a.q_lat, a.q_rope = q_lat.data_ptr(), q_rope.data_ptr()
    a.c_kv, a.k_rope = c_kv.data_ptr(), k_rope.data_ptr()
    a.ckv_batch_stride, a.ckv_row_stride = c_kv.stride(0), c_kv.stride(1)
    a.kr_batch_stride, a.kr_row_stride = k_rope.stride(0), k_rope.stride(1)
    a.mask = mask.data_ptr()
    a.softmax_scale = float(softmax_scale)
    a.out_dtype = DDT_F32 if (out is not None and out.dtype == torch.float32) else DDT_BF16
    a.out = out.data_ptr() if out is not None else None
    a.lse = lse.data_ptr() if lse is not None else None
    a.max_prefix = int(max_prefix)
    a.num_splits = int(num_splits)
    a.workspace = workspace.data_ptr() if workspace is not None else None
    a.workspace_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    a.status = status.data_ptr() if status is not None else None
    return a


def verify_attn_workspace_size(q_lat, q_rope, c_kv, k_rope, prefix_lens, mask, softmax_scale,
                               max_prefix: int, num_splits: int = 0) -> tuple[int, int]:
    """(workspace bytes, number of KV splits) the call will use."""
    a = _attn_args(q_lat, q_rope, c_kv, k_rope, prefix_lens, mask, softmax_scale, None, None,
                   max_prefix, num_splits, None, None)
    lib = load()
    return int(lib.ddt_verify_attn_workspace_size(ctypes.byref(a))), \
        int(lib.ddt_verify_attn_num_splits(ctypes.byref(a)))


def verify_attn(q_lat: torch.Tensor, q_rope: torch.Tensor, c_kv: torch.Tensor,
                k_rope: torch.Tensor, prefix_lens: torch.Tensor, mask: torch.Tensor,
                softmax_scale: float, *, max_prefix: int, out: Optional[torch.Tensor] = None,
                out_dtype: torch.dtype = torch.bfloat16, lse: Optional[torch.Tensor] = None,
                want_lse: bool = False, num_splits: int = 0,
                workspace: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                stream=None, split_tail: bool = False):
    """Tree-verify MLA-absorb attention.  q_lat bf16 [B,Q,64,512], q_rope bf16
    [B,Q,64,64], c_kv bf16 [B,cap,512] and k_rope bf16 [B,cap,64] (rows may be
    strided), prefix_lens int32 [B], mask from build_mask; softmax_scale must be
    positive and finite (the library rejects anything else).  Returns (out, lse).
    split_tail=True computes it as a prefix pass, a tree-block pass and an LSE
    merge (ddt_verify_attn_split_tail) instead of one fused pass."""
    for t, n in ((q_lat, "q_lat"), (q_rope, "q_rope")):
        _req(t, torch.bfloat16, n)
    _req(c_kv, torch.bfloat16, "c_kv", contiguous=False)
    _req(k_rope, torch.bfloat16, "k_rope", contiguous=False)
    if c_kv.stride(2) != 1 or k_rope.stride(2) != 1:
        raise DdtError("cache rows must be contiguous in their last dimension")
    _req(prefix_lens, torch.int32, "prefix_lens")
    _req(mask, torch.int64, "mask")
    B, Q, H, _ = q_lat.shape
    dev = q_lat.device
    if out is None:
        out = torch.empty((B, Q, H, 512), dtype=out_dtype, device=dev)
    if lse is None and want_lse:
        lse = torch.empty((B, Q, H), dtype=torch.float32, device=dev)
    a = _attn_args(q_lat, q_rope, c_kv, k_rope, prefix_lens, mask, softmax_scale, out, lse,
                   max_prefix, num_splits, workspace, status)
    lib = load()
    size_fn = (lib.ddt_verify_attn_split_tail_workspace_size if split_tail
               else lib.ddt_verify_attn_workspace_size)
    if workspace is None:
        need = int(size_fn(ctypes.byref(a)))
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
            a.workspace, a.workspace_bytes = workspace.data_ptr(), need
    if split_tail:
        _check(lib.ddt_verify_attn_split_tail(ctypes.byref(a), _stream(stream)),
               "ddt_verify_attn_split_tail")
    else:
        _check(lib.ddt_verify_attn(ctypes.byref(a), _stream(stream)), "ddt_verify_attn")
    return out, lse


def tree_accept(node_tokens, target_tokens, next_token, next_sibling, *, path=None,
                accept_len=None, bonus=None, status=None, stream=None):
    """Greedy accept.  Inputs int32 [B, Q] -> (path [B,Q], accept_len [B], bonus [B], status [B])."""
    for t, n in ((node_tokens, "node_tokens"), (target_tokens, "target_tokens"),
                 (next_token, "next_token"), (next_sibling, "next_sibling")):
        _req(t, torch.int32, n)
    B, Q = node_tokens.shape
    dev = node_tokens.device
    path = path if path is not None else torch.empty((B, Q), dtype=torch.int32, device=dev)
    accept_len = accept_len if accept_len is not None else torch.empty((B,), dtype=torch.int32, device=dev)
    bonus = bonus if bonus is not None else torch.empty((B,), dtype=torch.int32, device=dev)
    status = status if status is not None else torch.empty((B,), dtype=torch.int32, device=dev)
    rc = load().ddt_tree_accept(_ptr(node_tokens), _ptr(target_tokens), _ptr(next_token),
                                _ptr(next_sibling), B, Q, _ptr(path), _ptr(accept_len),
                                _ptr(bonus), _ptr(status), _stream(stream))
    _check(rc, "ddt_tree_accept")
    return path, accept_len, bonus, status


def kv_compact(c_kv, k_rope, prefix_lens, path, accept_len, *, new_prefix_lens=None,
               status=None, stream=None):
    """In-place compaction of the accepted rows.  Returns (new_prefix_lens, status)."""
    _req(c_kv, torch.bfloat16, "c_kv", contiguous=False)
    _req(k_rope, torch.bfloat16, "k_rope", contiguous=False)
    for t, n in ((prefix_lens, "prefix_lens"), (path, "path"), (accept_len, "accept_len")):
        _req(t, torch.int32, n)
    B, Q = path.shape
    dev = c_kv.device
    new_prefix_lens = new_prefix_lens if new_prefix_lens is not None else torch.empty((B,), dtype=torch.int32, device=dev)
    status = status if status is not None else torch.empty((B,), dtype=torch.int32, device=dev)
    rc = load().ddt_kv_compact(_ptr(c_kv), _ptr(k_rope), c_kv.stride(0), c_kv.stride(1),
                               k_rope.stride(0), k_rope.stride(1), c_kv.shape[1],
                               _ptr(prefix_lens), _ptr(path), _ptr(accept_len), B, Q,
                               _ptr(new_prefix_lens), _ptr(status), _stream(stream))
    _check(rc, "ddt_kv_compact")
    return new_prefix_lens, status


def accept_compact(node_tokens, target_tokens, next_token, next_sibling, c_kv, k_rope,
                   prefix_lens, *, path=None, accept_len=None, bonus=None, accept_status=None,
                   new_prefix_lens=None, compact_status=None, stream=None):
    """tree_accept then kv_compact of its path, in one launch.  Returns (path,
    accept_len, bonus, accept_status, new_prefix_lens, compact_status); pass
    new_prefix_lens=prefix_lens to update the prefix lengths in place."""
    for t, n in ((node_tokens, "node_tokens"), (target_tokens, "target_tokens"),
                 (next_token, "next_token"), (next_sibling, "next_sibling"),
                 (prefix_lens, "prefix_lens")):
        _req(t, torch.int32, n)
    _req(c_kv, torch.bfloat16, "c_kv", contiguous=False)
    _req(k_rope, torch.bfloat16, "k_rope", contiguous=False)
    B, Q = node_tokens.shape
    dev = node_tokens.device
    new = lambda shape: torch.empty(shape, dtype=torch.int32, device=dev)
    path = path if path is not None else new((B, Q))
    accept_len = accept_len if accept_len is not None else new((B,))
    bonus = bonus if bonus is not None else new((B,))
    accept_status = accept_status if accept_status is not None else new((B,))
    new_prefix_lens = new_prefix_lens if new_prefix_lens is not None else new((B,))
    compact_status = compact_status if compact_status is not None else new((B,))
    rc = load().ddt_accept_compact(_ptr(node_tokens), _ptr(target_tokens), _ptr(next_token),
                                   _ptr(next_sibling), B, Q, _ptr(c_kv), _ptr(k_rope),
                                   c_kv.stride(0), c_kv.stride(1), k_rope.stride(0),
                                   k_rope.stride(1), c_kv.shape[1], _ptr(prefix_lens), _ptr(path),
                                   _ptr(accept_len), _ptr(bonus), _ptr(accept_status),
                                   _ptr(new_prefix_lens), _ptr(compact_status), _stream(stream))
    _check(rc, "ddt_accept_compact")
    return path, accept_len, bonus, accept_status, new_prefix_lens, compact_status


def kv_write_block(c_kv, k_rope, prefix_lens, block_ckv, block_krope, *, status=None,
                   stream=None):
    """Tree-block KV rows [B, Q, 512] / [B, Q, 64] into the caches at the prefix.
    Returns status int32 [B]."""
    _req(c_kv, torch.bfloat16, "c_kv", contiguous=False)
    _req(k_rope, torch.bfloat16, "k_rope", contiguous=False)
    _req(block_ckv, torch.bfloat16, "block_ckv")
    _req(block_krope, torch.bfloat16, "block_krope")
    _req(prefix_lens, torch.int32, "prefix_lens")
    B, Q = block_ckv.shape[0], block_ckv.shape[1]
    status = status if status is not None else torch.empty((B,), dtype=torch.int32,
                                                           device=c_kv.device)
    rc = load().ddt_kv_write_block(_ptr(c_kv), _ptr(k_rope), c_kv.stride(0), c_kv.stride(1),
                                   k_rope.stride(0), k_rope.stride(1), c_kv.shape[1],
                                   _ptr(prefix_lens), _ptr(block_ckv), _ptr(block_krope), B, Q,
                                   _ptr(status), _stream(stream))
    _check(rc, "ddt_kv_write_block")
    return status


def decode_step_args(state: dict, step: dict, bufs: dict, softmax_scale: float,
                     max_prefix: int, num_splits: int = 0) -> DecodeArgs:
    """Marshal one decode step.  state: prefix_lens, root_token, c_kv, k_rope (updated
    in place by the step); step: lp, tok, q_lat, q_rope, block_ckv, block_krope,
    target_continuation (this step's inputs); bufs: mask, out, lse (or None),
    workspace (or None), verify_status, parents, node_tokens, depth, next_token,
    next_sibling, n_nodes, target_tokens, path, accept_len, status ([4, B])."""
    a = _attn_args(step["q_lat"], step["q_rope"], state["c_kv"], state["k_rope"],
                   state["prefix_lens"], bufs["mask"], softmax_scale, bufs["out"],
                   bufs.get("lse"), max_prefix, num_splits, bufs.get("workspace"),
                   bufs["verify_status"])
    B, D, K = step["lp"].shape
    d = DecodeArgs()
    d.attn = a
    d.depth_levels, d.topk = D, K
    for k in ("lp", "tok", "block_ckv", "block_krope", "target_continuation"):
        setattr(d, k, step[k].data_ptr())
    d.root_token = state["root_token"].data_ptr()
    for k in ("parents", "node_tokens", "depth", "next_token", "next_sibling", "n_nodes",
              "target_tokens", "path", "accept_len", "status"):
        t = bufs.get(k)
        setattr(d, k, t.data_ptr() if t is not None else None)
    return d


def decode_step(args: DecodeArgs, stream=None) -> None:
    """Launch one chained decode step (see decode_step_args)."""
    _check(load().ddt_decode_step(ctypes.byref(args), _stream(stream)), "ddt_decode_step")


def selftest_bounded_wait(timeout_us: int = 2000, stream=None) -> torch.Tensor:
    """Make one bounded wait give up (see ddt.h); returns the device flag it sets."""
    gave_up = torch.zeros((1,), dtype=torch.int32, device="cuda")
    _check(load().ddt_selftest_bounded_wait(int(timeout_us), _ptr(gave_up), _stream(stream)),
           "ddt_selftest_bounded_wait")
    return gave_up


def fault_flags(reset: bool = True) -> int:
    """The library's device fault word (synchronises the device)."""
    v = ctypes.c_uint32(0)
    _check(load().ddt_fault_flags(ctypes.byref(v), int(reset)), "ddt_fault_flags")
    return int(v.value)


def version() -> str:
    return load().ddt_version().decode()
