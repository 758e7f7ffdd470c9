"""CPU oracle of the tree-verify path — TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke check and the benchmark's CPU-baseline leg
may import this package.  The product path (the CUDA library and its Python
binding) never imports, links or runs it, and the two share no code: the only
thing both sides consume is the seeded input generator, which holds none of the
method's arithmetic.

The arithmetic lives in ``ddt_oracle.c`` (plain C, double precision, OpenMP over
query rows); this module compiles it on first use and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ddt_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libddt_oracle.so")
_lock = threading.Lock()
_default = None

# Status codes of the oracle (same meaning as the library's per-request codes).
OK, BAD_PARENT, BAD_INDEX, WALK_LIMIT, BAD_PREFIX, BAD_LENGTH = range(6)


def compile_oracle(src: str, out_path: str) -> str:
    """Compile an oracle C source into a shared library at out_path."""
    os.makedirs(os.path.dirname(out_path), exist_ok=True)
    tmp = out_path + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                           "-Wall", "-Wno-unknown-pragmas", src, "-o", tmp, "-lm"])
    os.replace(tmp, out_path)
    return out_path


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/_build/libddt_oracle.so."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_oracle(_SRC, _LIB_PATH)
    return _LIB_PATH


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


class Oracle:
    """One loaded copy of the oracle library (the default one, or a variant that a
    test compiled from a modified source)."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_int64
        lib.oracle_threads.restype = i32
        lib.oracle_visibility.argtypes = [P, i32, P, P]
        lib.oracle_visibility.restype = i32
        lib.oracle_build_mask.argtypes = [P, i32, i32, P, P, P]
        lib.oracle_build_mask.restype = None
        lib.oracle_attn_rows.argtypes = [P, P, P, P, i64, i64, i64, i64, P, P, i32, i32, i32,
                                         i32, i32, ctypes.c_float, P, i64, P, P, P, i64, i32]
        lib.oracle_attn_rows.restype = i32
        lib.oracle_tree_accept.argtypes = [P, P, P, P, i32, i32, P, P, P, P]
        lib.oracle_tree_accept.restype = None
        lib.oracle_tree_build.argtypes = [P, P, P, i32, i32, i32, i32, P, P, P, P, P, P, P, P]
        lib.oracle_tree_build.restype = None
        lib.oracle_kv_compact.argtypes = [P, P, i64, i64, i64, i64, i32, i32, i32, P, P, P,
                                          i32, i32, P, P]
        lib.oracle_kv_compact.restype = None
        self.lib = lib

    def threads(self) -> int:
        return int(self.lib.oracle_threads())

    def visibility(self, parents):
        """Explicit Q x Q visibility matrix (uint8), depths, status of one tree."""
        parents = _c(parents, np.int32)
        q = parents.shape[0]
        vis = np.zeros((q, q), dtype=np.uint8)
        depth = np.zeros(q, dtype=np.int32)
        st = self.lib.oracle_visibility(_p(parents), q, _p(vis), _p(depth))
        return vis, depth, int(st)

    def build_mask(self, parents):
        """parents [B, Q] -> (mask uint64 [B, Q, W], depth int32 [B, Q], status int32 [B])."""
        parents = _c(parents, np.int32)
        B, Q = parents.shape
        W = (Q + 63) // 64
        mask = np.zeros((B, Q, W), dtype=np.uint64)
        depth = np.zeros((B, Q), dtype=np.int32)
        status = np.zeros(B, dtype=np.int32)
        self.lib.oracle_build_mask(_p(parents), B, Q, _p(mask), _p(depth), _p(status))
        return mask, depth, status

    def attn_rows(self, q_lat, q_rope, c_kv, k_rope, prefix_lens, parents, softmax_scale, rows,
                  *, want_probs: bool = False, nthreads: int = 0):
        """Attention for selected query rows (flat index (b*Q + i)*H + h).

        q_lat uint16 [B,Q,H,DL], q_rope uint16 [B,Q,H,DR], c_kv uint16 [B,cap,DL],
        k_rope uint16 [B,cap,DR] (bf16 bit patterns).  Returns (out float64 [n, DL],
        lse float64 [n]) and, with want_probs, probs float64 [n, max T]."""
        q_lat = _c(q_lat, np.uint16)
        q_rope = _c(q_rope, np.uint16)
        c_kv = _c(c_kv, np.uint16)
        k_rope = _c(k_rope, np.uint16)
        prefix_lens = _c(prefix_lens, np.int32)
        parents = _c(parents, np.int32)
        rows = _c(rows, np.int64).reshape(-1)
        B, Q, H, DL = q_lat.shape
        DR = q_rope.shape[3]
        n = rows.shape[0]
        out = np.zeros((n, DL), dtype=np.float64)
        lse = np.zeros(n, dtype=np.float64)
        probs = None
        stride = 0
        if want_probs:
            stride = int(prefix_lens.max(initial=0)) + Q
            probs = np.zeros((n, stride), dtype=np.float64)
        cap = c_kv.shape[1]
        rc = self.lib.oracle_attn_rows(
            _p(q_lat), _p(q_rope), _p(c_kv), _p(k_rope), cap * DL, DL, cap * DR, DR,
            _p(prefix_lens), _p(parents), B, Q, H, DL, DR, float(softmax_scale), _p(rows), n,
            _p(out), _p(lse), _p(probs), stride, int(nthreads))
        if rc != 0:
            raise ValueError("oracle: malformed tree or negative prefix in a requested row")
        return (out, lse, probs) if want_probs else (out, lse)

    def attn_all(self, q_lat, q_rope, c_kv, k_rope, prefix_lens, parents, softmax_scale,
                 nthreads: int = 0):
        """Attention for every query row: out float64 [B,Q,H,DL], lse float64 [B,Q,H]."""
        B, Q, H, DL = np.shape(q_lat)
        rows = np.arange(B * Q * H, dtype=np.int64)
        out, lse = self.attn_rows(q_lat, q_rope, c_kv, k_rope, prefix_lens, parents,
                                  softmax_scale, rows, nthreads=nthreads)
        return out.reshape(B, Q, H, DL), lse.reshape(B, Q, H)

    def tree_accept(self, node_tokens, target_tokens, next_token, next_sibling):
        """Returns (path int32 [B,Q], accept_len [B], bonus [B], status [B])."""
        nt = _c(node_tokens, np.int32)
        tt = _c(target_tokens, np.int32)
        fc = _c(next_token, np.int32)
        ns = _c(next_sibling, np.int32)
        B, Q = nt.shape
        path = np.zeros((B, Q), dtype=np.int32)
        alen = np.zeros(B, dtype=np.int32)
        bonus = np.zeros(B, dtype=np.int32)
        status = np.zeros(B, dtype=np.int32)
        self.lib.oracle_tree_accept(_p(nt), _p(tt), _p(fc), _p(ns), B, Q, _p(path), _p(alen),
                                    _p(bonus), _p(status))
        return path, alen, bonus, status

    def tree_build(self, lp, tok, root_token, q_len):
        """Best-first draft tree from per-depth top-k log-probs.
        lp float32 [B,D,K], tok int32 [B,D,K], root_token int32 [B].  Returns a dict of
        parents, node_tokens, depth (int32 [B,Q]), logw (float32 [B,Q]), next_token,
        next_sibling (int32 [B,Q]), n_nodes, status (int32 [B])."""
        lp = _c(lp, np.float32)
        tok = _c(tok, np.int32)
        root = _c(root_token, np.int32)
        B, D, K = lp.shape
        Q = int(q_len)
        r = {k: np.zeros((B, Q), dtype=np.int32) for k in ("parents", "node_tokens", "depth",
                                                           "next_token", "next_sibling")}
        r["logw"] = np.zeros((B, Q), dtype=np.float32)
        r["n_nodes"] = np.zeros(B, dtype=np.int32)
        r["status"] = np.zeros(B, dtype=np.int32)
        self.lib.oracle_tree_build(_p(lp), _p(tok), _p(root), B, D, K, Q, _p(r["parents"]),
                                   _p(r["node_tokens"]), _p(r["depth"]), _p(r["logw"]),
                                   _p(r["next_token"]), _p(r["next_sibling"]), _p(r["n_nodes"]),
                                   _p(r["status"]))
        return r

    def kv_compact(self, c_kv, k_rope, prefix_lens, path, accept_len, capacity=None):
        """Compaction on copies of the caches (uint16 [B,cap,DL] / [B,cap,DR]).
        Returns (c_kv', k_rope', new_prefix_lens, status)."""
        ckv = np.array(c_kv, dtype=np.uint16, copy=True, order="C")
        kr = np.array(k_rope, dtype=np.uint16, copy=True, order="C")
        prefix_lens = _c(prefix_lens, np.int32)
        path = _c(path, np.int32)
        accept_len = _c(accept_len, np.int32)
        B, cap, DL = ckv.shape
        DR = kr.shape[2]
        Q = path.shape[1]
        if capacity is None:
            capacity = cap
        newp = np.zeros(B, dtype=np.int32)
        status = np.zeros(B, dtype=np.int32)
        self.lib.oracle_kv_compact(_p(ckv), _p(kr), cap * DL, DL, cap * DR, DR, int(capacity),
                                   DL, DR, _p(prefix_lens), _p(path), _p(accept_len), B, Q,
                                   _p(newp), _p(status))
        return ckv, kr, newp, status


def default() -> Oracle:
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def threads() -> int:
    return default().threads()


def visibility(parents):
    return default().visibility(parents)


def build_mask(parents):
    return default().build_mask(parents)


def attn_rows(*args, **kwargs):
    return default().attn_rows(*args, **kwargs)


def attn_all(*args, **kwargs):
    return default().attn_all(*args, **kwargs)


def tree_accept(*args, **kwargs):
    return default().tree_accept(*args, **kwargs)


def kv_compact(*args, **kwargs):
    return default().kv_compact(*args, **kwargs)


def tree_build(*args, **kwargs):
    return default().tree_build(*args, **kwargs)
