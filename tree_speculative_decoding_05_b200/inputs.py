"""Seeded synthetic inputs for the tree-verify path.

This module only draws inputs.  It holds none of the arithmetic of the method
(no masking, attention, acceptance or compaction) so that the CPU oracle and the
CUDA path can both be fed from it without sharing any of their own code.

Random numbers come from splitmix64 (Steele, Lea, Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014): element k of a stream with base
state s is mix(s + (k+1) * 0x9E3779B97F4A7C15).  Uniforms take the top 53 bits.
Normals use the Box-Muller transform in float64; values are then rounded to
float32 and to bfloat16, both round-to-nearest-even.

Shapes follow the workloads of the tree-verify step: 64 heads, a 512-wide latent
cache row plus a 64-wide rope row, trees of q_len nodes with depth <= 15 (the
limits of "Building the Foundation: Architecting a Native CUDA DDTree Inference
Engine", section "The Single-Threaded Heap Design").
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

NUM_HEADS = 64
D_LATENT = 512
D_ROPE = 64
MAX_DEPTH = 15
VOCAB = 32000

# Stream tags: each array draws from its own stream of the request's seed.
TAG_PARENTS, TAG_QLAT, TAG_QROPE, TAG_CKV, TAG_KROPE, TAG_TOKENS, TAG_SCALE, TAG_PREFIX = range(8)
TAG_DRAFT_LOGITS, TAG_DRAFT_TOKENS = 8, 9


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_base(seed: int, tag: int, sub: int = 0) -> np.uint64:
    """Base state of the stream (seed, tag, sub)."""
    with np.errstate(over="ignore"):
        s = np.array([(seed * 1_000_003 + tag * 7919 + sub * 104_729) & 0xFFFFFFFFFFFFFFFF],
                     dtype=np.uint64)
        return _mix(s)[0]


def raw_u64(base: np.uint64, start: int, count: int) -> np.ndarray:
    with np.errstate(over="ignore"):
        k = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
        return _mix(np.uint64(base) + k * GOLDEN)


def uniform(base: np.uint64, start: int, count: int) -> np.ndarray:
    """Uniform float64 in [0, 1)."""
    return (raw_u64(base, start, count) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(base: np.uint64, count: int) -> np.ndarray:
    """count standard normals (Box-Muller on consecutive uniform pairs)."""
    pairs = (count + 1) // 2
    u = uniform(base, 0, 2 * pairs)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log1p(-u1))
    th = 2.0 * math.pi * u2
    out = np.empty(2 * pairs, dtype=np.float64)
    out[0::2] = r * np.cos(th)
    out[1::2] = r * np.sin(th)
    return out[:count]


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float -> bfloat16 bit patterns (uint16), via float32, both steps RNE."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# Trees
# --------------------------------------------------------------------------

def random_parents(seed: int, b: int, q_len: int, max_depth: int = MAX_DEPTH) -> np.ndarray:
    """parents[0] = -1; parents[i] uniform over j < i with depth[j] <= max_depth-1."""
    base = stream_base(seed, TAG_PARENTS, b)
    u = uniform(base, 0, max(q_len, 1))
    parents = np.full(q_len, -1, dtype=np.int32)
    depth = np.zeros(q_len, dtype=np.int32)
    for i in range(1, q_len):
        cand = [j for j in range(i) if depth[j] <= max_depth - 1]
        j = cand[min(int(u[i] * len(cand)), len(cand) - 1)]
        parents[i] = j
        depth[i] = depth[j] + 1
    return parents


def chain_parents(q_len: int) -> np.ndarray:
    p = np.arange(-1, q_len - 1, dtype=np.int32)
    return p


def star_parents(q_len: int) -> np.ndarray:
    p = np.zeros(q_len, dtype=np.int32)
    p[0] = -1
    return p


def parents_with_chain(seed: int, b: int, q_len: int, chain_len: int) -> tuple[np.ndarray, np.ndarray]:
    """Random tree (depth <= 15) containing a chain root -> c1 -> ... -> c_chain_len on
    random increasing node indices.  Returns (parents, chain) with chain[0] = 0."""
    assert chain_len <= min(MAX_DEPTH, q_len - 1)
    base = stream_base(seed, TAG_PARENTS, 1000 + b)
    u = uniform(base, 0, 4 * q_len + 8)
    # choose chain_len distinct indices from 1..q_len-1 (partial Fisher-Yates)
    pool = list(range(1, q_len))
    for k in range(chain_len):
        r = k + min(int(u[k] * (len(pool) - k)), len(pool) - k - 1)
        pool[k], pool[r] = pool[r], pool[k]
    chain_nodes = sorted(pool[:chain_len])
    chain = [0] + chain_nodes
    parents = np.full(q_len, -1, dtype=np.int32)
    depth = np.zeros(q_len, dtype=np.int32)
    on_chain = {c: k for k, c in enumerate(chain)}
    for i in range(1, q_len):
        if i in on_chain:
            j = chain[on_chain[i] - 1]
        else:
            cand = [j for j in range(i) if depth[j] <= MAX_DEPTH - 1]
            j = cand[min(int(u[q_len + i] * len(cand)), len(cand) - 1)]
        parents[i] = j
        depth[i] = depth[j] + 1
    assert depth.max() <= MAX_DEPTH
    return parents, np.array(chain, dtype=np.int32)


def retrieve_pointers(parents: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """First-child / next-sibling pointers of a parent array (children in ascending
    node order, -1 terminated).  Input preparation for the accept walk."""
    q = len(parents)
    first = np.full(q, -1, dtype=np.int32)
    nxt = np.full(q, -1, dtype=np.int32)
    last = {}
    for i in range(1, q):
        p = int(parents[i])
        if first[p] == -1:
            first[p] = i
        else:
            nxt[last[p]] = i
        last[p] = i
    return first, nxt


def tree_tokens(seed: int, b: int, parents: np.ndarray, match_prob: float = 0.7,
                force_path: Optional[np.ndarray] = None) -> tuple[np.ndarray, np.ndarray]:
    """Draft tokens (distinct within each sibling set) and target tokens.

    target[cur] equals the token of one of cur's children (uniform) with
    probability match_prob, otherwise a token that no child of cur carries.  With
    force_path, target follows that path exactly and then misses."""
    q = len(parents)
    base = stream_base(seed, TAG_TOKENS, b)
    u = uniform(base, 0, 8 * q + 64)
    k = 0

    def draw() -> float:
        nonlocal k
        v = u[k % len(u)]
        k += 1
        return v

    children: dict[int, list[int]] = {i: [] for i in range(q)}
    for i in range(1, q):
        children[int(parents[i])].append(i)
    node_tokens = np.zeros(q, dtype=np.int32)
    node_tokens[0] = int(draw() * VOCAB)
    for p in range(q):
        used: set[int] = set()
        for c in children[p]:
            t = int(draw() * VOCAB)
            while t in used:
                t = (t + 1) % VOCAB
            used.add(t)
            node_tokens[c] = t
    target = np.zeros(q, dtype=np.int32)
    forced = {}
    if force_path is not None:
        for a, c in zip(force_path[:-1], force_path[1:]):
            forced[int(a)] = int(c)
    for cur in range(q):
        kids = children[cur]
        child_tokens = {int(node_tokens[c]) for c in kids}
        if cur in forced:
            target[cur] = node_tokens[forced[cur]]
            continue
        if force_path is None and kids and draw() < match_prob:
            target[cur] = node_tokens[kids[min(int(draw() * len(kids)), len(kids) - 1)]]
        else:
            t = int(draw() * VOCAB)
            while t in child_tokens:
                t = (t + 1) % VOCAB
            target[cur] = t
    return node_tokens, target


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    """One batch of the tree-verify step.  Arrays are host numpy; bf16 arrays are
    uint16 bit patterns."""
    name: str
    seed: int
    B: int
    q_len: int
    prefix_lens: np.ndarray      # int32 [B]
    capacity: int                # cache rows per request
    parents: np.ndarray          # int32 [B, Q]
    q_lat: np.ndarray            # uint16 [B, Q, H, 512]
    q_rope: np.ndarray           # uint16 [B, Q, H, 64]
    c_kv: np.ndarray             # uint16 [B, capacity, 512]
    k_rope: np.ndarray           # uint16 [B, capacity, 64]
    node_tokens: np.ndarray      # int32 [B, Q]
    target_tokens: np.ndarray    # int32 [B, Q]
    next_token: np.ndarray       # int32 [B, Q]
    next_sibling: np.ndarray     # int32 [B, Q]
    softmax_scale: float
    out_dtype: str               # "f32" or "bf16"
    want_lse: bool
    forced_path: Optional[np.ndarray] = None  # [B, alen] when a path is planted

    @property
    def num_heads(self) -> int:
        return self.q_lat.shape[2]


def _normals_bf16(seed: int, tag: int, sub: int, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return to_bf16_bits(normal(stream_base(seed, tag, sub), n)).reshape(shape)


def make_workload(name: str, seed: int, B: int, q_len: int, prefix_lens, *,
                  heads: int = NUM_HEADS, d_latent: int = D_LATENT, d_rope: int = D_ROPE,
                  out_dtype: str = "bf16", want_lse: bool = False,
                  row_scale_range: Optional[tuple[float, float]] = None,
                  tree: str = "random", chain_len: int = 0,
                  capacity: Optional[int] = None, match_prob: float = 0.7) -> Workload:
    """Draw a batch.  Arrays are drawn in the order parents -> q_lat -> q_rope ->
    c_kv -> k_rope -> tokens, each request from its own sub-stream."""
    prefix_lens = np.asarray(prefix_lens, dtype=np.int32).reshape(B)
    cap = int(capacity) if capacity is not None else int(prefix_lens.max(initial=0)) + q_len
    parents = np.zeros((B, q_len), dtype=np.int32)
    forced = []
    for b in range(B):
        if tree == "random":
            parents[b] = random_parents(seed, b, q_len)
        elif tree == "chain":
            parents[b] = chain_parents(q_len)
        elif tree == "star":
            parents[b] = star_parents(q_len)
        elif tree == "planted":
            p, ch = parents_with_chain(seed, b, q_len, chain_len)
            parents[b] = p
            forced.append(ch)
        else:
            raise ValueError(tree)
    q_lat = np.stack([_normals_bf16(seed, TAG_QLAT, b, (q_len, heads, d_latent)) for b in range(B)]) \
        if B else np.zeros((0, q_len, heads, d_latent), np.uint16)
    q_rope = np.stack([_normals_bf16(seed, TAG_QROPE, b, (q_len, heads, d_rope)) for b in range(B)]) \
        if B else np.zeros((0, q_len, heads, d_rope), np.uint16)
    c_kv = np.zeros((B, cap, d_latent), dtype=np.uint16)
    k_rope = np.zeros((B, cap, d_rope), dtype=np.uint16)
    for b in range(B):
        rows = int(prefix_lens[b]) + q_len
        if row_scale_range is None:
            c_kv[b, :rows] = _normals_bf16(seed, TAG_CKV, b, (rows, d_latent))
            k_rope[b, :rows] = _normals_bf16(seed, TAG_KROPE, b, (rows, d_rope))
        else:
            lo, hi = row_scale_range
            s = lo + (hi - lo) * uniform(stream_base(seed, TAG_SCALE, b), 0, rows)
            z1 = normal(stream_base(seed, TAG_CKV, b), rows * d_latent).reshape(rows, d_latent)
            z2 = normal(stream_base(seed, TAG_KROPE, b), rows * d_rope).reshape(rows, d_rope)
            c_kv[b, :rows] = to_bf16_bits(z1 * s[:, None])
            k_rope[b, :rows] = to_bf16_bits(z2 * s[:, None])
    node_tokens = np.zeros((B, q_len), dtype=np.int32)
    target = np.zeros((B, q_len), dtype=np.int32)
    nt = np.zeros((B, q_len), dtype=np.int32)
    ns = np.zeros((B, q_len), dtype=np.int32)
    for b in range(B):
        fp = forced[b] if forced else None
        node_tokens[b], target[b] = tree_tokens(seed, b, parents[b], match_prob, fp)
        nt[b], ns[b] = retrieve_pointers(parents[b])
    return Workload(name=name, seed=seed, B=B, q_len=q_len, prefix_lens=prefix_lens, capacity=cap,
                    parents=parents, q_lat=q_lat, q_rope=q_rope, c_kv=c_kv, k_rope=k_rope,
                    node_tokens=node_tokens, target_tokens=target, next_token=nt, next_sibling=ns,
                    softmax_scale=float(np.float32(1.0 / math.sqrt(192.0))), out_dtype=out_dtype,
                    want_lse=want_lse, forced_path=np.stack(forced) if forced else None)


@dataclasses.dataclass
class DraftBatch:
    """Per-depth top-k draft distributions of a batch: lp float32 [B, D, K] (log-
    probabilities, each row descending), tok int32 [B, D, K] (distinct per row),
    root_token int32 [B]."""
    lp: np.ndarray
    tok: np.ndarray
    root_token: np.ndarray


def draft_batch(seed: int, B: int, D: int, K: int, *, vocab: int = VOCAB,
                temperature: float = 8.0, quantum: float = 0.0, sort: bool = True) -> DraftBatch:
    """Synthetic drafter output.  Row (b, d) has K logits z ~ N(0, 1) * temperature
    and one tail logit ln(vocab - K) standing for the rest of the vocabulary (each of
    its tokens at logit 0); lp is the log-softmax of the K head logits over all
    K + 1, rounded to float32 and sorted descending.  quantum > 0 rounds lp to
    multiples of quantum (to force equal weights); sort=False keeps draw order."""
    z = normal(stream_base(seed, TAG_DRAFT_LOGITS, 0), B * D * K).reshape(B, D, K) * temperature
    tail = math.log(vocab - K)
    m = np.maximum(z.max(axis=2, keepdims=True), tail)
    lse = m + np.log(np.exp(z - m).sum(axis=2, keepdims=True) + np.exp(tail - m))
    lp = z - lse
    if quantum > 0:
        lp = np.round(lp / quantum) * quantum
    if sort:
        lp = -np.sort(-lp, axis=2)
    tok = np.zeros((B, D, K), dtype=np.int32)
    roots = np.zeros(B, dtype=np.int32)
    for b in range(B):
        r = raw_u64(stream_base(seed, TAG_DRAFT_TOKENS, b), 0, 1 + D * K)
        roots[b] = int(r[0] % np.uint64(vocab))
        for d in range(D):
            row: list[int] = []
            for x in r[1 + d * K: 1 + (d + 1) * K]:
                t = int(x % np.uint64(vocab))
                while t in row:  # distinct within a row
                    t = (t + 1) % vocab
                row.append(t)
            tok[b, d] = row
    return DraftBatch(lp=lp.astype(np.float32), tok=tok, root_token=roots)


def subset(w: Workload, idx) -> Workload:
    """The requests `idx` of a workload (every per-request array sliced alike)."""
    idx = np.asarray(idx, dtype=np.int64)
    per_request = ("prefix_lens", "parents", "q_lat", "q_rope", "c_kv", "k_rope", "node_tokens",
                   "target_tokens", "next_token", "next_sibling")
    kw = {k: np.ascontiguousarray(getattr(w, k)[idx]) for k in per_request}
    if w.forced_path is not None:
        kw["forced_path"] = np.ascontiguousarray(w.forced_path[idx])
    return dataclasses.replace(w, B=int(len(idx)), **kw)


def ragged_prefixes(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    u = uniform(stream_base(seed, TAG_PREFIX, 0), 0, B)
    return (lo + np.floor(u * (hi - lo + 1))).astype(np.int32)


# The five tree-verify workloads.  Seeds are 1000 + index.
CONFIG_NAMES = {
    0: "1 req x q9 x P256 (fp32 out)",
    1: "8 req x q33 x P1024",
    2: "64 req x q33 x P4096",
    3: "64 req x q65 x P~U[256,8192] (row-scaled cache, lse)",
    4: "1 req x q33 x P32768 (split-KV, planted depth-15 path)",
}


def config(idx: int, **overrides) -> Workload:
    seed = 1000 + idx
    if idx == 0:
        kw = dict(B=1, q_len=9, prefix_lens=[256], out_dtype="f32")
    elif idx == 1:
        kw = dict(B=8, q_len=33, prefix_lens=[1024] * 8)
    elif idx == 2:
        kw = dict(B=64, q_len=33, prefix_lens=[4096] * 64)
    elif idx == 3:
        kw = dict(B=64, q_len=65, prefix_lens=ragged_prefixes(seed, 64, 256, 8192),
                  want_lse=True, row_scale_range=(0.5, 2.0))
    elif idx == 4:
        kw = dict(B=1, q_len=33, prefix_lens=[32768], tree="planted", chain_len=15)
    else:
        raise ValueError(idx)
    kw.update(overrides)
    return make_workload(CONFIG_NAMES[idx], seed, **kw)
