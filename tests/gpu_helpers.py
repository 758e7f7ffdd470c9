"""Helpers of the GPU parity tests: move a seeded workload to the device, run the
library's calls, and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

from tree_speculative_decoding_05_b200 import ddt, inputs

# Tolerances for the attention output against the float64 oracle.  MAX_ABS bounds
# the error of the computation: the weights enter P V as bf16 (rounding to
# nearest: relative error <= 2^-8 each, largely averaging out over many keys) and
# everything else accumulates in fp32.  The output's own rounding to its dtype is
# allowed on top, elementwise: half an ulp of the output dtype at the exact value
# (bf16: 0.0156 for |o| in [4, 8), 0.03125 for |o| in [8, 16)).  No output in that
# dtype can be closer to the exact value than that, and the row-scaled workload
# (cache rows N(0,1) x U(0.5, 2)) has outputs above 8, where a literal 2e-2 bound
# on a bf16 value cannot be met.  The relative L2 bound 5e-3 (over the whole
# compared tensor) and the lse bound 5e-3 take no such allowance.
MAX_ABS = 2e-2
REL_L2 = 5e-3
LSE_MAX_ABS = 5e-3


def out_format(t: torch.Tensor) -> str:
    """Output dtype of a verify call's result: "bf16" or "f32"."""
    return "bf16" if t.dtype == torch.bfloat16 else "f32"


def half_ulp(ref: np.ndarray, fmt: str) -> np.ndarray:
    """Half a unit in the last place of the output dtype at |ref| (the largest
    error of a round-to-nearest conversion of ref to that dtype): bf16 keeps 8
    significant bits, fp32 24; magnitudes below the smallest normal use its ulp."""
    bits = 8 if fmt == "bf16" else 24
    _, ex = np.frexp(np.abs(ref))            # |ref| = m * 2^ex, m in [0.5, 1)
    ex = np.maximum(ex, -125)                # fp32/bf16 smallest normal: 2^-126
    return np.ldexp(1.0, ex - bits - 1)


# Achieved errors of every attention comparison in this session, printed at the
# end of the run by the terminal summary in conftest.py: (label, max-abs, rel-L2,
# lse max-abs, rows compared, rows in the output, largest error beyond the
# output's own rounding).
ERROR_LOG: list[tuple] = []


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def i32(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


class DeviceWorkload:
    def __init__(self, w: inputs.Workload, device="cuda"):
        self.w = w
        self.q_lat = bf16_tensor(w.q_lat, device)
        self.q_rope = bf16_tensor(w.q_rope, device)
        self.c_kv = bf16_tensor(w.c_kv, device)
        self.k_rope = bf16_tensor(w.k_rope, device)
        self.prefix = i32(w.prefix_lens, device)
        self.parents = i32(w.parents, device)
        self.node_tokens = i32(w.node_tokens, device)
        self.target_tokens = i32(w.target_tokens, device)
        self.next_token = i32(w.next_token, device)
        self.next_sibling = i32(w.next_sibling, device)

    def verify(self, num_splits=0, out_dtype=None, want_lse=None, mask=None):
        w = self.w
        if mask is None:
            mask, _, _ = ddt.build_mask(self.parents)
        od = out_dtype or (torch.float32 if w.out_dtype == "f32" else torch.bfloat16)
        status = torch.empty(w.B, dtype=torch.int32, device=self.q_lat.device)
        out, lse = ddt.verify_attn(self.q_lat, self.q_rope, self.c_kv, self.k_rope, self.prefix,
                                   mask, w.softmax_scale, max_prefix=int(w.prefix_lens.max()),
                                   out_dtype=od, want_lse=True if want_lse is None else want_lse,
                                   num_splits=num_splits, status=status)
        return out, lse, status


def compare_attention(out_gpu: np.ndarray, ref: np.ndarray, what: str = "", *, fmt: str):
    """Errors of a GPU result (values of output dtype `fmt`) against float64
    values: max-abs, relative L2 over the compared rows, and the largest error
    beyond the output's own rounding (|gpu - ref| - half_ulp(ref)), which must
    stay within MAX_ABS."""
    g = out_gpu.astype(np.float64)
    err = np.abs(g - ref)
    max_abs = float(err.max()) if err.size else 0.0
    excess = float((err - half_ulp(ref, fmt)).max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(g - ref) / denom) if denom > 0 else float(np.linalg.norm(g - ref))
    ERROR_LOG.append((what, max_abs, rel, None, int(g.shape[0]), None, excess))
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    assert excess <= MAX_ABS, (f"{what}: error beyond the output's rounding {excess:.3e} > "
                               f"{MAX_ABS} (max abs {max_abs:.3e})")
    assert rel <= REL_L2, f"{what}: rel L2 err {rel:.3e} > {REL_L2}"
    return max_abs, rel


def compare_whole(out: torch.Tensor, lse: torch.Tensor | None, w: inputs.Workload, oracle,
                  what: str = "", requests_per_chunk: int | None = None):
    """Every output row of a verify call against the float64 oracle.

    The oracle runs request by request (a chunk of requests at a time, so its
    float64 output stays a few hundred MB at most).  max-abs and the error beyond
    the output's own rounding are over every element (the latter must stay
    within MAX_ABS); relative L2 is ||gpu - ref||_2 / ||ref||_2 over the WHOLE
    output tensor (the sums of squares are accumulated across chunks); lse
    max-abs is over every row.  Returns (max_abs, rel_l2, lse_max_abs) and
    records them."""
    H, DL = w.q_lat.shape[2], w.q_lat.shape[3]
    rows_per_req = w.q_len * H
    if requests_per_chunk is None:
        requests_per_chunk = max(1, (1 << 15) // rows_per_req)
    fmt = out_format(out)
    flat = out.reshape(-1, DL)
    lse_flat = None if lse is None else lse.reshape(-1).cpu().numpy().astype(np.float64)
    max_abs, err2, ref2, lse_err, excess = 0.0, 0.0, 0.0, 0.0, -np.inf
    for b0 in range(0, w.B, requests_per_chunk):
        b1 = min(w.B, b0 + requests_per_chunk)
        rows = np.arange(b0 * rows_per_req, b1 * rows_per_req, dtype=np.int64)
        o_ref, l_ref = oracle.attn_rows(w.q_lat, w.q_rope, w.c_kv, w.k_rope, w.prefix_lens,
                                        w.parents, w.softmax_scale, rows)
        g = flat[b0 * rows_per_req:b1 * rows_per_req].float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all(), f"{what}: non-finite output in requests {b0}..{b1 - 1}"
        d = g - o_ref
        max_abs = max(max_abs, float(np.abs(d).max()))
        excess = max(excess, float((np.abs(d) - half_ulp(o_ref, fmt)).max()))
        err2 += float(np.square(d).sum())
        ref2 += float(np.square(o_ref).sum())
        if lse_flat is not None:
            lse_err = max(lse_err, float(np.abs(lse_flat[rows] - l_ref).max()))
    rel = float(np.sqrt(err2 / ref2)) if ref2 > 0 else float(np.sqrt(err2))
    total = w.B * rows_per_req
    ERROR_LOG.append((what, max_abs, rel, lse_err if lse_flat is not None else None, total,
                      total, excess))
    assert excess <= MAX_ABS, (f"{what}: error beyond the output's rounding {excess:.3e} > "
                               f"{MAX_ABS} (max abs {max_abs:.3e})")
    assert rel <= REL_L2, f"{what}: rel L2 err {rel:.3e} > {REL_L2} (whole output)"
    if lse_flat is not None:
        assert lse_err <= LSE_MAX_ABS, f"{what}: lse err {lse_err:.3e} > {LSE_MAX_ABS}"
    return max_abs, rel, lse_err


def rows_of(out: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    flat = out.reshape(-1, out.shape[-1])
    idx = torch.from_numpy(rows).to(out.device)
    return flat.index_select(0, idx).float().cpu().numpy()


def sample_rows(B, Q, H, n, seed=0, must=()):
    """n distinct flat rows (b*Q + i)*H + h, always including `must`."""
    total = B * Q * H
    rng = np.random.RandomState(seed)
    pick = set(int(r) for r in must if 0 <= r < total)
    if n >= total:
        return np.arange(total, dtype=np.int64)
    while len(pick) < n:
        pick.add(int(rng.randint(total)))
    return np.array(sorted(pick), dtype=np.int64)
