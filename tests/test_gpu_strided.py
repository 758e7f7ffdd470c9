"""Caches with non-trivial strides (needs a B200).

A serving engine often keeps the 512-wide latent row and the 64-wide rope row of a
token side by side in one 576-wide row, with spare rows per request: c_kv and
k_rope are then views with row stride 576 and a padded batch stride.  Every call
that touches the cache must give, on such views, exactly what it gives on
contiguous arrays (attention within its tolerance against the oracle; the
integer and copy calls bit for bit)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (DeviceWorkload, LSE_MAX_ABS, bf16_tensor, compare_attention, i32,
                         out_format)
from tree_speculative_decoding_05_b200 import ddt, inputs

pytestmark = pytest.mark.gpu

PAD_ROWS = 13


def _combined(w):
    """One [B, cap + PAD_ROWS, 576] buffer holding both caches; returns (buf, c_kv view,
    k_rope view)."""
    B, cap = w.c_kv.shape[:2]
    bits = np.zeros((B, cap + PAD_ROWS, 576), dtype=np.uint16)
    bits[:, :cap, :512] = w.c_kv
    bits[:, :cap, 512:] = w.k_rope
    bits[:, cap:, :] = 0x7FC0  # NaN in the spare rows: never read
    buf = bf16_tensor(bits)
    return buf, buf[:, :, :512], buf[:, :, 512:]


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("split_tail", [False, True])
def test_verify_on_interleaved_cache(split_tail):
    w = inputs.make_workload("strided", 31, 3, 17, [300, 41, 1000], want_lse=True)
    dw = DeviceWorkload(w)
    _, ckv, kr = _combined(w)
    assert ckv.stride(1) == 576 and ckv.stride(0) == (w.capacity + PAD_ROWS) * 576
    mask, _, _ = ddt.build_mask(dw.parents)
    out, lse = ddt.verify_attn(dw.q_lat, dw.q_rope, ckv, kr, dw.prefix, mask, w.softmax_scale,
                               max_prefix=1000, want_lse=True, split_tail=split_tail)
    torch.cuda.synchronize()
    rows = np.arange(w.B * w.q_len * 64, dtype=np.int64)
    o_ref, l_ref = oracle.attn_rows(w.q_lat, w.q_rope, w.c_kv, w.k_rope, w.prefix_lens,
                                    w.parents, w.softmax_scale, rows)
    compare_attention(out.float().cpu().numpy().reshape(-1, 512), o_ref, "interleaved cache",
                      fmt=out_format(out))
    assert np.abs(lse.reshape(-1).cpu().numpy() - l_ref).max() <= LSE_MAX_ABS


def test_compaction_calls_on_interleaved_cache():
    w = inputs.make_workload("strided-c", 32, 4, 33, [0, 7, 128, 500], match_prob=0.9)
    dw = DeviceWorkload(w)
    path, alen, _, _ = oracle.tree_accept(w.node_tokens, w.target_tokens, w.next_token,
                                          w.next_sibling)
    c_ref, k_ref, p_ref, s_ref = oracle.kv_compact(w.c_kv, w.k_rope, w.prefix_lens, path, alen)
    assert (alen > 1).any()
    cap = w.capacity

    buf, ckv, kr = _combined(w)
    newp, st = ddt.kv_compact(ckv, kr, dw.prefix, i32(path), i32(alen))
    torch.cuda.synchronize()
    assert np.array_equal(_u16(ckv)[:, :cap], c_ref) and np.array_equal(_u16(kr)[:, :cap], k_ref)
    assert (_u16(buf)[:, cap:] == 0x7FC0).all()
    assert np.array_equal(newp.cpu().numpy(), p_ref) and np.array_equal(st.cpu().numpy(), s_ref)

    buf, ckv, kr = _combined(w)
    outs = ddt.accept_compact(dw.node_tokens, dw.target_tokens, dw.next_token, dw.next_sibling,
                              ckv, kr, dw.prefix)
    torch.cuda.synchronize()
    assert np.array_equal(outs[0].cpu().numpy(), path)
    assert np.array_equal(_u16(ckv)[:, :cap], c_ref) and np.array_equal(_u16(kr)[:, :cap], k_ref)
    assert np.array_equal(outs[4].cpu().numpy(), p_ref)


def test_block_write_on_interleaved_cache():
    w = inputs.make_workload("strided-w", 33, 3, 9, [0, 20, 77])
    buf, ckv, kr = _combined(w)
    rng = np.random.RandomState(3)
    blk_l = rng.randint(0, 65535, size=(3, 9, 512)).astype(np.uint16)
    blk_r = rng.randint(0, 65535, size=(3, 9, 64)).astype(np.uint16)
    st = ddt.kv_write_block(ckv, kr, i32(w.prefix_lens), bf16_tensor(blk_l), bf16_tensor(blk_r))
    torch.cuda.synchronize()
    want_l, want_r = w.c_kv.copy(), w.k_rope.copy()
    for b in range(3):
        P = int(w.prefix_lens[b])
        want_l[b, P:P + 9] = blk_l[b]
        want_r[b, P:P + 9] = blk_r[b]
    cap = w.capacity
    assert np.array_equal(_u16(ckv)[:, :cap], want_l) and np.array_equal(_u16(kr)[:, :cap], want_r)
    assert (st.cpu().numpy() == 0).all()
