"""ddt_decode_step: tree build -> tree-block write -> verify -> accept + compaction,
chained on the device over several steps, eagerly and replayed from a CUDA graph,
against the same chain run by the oracle (needs a B200).

Sources: "Race Conditions, Buffer Aliasing, and the Architecture of a Native
DDTree Inference Engine" ("The Mission: A Native DDTree Engine", "The Cache
Compaction Problem") and "The Microsecond Verdict: Validating a DDTree Kernel Fix
Under Time Pressure" ("What Was Learned": the tree builder's output chained into
the accept walk)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import MAX_ABS, REL_L2, bf16_tensor, compare_attention, i32, out_format
from tree_speculative_decoding_05_b200 import ddt, inputs

pytestmark = pytest.mark.gpu

H, DL, DR = 64, 512, 64


def _continuation(seed, draft, Q):
    """The target's greedy token after the accepted path of each depth: the drafter's
    top token with probability 0.6, its second with 0.2, else a token it did not
    propose (so accepted lengths vary)."""
    B, D, K = draft.tok.shape
    u = inputs.uniform(inputs.stream_base(seed, 95, 0), 0, B * Q).reshape(B, Q)
    cont = np.full((B, Q), 31999, dtype=np.int32)
    for b in range(B):
        for d in range(Q):
            if d < D and u[b, d] < 0.6:
                cont[b, d] = draft.tok[b, d, 0]
            elif d < D and u[b, d] < 0.8 and K > 1:
                cont[b, d] = draft.tok[b, d, 1]
    return cont


def _steps(seed, B, Q, D, K, n):
    out = []
    for s in range(n):
        sd = seed * 100 + s
        draft = inputs.draft_batch(sd, B, D, K)
        mk = lambda tag, shape: inputs.to_bf16_bits(
            inputs.normal(inputs.stream_base(sd, tag, 0), int(np.prod(shape)))).reshape(shape)
        out.append(dict(draft=draft, q_lat=mk(1, (B, Q, H, DL)), q_rope=mk(2, (B, Q, H, DR)),
                        block_ckv=mk(3, (B, Q, DL)), block_krope=mk(4, (B, Q, DR)),
                        cont=_continuation(sd, draft, Q)))
    return out


def _oracle_chain(steps, c_kv, k_rope, P, root, Q, scale):
    c_kv, k_rope, P, root = c_kv.copy(), k_rope.copy(), P.copy(), root.copy()
    B, cap = c_kv.shape[0], c_kv.shape[1]
    res = []
    for st in steps:
        t = oracle.tree_build(st["draft"].lp, st["draft"].tok, root, Q)
        for b in range(B):
            c_kv[b, P[b]:P[b] + Q] = st["block_ckv"][b]
            k_rope[b, P[b]:P[b] + Q] = st["block_krope"][b]
        tgt = np.take_along_axis(st["cont"], t["depth"], axis=1).astype(np.int32)
        out, lse = oracle.attn_all(st["q_lat"], st["q_rope"], c_kv, k_rope, P, t["parents"], scale)
        path, alen, bonus, ast = oracle.tree_accept(t["node_tokens"], tgt, t["next_token"],
                                                    t["next_sibling"])
        c_kv, k_rope, newp, cst = oracle.kv_compact(c_kv, k_rope, P, path, alen, capacity=cap)
        res.append(dict(tree=t, out=out, path=path, alen=alen, bonus=bonus))
        P, root = newp, bonus
    return res, c_kv, k_rope, P, root


class Chain:
    """Device state, per-step inputs and per-step output buffers of a decode loop."""

    def __init__(self, steps, c_kv, k_rope, P, root, Q, scale, max_prefix):
        dev = torch.device("cuda")
        B = c_kv.shape[0]
        self.state = dict(c_kv=bf16_tensor(c_kv), k_rope=bf16_tensor(k_rope), prefix_lens=i32(P),
                          root_token=i32(root))
        self.init = {k: v.clone() for k, v in self.state.items()}
        self.args, self.bufs = [], []
        W = (Q + 63) // 64
        for st in steps:
            step = dict(lp=torch.from_numpy(st["draft"].lp).to(dev),
                        tok=torch.from_numpy(st["draft"].tok).to(dev),
                        q_lat=bf16_tensor(st["q_lat"]), q_rope=bf16_tensor(st["q_rope"]),
                        block_ckv=bf16_tensor(st["block_ckv"]),
                        block_krope=bf16_tensor(st["block_krope"]),
                        target_continuation=i32(st["cont"]))
            z = lambda *s: torch.zeros(s, dtype=torch.int32, device=dev)
            bufs = dict(mask=torch.zeros((B, Q, W), dtype=torch.int64, device=dev),
                        out=torch.zeros((B, Q, H, DL), dtype=torch.bfloat16, device=dev),
                        verify_status=z(B), parents=z(B, Q), node_tokens=z(B, Q), depth=z(B, Q),
                        next_token=z(B, Q), next_sibling=z(B, Q), n_nodes=z(B),
                        target_tokens=z(B, Q), path=z(B, Q), accept_len=z(B), status=z(4, B))
            a = ddt.decode_step_args(self.state, step, bufs, scale, max_prefix)
            ws, _ = ddt.verify_attn_workspace_size(step["q_lat"], step["q_rope"],
                                                   self.state["c_kv"], self.state["k_rope"],
                                                   self.state["prefix_lens"], bufs["mask"], scale,
                                                   max_prefix)
            if ws:
                bufs["workspace"] = torch.empty(ws, dtype=torch.uint8, device=dev)
                a = ddt.decode_step_args(self.state, step, bufs, scale, max_prefix)
            self.args.append((a, step))
            self.bufs.append(bufs)

    def reset(self):
        for k, v in self.init.items():
            self.state[k].copy_(v)

    def run(self):
        for a, _ in self.args:
            ddt.decode_step(a)


def _compare(chain, ref, c_ref, k_ref, P_ref, root_ref):
    torch.cuda.synchronize()
    for bufs, r in zip(chain.bufs, ref):
        t = r["tree"]
        for k in ("parents", "node_tokens", "depth", "next_token", "next_sibling", "n_nodes"):
            assert np.array_equal(bufs[k].cpu().numpy(), t[k]), k
        assert np.array_equal(bufs["mask"].cpu().numpy().view(np.uint64),
                              oracle.build_mask(t["parents"])[0])
        assert (bufs["status"].cpu().numpy() == 0).all()
        assert (bufs["verify_status"].cpu().numpy() == 0).all()
        compare_attention(bufs["out"].float().cpu().numpy().reshape(-1, DL),
                          r["out"].reshape(-1, DL), "decode-step attention",
                          fmt=out_format(bufs["out"]))
        assert np.array_equal(bufs["path"].cpu().numpy(), r["path"])
        assert np.array_equal(bufs["accept_len"].cpu().numpy(), r["alen"])
    s = chain.state
    assert np.array_equal(s["c_kv"].view(torch.int16).cpu().numpy().view(np.uint16), c_ref)
    assert np.array_equal(s["k_rope"].view(torch.int16).cpu().numpy().view(np.uint16), k_ref)
    assert np.array_equal(s["prefix_lens"].cpu().numpy(), P_ref)
    assert np.array_equal(s["root_token"].cpu().numpy(), root_ref)


@pytest.mark.parametrize("B,Q,D,K,n,P0", [(4, 17, 15, 4, 3, [100, 257, 600, 31]),
                                           (2, 33, 15, 8, 4, [100, 257]),
                                           (1, 17, 15, 8, 2, [2000])])
def test_decode_chain_eager_and_graph(B, Q, D, K, n, P0):
    """Few work items for 148 SMs, so every case's verify runs split-KV with the
    caller's workspace, inside the chain and inside the graph; the last case (one
    request, a 2000-row prefix) splits its keys six ways."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    steps = _steps(7 + Q, B, Q, D, K, n)
    P0 = np.array(P0, dtype=np.int32)
    cap = int(P0.max()) + (n + 1) * Q
    g = inputs.normal(inputs.stream_base(3, 96, 0), B * cap * (DL + DR))
    bits = inputs.to_bf16_bits(g).reshape(B, cap, DL + DR)
    c_kv, k_rope = np.ascontiguousarray(bits[:, :, :DL]), np.ascontiguousarray(bits[:, :, DL:])
    root = np.array([11, 22, 33, 44][:B], dtype=np.int32)
    scale = float(np.float32(1.0 / np.sqrt(192.0)))
    ref, c_ref, k_ref, P_ref, root_ref = _oracle_chain(steps, c_kv, k_rope, P0, root, Q, scale)
    assert any((r["alen"] > 1).any() for r in ref)

    chain = Chain(steps, c_kv, k_rope, P0, root, Q, scale, max_prefix=cap - Q)
    assert all("workspace" in b for b in chain.bufs)
    ddt.fault_flags(reset=True)
    chain.run()
    _compare(chain, ref, c_ref, k_ref, P_ref, root_ref)

    # The same loop captured once in a CUDA graph and replayed from the initial state.
    chain.reset()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            chain.run()
    torch.cuda.current_stream().wait_stream(stream)
    chain.reset()
    for bufs in chain.bufs:
        for v in bufs.values():
            if v is not None:
                v.zero_()
    graph.replay()
    _compare(chain, ref, c_ref, k_ref, P_ref, root_ref)
    assert ddt.fault_flags(reset=True) == 0
