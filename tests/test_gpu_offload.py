"""GPU tests of the asynchronous offload engine (incremental block prefetch).

The AR(1) query stream of the 96k GQA workload runs step by step with the
full KV in pinned host memory and a 2*K_b-slot block cache on the GPU:
  step t, compute stream: block top-K_b from q_t -> S(t); event
  step t, copy stream:    wait; tls_prefetch_diff(S(t-1) -> S(t)); event
  step t, compute stream: token top-K_t from q_t inside S(t-1); wait for the
                          copy of step t-1; paged attention over the cache.
Checked against the oracle's stream (same reading: attention at t uses the
blocks selected at t-1) at every step, plus the slot table, the cache
contents and the number of blocks copied.  Also: the bounded host wait.
"""
import numpy as np
import pytest
import torch

from two_level_sparse_quest_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from two_level_sparse_quest_b200 import build

    build.build()


def run_stream(w: W.Workload, check_cache_every: int = 16):
    from oracle import oracle as O
    from tests import _parity as P
    from two_level_sparse_quest_b200 import tls as T

    inp = W.make_decode_inputs(w)
    qs = W.make_query_stream(w)
    steps = qs.shape[0]
    s = T.shape_from_workload(w)
    B, H, nb, bs, d = w.batch, w.n_kv_heads, w.n_blocks, w.block_size, w.d_qk
    n_slots = 2 * w.k_b
    # resident on the GPU: block summary and label slab (built once from K)
    K = P.to_dev(inp.K)
    sl, lab = P.to_dev(inp.seq_lens), P.to_dev(inp.label_idx)
    meta = torch.zeros((B, H, nb, 2, d), dtype=torch.int16, device="cuda")
    slab = torch.zeros((B, H, w.ctx, w.n_label), dtype=torch.int16, device="cuda")
    T.tls_build_block_meta(s, K, sl, lab, meta, slab)
    torch.cuda.synchronize()
    del K
    # offloaded: the full KV, block-major, in pinned host memory
    host_np = W.paged_host_kv(inp)
    host_kv = torch.from_numpy(host_np.view(np.int16)).pin_memory()
    cache = torch.zeros((B, H, n_slots, 2, bs, d), dtype=torch.int16, device="cuda")
    sob = torch.empty((B, H, nb), dtype=torch.int32, device="cuda")
    bos = torch.empty((B, H, n_slots), dtype=torch.int32, device="cuda")
    jobs = torch.empty((B, H, w.k_b, 2), dtype=torch.int32, device="cuda")
    n_new = torch.empty((B, H), dtype=torch.int32, device="cuda")
    ws = torch.zeros(T.tls_workspace_size(s), dtype=torch.uint8, device="cuda")
    T.tls_offload_reset(s, n_slots, sob, bos)
    ring = [torch.empty((B, H, w.k_b), dtype=torch.int32, device="cuda") for _ in range(3)]
    tidx = torch.empty((B, H, w.k_t), dtype=torch.int32, device="cuda")
    out = torch.empty((B, w.n_q_heads, w.d_v), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, w.n_q_heads), dtype=torch.float32, device="cuda")
    compute = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    q_dev = [P.to_dev(qs[t]) for t in range(steps)]

    os_ = O.shape_of(w)
    meta_o = O.build_meta(os_, inp.K, inp.seq_lens)
    ref = O.stream_decode(os_, qs, inp.K, inp.V, meta_o, inp.seq_lens, inp.label_idx)

    block_bytes = 2 * bs * d * 2
    resident_prev = [set() for _ in range(B * H)]
    total_new = 0
    ev_copy_prev = None
    for t in range(steps):
        cur, prev = ring[t % 3], (ring[(t - 1) % 3] if t else None)
        T.tls_block_score_topk(s, q_dev[t], meta, sl, cur, None, ws)
        ev_sel = torch.cuda.Event()
        ev_sel.record(compute)
        copy.wait_event(ev_sel)
        T.tls_prefetch_diff(s, n_slots, host_kv, cache, sob, bos, prev, cur, n_new, jobs, stream=copy)
        ev_copy = torch.cuda.Event()
        ev_copy.record(copy)
        attend_blocks = cur if t == 0 else prev
        T.tls_token_score_topk(s, q_dev[t], slab, lab, attend_blocks, sl, tidx, None, ws)
        compute.wait_event(ev_copy if t == 0 else ev_copy_prev)
        T.tls_sparse_attn_decode_paged(s, q_dev[t], cache, sob, n_slots, tidx, out, lse, ws)
        torch.cuda.synchronize()
        ev_copy_prev = ev_copy
        gb = cur.cpu().numpy()
        gt = tidx.cpu().numpy()
        # selections equal the oracle stream (no boundary swaps expected on these inputs)
        np.testing.assert_array_equal(gb, ref["block_idx"][t], err_msg=f"step {t} blocks")
        np.testing.assert_array_equal(gt, ref["token_idx"][t], err_msg=f"step {t} tokens")
        P.check_attention(out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                          ref["out"][t], ref["lse"][t], f"step {t} attention")
        # blocks copied = blocks of S(t) that were not resident (resident = S(t-2) u S(t-1))
        nn = n_new.cpu().numpy()
        for gi in range(B * H):
            b, g = divmod(gi, H)
            nxt = set(gb[b, g][gb[b, g] >= 0].tolist())
            want_new = len(nxt - resident_prev[gi])
            assert nn[b, g] == want_new, f"step {t} group {gi}: copied {nn[b, g]}, expected {want_new}"
            prev_sel = (set(ref["block_idx"][t - 1][b, g].tolist()) - {-1}) if t else set()
            keep = nxt | prev_sel
            resident_prev[gi] = keep
        total_new += int(nn.sum())
        if t % check_cache_every == 0 or t == steps - 1:
            so, bo, cc = sob.cpu().numpy(), bos.cpu().numpy(), cache.cpu().numpy()
            for gi in range(B * H):
                b, g = divmod(gi, H)
                res_blocks = np.nonzero(so[b, g] >= 0)[0]
                assert set(res_blocks.tolist()) == resident_prev[gi], f"step {t}: resident set"
                for blk in res_blocks:
                    slot = so[b, g, blk]
                    assert bo[b, g, slot] == blk
                    np.testing.assert_array_equal(cc[b, g, slot], host_np[b, g, blk].view(np.int16))
                assert (bo[b, g] >= 0).sum() == len(res_blocks)
    first = int(ref["n_new"][0].sum())
    return {"steps": steps, "blocks_copied": total_new, "bytes_copied": total_new * block_bytes,
            "first_step_blocks": first,
            "oracle_diff_blocks": int(sum(int(n.sum()) for n in ref["n_new"][1:])),
            "mean_overlap": float(np.mean([1 - n.sum() / (B * H * w.k_b) for n in ref["n_new"][1:]]))}


def test_stream_small():
    w = W.WORKLOADS["stream96k_bf16"].with_(ctx=8192, k_b=32, k_t=512, steps=12)
    res = run_stream(w, check_cache_every=1)
    assert res["blocks_copied"] <= res["first_step_blocks"] + res["oracle_diff_blocks"]


def test_stream_full_size():
    from tests import _parity as P

    res = run_stream(W.WORKLOADS["stream96k_bf16"])
    P.report("stream96k_bf16", **res)
    assert res["blocks_copied"] < res["steps"] * 8 * 192  # incremental: far below a full reload per step


def test_bounded_wait_times_out_and_recovers():
    from two_level_sparse_quest_b200 import tls as T

    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        torch.cuda._sleep(int(1.5e9))  # a bounded device spin (~1 s), ends by itself
    ev = torch.cuda.Event()
    ev.record(side)
    assert T.tls_wait_event(ev, 5) == T.TLS_ERR_TIMEOUT
    assert "not complete" in T.tls_last_error()
    assert T.tls_wait_event(ev, 30000) == T.TLS_OK
    torch.cuda.synchronize()
