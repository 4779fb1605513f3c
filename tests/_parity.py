"""Shared helpers of the GPU parity tests: run the CUDA stages through the C ABI,
run the oracle on the same seeded inputs, and compare with the rules below.

Comparison rules:
  * block summary and label slab: bit-exact (they are min / max / copies of
    stored values);
  * index sets (blocks, tokens): bit-exact, except swaps at the K-th boundary
    whose two oracle fp64 scores differ by less than 1e-4 relative; swaps are
    counted and reported;
  * fp32 scores: within a bound derived from fp32 rounding of the kernel's
    summation (block_score_bound, token_score_bound);
  * attention output and lse: |gpu - oracle| <= 2e-3 + 2e-3 |oracle|.
Inputs flow oracle -> GPU only (the oracle's selections may be fed to the next
GPU stage to test it alone); no oracle input comes from the GPU.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from oracle import oracle as O
from two_level_sparse_quest_b200 import workloads as W

U32 = 2.0 ** -24  # unit roundoff of fp32
ATOL = 2e-3
RTOL = 2e-3
SWAP_RTOL = 1e-4

REPORT = os.environ.get("TLS_PARITY_REPORT")

# Every parity case's swap counts, printed at the end of the pytest session
# (tests/conftest.py) so that they appear in the run's output.
RESULTS: list = []


def report(name: str, **kv):
    RESULTS.append({"case": name, **kv})
    if not REPORT:
        return
    os.makedirs(os.path.dirname(REPORT) or ".", exist_ok=True)
    with open(REPORT, "a") as f:
        f.write(json.dumps({"case": name, **kv}) + "\n")


def tls():
    from two_level_sparse_quest_b200 import tls as T

    return T


def to_dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def from_dev_elems(t: torch.Tensor, dtype: int) -> np.ndarray:
    a = t.cpu().numpy()
    return W.to_f64(a.view(np.uint16) if dtype == W.BF16 else a, dtype)


class GpuInputs:
    """Device copies of one decode step's inputs, plus the built summary and slab."""

    def __init__(self, w: W.Workload, inp: W.DecodeInputs, out_dtype=0):
        T = tls()
        self.w, self.inp = w, inp
        self.shape = T.shape_from_workload(w, out_dtype=out_dtype)
        self.q = to_dev(inp.q)
        self.K = to_dev(inp.K)
        self.V = to_dev(inp.V) if inp.V is not None else None
        self.seq_lens = to_dev(inp.seq_lens)
        self.label = to_dev(inp.label_idx)
        edt = torch.int16 if w.dtype == W.BF16 else torch.float32
        B, H, nb, d = w.batch, w.n_kv_heads, w.n_blocks, w.d_qk
        self.meta = torch.zeros((B, H, nb, 2, d), dtype=edt, device="cuda")
        if getattr(w, "slab_bits", 0) == 8:  # int8 codes + fp32 scales in one buffer
            self.slab = torch.zeros(T.tls_slab_bytes(self.shape), dtype=torch.uint8, device="cuda")
        else:
            self.slab = torch.zeros((B, H, w.ctx, w.n_label), dtype=edt, device="cuda")
        T.tls_build_block_meta(self.shape, self.K, self.seq_lens, self.label, self.meta, self.slab)
        self.ws = torch.zeros(T.tls_workspace_size(self.shape), dtype=torch.uint8, device="cuda")

    def block_stage(self, with_scores=True):
        T, w = tls(), self.w
        bidx = torch.full((w.batch, w.n_kv_heads, w.k_b), -7, dtype=torch.int32, device="cuda")
        sc = torch.zeros((w.batch, w.n_kv_heads, w.n_blocks), dtype=torch.float32, device="cuda") if with_scores else None
        T.tls_block_score_topk(self.shape, self.q, self.meta, self.seq_lens, bidx, sc, self.ws)
        return bidx, sc

    def token_stage(self, block_idx: torch.Tensor, with_scores=True):
        T, w = tls(), self.w
        tidx = torch.full((w.batch, w.n_kv_heads, w.k_t), -7, dtype=torch.int32, device="cuda")
        C = w.k_b * w.block_size
        sc = torch.zeros((w.batch, w.n_kv_heads, C), dtype=torch.float32, device="cuda") if with_scores else None
        T.tls_token_score_topk(self.shape, self.q, self.slab, self.label, block_idx, self.seq_lens, tidx, sc, self.ws)
        return tidx, sc

    def attention(self, token_idx: torch.Tensor):
        T, w = tls(), self.w
        odt = torch.int16 if self.shape.out_dtype == W.BF16 else torch.float32
        out = torch.zeros((w.batch, w.n_q_heads, w.d_v), dtype=odt, device="cuda")
        lse = torch.zeros((w.batch, w.n_q_heads), dtype=torch.float32, device="cuda")
        T.tls_sparse_attn_decode(self.shape, self.q, self.K, self.V, token_idx, out, lse, self.ws)
        return out, lse

    def out_f64(self, out: torch.Tensor) -> np.ndarray:
        return from_dev_elems(out, self.shape.out_dtype)


class OracleRun:
    """The oracle's own chain on the same inputs."""

    def __init__(self, w: W.Workload, inp: W.DecodeInputs):
        s = O.shape_of(w)
        self.s = s
        self.meta = O.build_meta(s, inp.K, inp.seq_lens)
        self.block_scores = O.block_scores(s, inp.q, self.meta, inp.seq_lens)
        self.block_idx = O.select_blocks(s, self.block_scores, inp.seq_lens)
        self.cand_scores, self.cand_tok = O.token_scores(s, inp.q, inp.K, inp.label_idx, self.block_idx, inp.seq_lens)
        self.token_idx = O.select_tokens(s, self.cand_scores, self.cand_tok)
        self.out, self.lse = O.attention(s, inp.q, inp.K, inp.V, self.token_idx)


# ---------------------------------------------------------------- comparisons
def check_meta(w, inp, gpu: GpuInputs, orc: OracleRun):
    gm = from_dev_elems(gpu.meta, w.dtype)
    for b in range(w.batch):
        nb = -(-int(inp.seq_lens[b]) // w.block_size)
        np.testing.assert_array_equal(gm[b, :, :nb], orc.meta[b, :, :nb])
    if getattr(w, "slab_bits", 0) == 8:
        check_slab_q8(w, inp, gpu)
        return
    # the slab is a copy of stored values: compare the stored bits
    gs = gpu.slab.cpu().numpy()
    gs = gs.view(np.uint16) if w.dtype == W.BF16 else gs.view(np.uint32)
    Kr = inp.K.view(np.uint16) if w.dtype == W.BF16 else inp.K.view(np.uint32)
    for b in range(w.batch):
        L = int(inp.seq_lens[b])
        np.testing.assert_array_equal(gs[b, :, :L], Kr[b, :, :L][..., inp.label_idx])


def slab_q8_views(w, slab: np.ndarray):
    """(codes [B][H][ctx][r] int8, scales [B][H][r] fp32) of an int8 slab buffer:
    the codes, then the scales at the next multiple of 256 bytes."""
    n = w.batch * w.n_kv_heads * w.ctx * w.n_label
    off = -(-n // 256) * 256
    codes = slab[:n].view(np.int8).reshape(w.batch, w.n_kv_heads, w.ctx, w.n_label)
    scales = slab[off:off + 4 * w.batch * w.n_kv_heads * w.n_label].view(np.float32)
    return codes, scales.reshape(w.batch, w.n_kv_heads, w.n_label)


def check_slab_q8(w, inp, gpu: GpuInputs):
    """Codes and scales are integers / fp32 values decided in fp32 on both
    sides: bit-exact on the valid rows."""
    codes, scales = slab_q8_views(w, gpu.slab.cpu().numpy())
    oc, osc = O.quantize_labels(O.shape_of(w), inp.K, inp.seq_lens, inp.label_idx)
    np.testing.assert_array_equal(scales.view(np.uint32), osc.view(np.uint32))
    for b in range(w.batch):
        L = int(inp.seq_lens[b])
        np.testing.assert_array_equal(codes[b, :, :L], oc[b, :, :L])


def block_score_bound(w, inp, orc: OracleRun) -> np.ndarray:
    """fp32 rounding bound of the kernel's block score: the head sum folded into
    Q+/Q- (G terms) and a 2d-term dot, each term bounded by |q| max(|M|,|m|)."""
    q = W.to_f64(inp.q, w.dtype).reshape(w.batch, w.n_kv_heads, w.group, w.d_qk)
    A = np.abs(q).sum(axis=2)  # [B][H][d]
    mag = np.maximum(np.abs(orc.meta[:, :, :, 0]), np.abs(orc.meta[:, :, :, 1]))  # [B][H][nb][d]
    mag = np.nan_to_num(mag)
    return 2.0 * (2 * w.d_qk + w.group + 2) * U32 * np.einsum("bhd,bhnd->bhn", A, mag)


def token_score_bound(w, inp, orc: OracleRun, block_idx: np.ndarray) -> np.ndarray:
    """fp32 rounding bound of the kernel's token score: Qbar_L = sum of G heads,
    then an r-term dot; each term bounded by |q_{h,c}| |K[t,c]| (int8 slab:
    |q_{h,c}| |scale_c code|, one more rounding for the folded scale)."""
    q8 = O.quantize_labels(O.shape_of(w), inp.K, inp.seq_lens, inp.label_idx) if getattr(w, "slab_bits", 0) == 8 else None
    q = W.to_f64(inp.q, w.dtype).reshape(w.batch, w.n_kv_heads, w.group, w.d_qk)[..., inp.label_idx]
    C = w.k_b * w.block_size
    out = np.zeros((w.batch, w.n_kv_heads, C))
    j = np.arange(C)
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            blk = block_idx[b, g][j // w.block_size]
            t = blk * w.block_size + j % w.block_size
            ok = (blk >= 0) & (t < inp.seq_lens[b])
            if q8 is not None:  # |scale_c * code| in place of |K[t, L_c]|
                kk = np.abs(q8[0][b, g][np.where(ok, t, 0)].astype(np.float64) * q8[1][b, g].astype(np.float64))
            else:
                rows = inp.K[b, g][np.where(ok, t, 0)][:, inp.label_idx]
                kk = np.abs(W.to_f64(rows, w.dtype))
            out[b, g] = np.where(ok, kk @ np.abs(q[b, g]).sum(axis=0), 0.0)
    return 2.0 * (w.n_label + w.group + 2 + (q8 is not None)) * U32 * out


def check_scores(gpu_scores: np.ndarray, ora_scores: np.ndarray, bound: np.ndarray, what: str):
    g = gpu_scores.astype(np.float64)
    o = ora_scores
    inval = np.isneginf(o)
    assert (np.isneginf(g) == inval).all(), f"{what}: invalid-entry pattern differs"
    err = np.abs(g[~inval] - o[~inval])
    lim = bound[~inval] + 1e-30
    bad = err > lim
    assert not bad.any(), f"{what}: {bad.sum()} scores outside the fp32 bound; worst {err.max():.3e}"


def check_selection(gpu_ids: np.ndarray, ids: np.ndarray, scores: np.ndarray, k: int, what: str) -> int:
    """gpu_ids: kernel output (ascending, -1 padded).  ids/scores: the oracle's
    candidate ids and fp64 scores.  Returns the number of boundary swaps."""
    sel = gpu_ids[gpu_ids >= 0]
    m = min(k, len(ids))
    assert len(sel) == m, f"{what}: {len(sel)} selected, expected {m}"
    assert (gpu_ids[m:] == -1).all(), f"{what}: padding"
    assert (np.diff(sel) > 0).all(), f"{what}: not strictly ascending"
    want, _ = O.topk(scores, k, ids=ids, out_cap=k)
    want = want[want >= 0]
    A, B = set(sel.tolist()), set(want.tolist())
    if A == B:
        return 0
    sc = dict(zip(ids.tolist(), scores.tolist()))
    assert A <= set(sc), f"{what}: selected ids that are not candidates"
    s_in = [sc[x] for x in A - B]     # selected by the GPU only
    s_out = [sc[y] for y in B - A]    # selected by the oracle only
    hi, lo = max(s_out), min(s_in)
    assert hi - lo <= SWAP_RTOL * max(abs(hi), abs(lo)), f"{what}: swap beyond 1e-4 relative ({hi} vs {lo})"
    return len(A - B)


def check_selection_self_consistent(gpu_ids: np.ndarray, cand_ids: np.ndarray, gpu_scores: np.ndarray, what: str):
    """Property of a correct top-k on the kernel's own fp32 scores: every kept
    score >= every dropped score, and among equal scores at the boundary the
    kept ids are the lower ones."""
    sel = set(gpu_ids[gpu_ids >= 0].tolist())
    if not sel:
        return
    keep = np.array([c in sel for c in cand_ids.tolist()])
    s = gpu_scores.astype(np.float32)
    if keep.all() or not keep.any():
        return
    kmin = s[keep].min()
    dmax = s[~keep].max()
    assert kmin >= dmax, f"{what}: kept score {kmin} < dropped score {dmax}"
    if kmin == dmax:
        kept_eq = cand_ids[keep & (s == kmin)]
        drop_eq = cand_ids[~keep & (s == kmin)]
        assert kept_eq.max() < drop_eq.min(), f"{what}: tie not broken toward the lower id"


def check_attention(gout: np.ndarray, glse: np.ndarray, oout: np.ndarray, olse: np.ndarray, what: str):
    err = np.abs(gout - oout)
    lim = ATOL + RTOL * np.abs(oout)
    assert (err <= lim).all(), f"{what}: out error {err.max():.3e} ({(err > lim).sum()} elements)"
    inf = np.isneginf(olse)
    assert (np.isneginf(glse) == inf).all(), f"{what}: lse -inf pattern"
    e2 = np.abs(glse[~inf] - olse[~inf])
    assert (e2 <= ATOL + RTOL * np.abs(olse[~inf])).all(), f"{what}: lse error {e2.max() if e2.size else 0:.3e}"
    return float(err.max()) if err.size else 0.0


def full_stage_parity(w: W.Workload, seq_lens=None, out_dtype=0, name=None, inp=None):
    """Every stage against the oracle on one seeded input (or the given one);
    returns a summary dict."""
    name = name or w.name
    if inp is None:
        inp = W.make_decode_inputs(w, seq_lens=seq_lens)
    orc = OracleRun(w, inp)
    gpu = GpuInputs(w, inp, out_dtype=out_dtype)
    check_meta(w, inp, gpu, orc)
    # stage 1+2
    bidx, bsc = gpu.block_stage()
    torch.cuda.synchronize()
    bidx, bsc = bidx.cpu().numpy(), bsc.cpu().numpy()
    check_scores(bsc, orc.block_scores, block_score_bound(w, inp, orc), f"{name} block scores")
    swaps_b = 0
    for b in range(w.batch):
        nb = -(-int(inp.seq_lens[b]) // w.block_size)
        ids = np.arange(nb, dtype=np.int32)
        for g in range(w.n_kv_heads):
            swaps_b += check_selection(bidx[b, g], ids, orc.block_scores[b, g, :nb], w.k_b, f"{name} blocks b{b} g{g}")
            check_selection_self_consistent(bidx[b, g], ids, bsc[b, g, :nb], f"{name} blocks b{b} g{g}")
    # stage 3+4 on the oracle's block selection
    tidx, tsc = gpu.token_stage(to_dev(orc.block_idx))
    torch.cuda.synchronize()
    tidx, tsc = tidx.cpu().numpy(), tsc.cpu().numpy()
    check_scores(tsc, orc.cand_scores, token_score_bound(w, inp, orc, orc.block_idx), f"{name} token scores")
    swaps_t = 0
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            ok = orc.cand_tok[b, g] >= 0
            ids = orc.cand_tok[b, g][ok]
            swaps_t += check_selection(tidx[b, g], ids, orc.cand_scores[b, g][ok], w.k_t, f"{name} tokens b{b} g{g}")
            check_selection_self_consistent(tidx[b, g], ids, tsc[b, g][ok], f"{name} tokens b{b} g{g}")
    # stage 5 on the oracle's token selection
    out, lse = gpu.attention(to_dev(orc.token_idx))
    torch.cuda.synchronize()
    err = check_attention(gpu.out_f64(out), lse.cpu().numpy().astype(np.float64), orc.out, orc.lse, f"{name} attention")
    # stages 1-4 in one launch (tls_select_step, the call the benchmark times)
    # against the oracle: block ids directly; token ids wherever the launch's
    # own block selection equals the oracle's (elsewhere the candidates differ
    # by a counted block swap and only the self-consistency of the kernel's
    # token ranking on its own fp32 scores is checked)
    fb = torch.full((w.batch, w.n_kv_heads, w.k_b), -7, dtype=torch.int32, device="cuda")
    ft = torch.full((w.batch, w.n_kv_heads, w.k_t), -7, dtype=torch.int32, device="cuda")
    fbs = torch.zeros((w.batch, w.n_kv_heads, w.n_blocks), dtype=torch.float32, device="cuda")
    fts = torch.zeros((w.batch, w.n_kv_heads, w.k_b * w.block_size), dtype=torch.float32, device="cuda")
    tls().tls_select_step(gpu.shape, gpu.q, gpu.meta, gpu.slab, gpu.label, gpu.seq_lens, fb, ft, fbs, fts)
    torch.cuda.synchronize()
    fb, ft, fbs, fts = fb.cpu().numpy(), ft.cpu().numpy(), fbs.cpu().numpy(), fts.cpu().numpy()
    check_scores(fbs, orc.block_scores, block_score_bound(w, inp, orc), f"{name} select_step block scores")
    step_swaps_b = step_swaps_t = 0
    C = w.k_b * w.block_size
    for b in range(w.batch):
        nb = -(-int(inp.seq_lens[b]) // w.block_size)
        ids = np.arange(nb, dtype=np.int32)
        for g in range(w.n_kv_heads):
            what = f"{name} select_step b{b} g{g}"
            step_swaps_b += check_selection(fb[b, g], ids, orc.block_scores[b, g, :nb], w.k_b, what + " blocks")
            j = np.arange(C)
            blk = fb[b, g][j // w.block_size]
            cand = np.where(blk >= 0, blk * w.block_size + j % w.block_size, -1)
            ok = (cand >= 0) & (cand < inp.seq_lens[b])
            if (fb[b, g] == orc.block_idx[b, g]).all():
                oko = orc.cand_tok[b, g] >= 0
                step_swaps_t += check_selection(ft[b, g], orc.cand_tok[b, g][oko], orc.cand_scores[b, g][oko], w.k_t,
                                                what + " tokens")
            check_selection_self_consistent(ft[b, g], cand[ok].astype(np.int32), fts[b, g][ok], what + " tokens")
    # the same selection with tls_decode_step's workspace (its launches: the
    # two-phase path may fold the queries once and select the blocks per CTA):
    # the same bits
    wb = torch.full_like(torch.from_numpy(fb), -7).cuda()
    wt = torch.full_like(torch.from_numpy(ft), -7).cuda()
    wbs = torch.zeros(fbs.shape, dtype=torch.float32, device="cuda")
    wts = torch.zeros(fts.shape, dtype=torch.float32, device="cuda")
    tls().tls_select_step_ws(gpu.shape, gpu.q, gpu.meta, gpu.slab, gpu.label, gpu.seq_lens, wb, wt, gpu.ws, wbs, wts)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(wb.cpu().numpy(), fb, err_msg=f"{name} select_step_ws block ids")
    np.testing.assert_array_equal(wt.cpu().numpy(), ft, err_msg=f"{name} select_step_ws token ids")
    np.testing.assert_array_equal(wbs.cpu().numpy().view(np.uint32), fbs.view(np.uint32),
                                  err_msg=f"{name} select_step_ws block scores")
    np.testing.assert_array_equal(wts.cpu().numpy().view(np.uint32), fts.view(np.uint32),
                                  err_msg=f"{name} select_step_ws token scores")
    # stages 1-5 in one call (tls_decode_step, the call the benchmark times):
    # block / token ids and both score arrays identical to the select_step
    # launch above, attention against the oracle wherever the token ids equal
    # the oracle's.  Called twice on one workspace, with and without the
    # optional score outputs.
    step_groups = 0
    for call in range(2):
        db = torch.full((w.batch, w.n_kv_heads, w.k_b), -7, dtype=torch.int32, device="cuda")
        dt = torch.full((w.batch, w.n_kv_heads, w.k_t), -7, dtype=torch.int32, device="cuda")
        dbs = torch.zeros((w.batch, w.n_kv_heads, w.n_blocks), dtype=torch.float32, device="cuda")
        dts = torch.zeros((w.batch, w.n_kv_heads, w.k_b * w.block_size), dtype=torch.float32, device="cuda")
        odt = torch.int16 if gpu.shape.out_dtype == W.BF16 else torch.float32
        dout = torch.zeros((w.batch, w.n_q_heads, w.d_v), dtype=odt, device="cuda")
        dlse = torch.zeros((w.batch, w.n_q_heads), dtype=torch.float32, device="cuda")
        with_scores = call == 0
        tls().tls_decode_step(gpu.shape, gpu.q, gpu.meta, gpu.slab, gpu.label, gpu.seq_lens, gpu.K, gpu.V, db, dt,
                              dout, dlse, dbs if with_scores else None, dts if with_scores else None, gpu.ws)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(db.cpu().numpy(), fb, err_msg=f"{name} decode_step block ids, call {call}")
        np.testing.assert_array_equal(dt.cpu().numpy(), ft, err_msg=f"{name} decode_step token ids, call {call}")
        if with_scores:
            np.testing.assert_array_equal(dbs.cpu().numpy().view(np.uint32), fbs.view(np.uint32),
                                          err_msg=f"{name} decode_step block scores")
            np.testing.assert_array_equal(dts.cpu().numpy().view(np.uint32), fts.view(np.uint32),
                                          err_msg=f"{name} decode_step token scores")
        dout, dlse = gpu.out_f64(dout), dlse.cpu().numpy().astype(np.float64)
        G = w.group
        step_groups = 0
        for b in range(w.batch):
            for g in range(w.n_kv_heads):
                if (ft[b, g] == orc.token_idx[b, g]).all():
                    step_groups += 1
                    hs = slice(g * G, (g + 1) * G)
                    check_attention(dout[b, hs], dlse[b, hs], orc.out[b, hs], orc.lse[b, hs],
                                    f"{name} decode_step attention b{b} g{g} call {call}")
    # chained: the GPU's own selections all the way
    cb, _ = gpu.block_stage(with_scores=False)
    ct, _ = gpu.token_stage(cb, with_scores=False)
    cout, clse = gpu.attention(ct)
    torch.cuda.synchronize()
    cb, ct = cb.cpu().numpy(), ct.cpu().numpy()
    cout, clse = gpu.out_f64(cout), clse.cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(cb, bidx)  # deterministic
    same_groups = 0
    G = w.group
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            if (cb[b, g] == orc.block_idx[b, g]).all():
                np.testing.assert_array_equal(ct[b, g], tidx[b, g])
            if (ct[b, g] == orc.token_idx[b, g]).all():
                same_groups += 1
                hs = slice(g * G, (g + 1) * G)
                check_attention(cout[b, hs], clse[b, hs], orc.out[b, hs], orc.lse[b, hs], f"{name} chained b{b} g{g}")
    assert tls().tls_device_error(clear=True) == 0, f"{name}: a kernel's bounded wait gave up"
    res = dict(block_swaps=swaps_b, token_swaps=swaps_t, step_block_swaps=step_swaps_b,
               step_token_swaps=step_swaps_t, decode_step_groups_vs_oracle=step_groups, attn_max_abs_err=err,
               chained_groups_identical=same_groups, groups=w.batch * w.n_kv_heads)
    report(name, **res)
    return res
