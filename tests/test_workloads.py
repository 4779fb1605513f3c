"""Seeded workload generator: encoding, determinism, structure (CPU only)."""
import numpy as np
import torch

from two_level_sparse_quest_b200 import workloads as W


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-8, 8, 100000),
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1.0000001, 1.00390625, 1.01171875], np.float32)])
    ours = W.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = W.bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generation_is_deterministic_and_per_sequence():
    w = W.WORKLOADS["gqa48k_bf16"].with_(batch=2, ctx=256, k_b=4, k_t=32)
    a = W.make_decode_inputs(w)
    b = W.make_decode_inputs(w)
    np.testing.assert_array_equal(a.K, b.K)
    np.testing.assert_array_equal(a.q, b.q)
    only1 = W.make_decode_inputs(w, batches=[1])
    np.testing.assert_array_equal(only1.K[1], a.K[1])
    assert (only1.K[0] == 0).all()


def test_structure_outliers_needles_labels():
    w = W.WORKLOADS["gqa48k_bf16"].with_(ctx=2048)
    inp = W.make_decode_inputs(w)
    K = W.to_f64(inp.K[0], w.dtype)
    assert len(inp.outlier_idx) == 8 and len(inp.label_idx) == 16
    assert set(inp.outlier_idx.tolist()) <= set(inp.label_idx.tolist())
    assert (np.diff(inp.label_idx) > 0).all()
    std = K.reshape(-1, w.d_qk).std(axis=0)
    assert (std[inp.outlier_idx] > 4.0).all()
    others = np.setdiff1d(np.arange(w.d_qk), inp.outlier_idx)
    assert (std[others] < 1.3).all()
    for g in range(w.n_kv_heads):
        pos = inp.needle_pos[0, g]
        norms = np.linalg.norm(K[g, pos], axis=1)
        np.testing.assert_allclose(norms, 4.0, rtol=1e-2)


def test_query_stream_is_ar1():
    w = W.WORKLOADS["stream96k_bf16"].with_(ctx=256, steps=64)
    qs = W.to_f64(W.make_query_stream(w), w.dtype)
    x = qs[:-1].ravel()
    y = qs[1:].ravel()
    rho = np.corrcoef(x, y)[0, 1]
    assert abs(rho - 0.9) < 0.02
    inp = W.make_decode_inputs(w)
    np.testing.assert_array_equal(W.make_query_stream(w)[0], inp.q)


def test_paged_host_layout():
    w = W.WORKLOADS["stream96k_bf16"].with_(ctx=100, n_needles=2)
    inp = W.make_decode_inputs(w)
    hk = W.paged_host_kv(inp)
    assert hk.shape == (1, 8, 4, 2, 32, 128)
    np.testing.assert_array_equal(hk[0, 3, 1, 0], inp.K[0, 3, 32:64])
    np.testing.assert_array_equal(hk[0, 3, 3, 1, :4], inp.V[0, 3, 96:100])
    assert (hk[0, 3, 3, :, 4:] == 0).all()
