"""Host-side logic of bench.py that the reported numbers rest on (no GPU)."""
import json

import bench
from two_level_sparse_quest_b200 import workloads as W


def test_algorithmic_bytes_of_the_benchmark_workload():
    w = W.WORKLOADS["gqa96k_b8_bf16"]
    ab = bench.algorithmic_bytes(w)
    G = 8 * 8
    assert ab["block_summary"] == G * 3072 * 2 * 128 * 2          # every block's max and min rows
    assert ab["label_slab"] == G * 256 * 32 * 16 * 2              # the K_b * bs candidates' label rows
    assert ab["gathered_kv"] == G * 4096 * (128 + 128) * 2        # K and V rows of the kept tokens
    assert ab["total"] == 254084096
    assert ab["stage_select"] == ab["stage_block"] + ab["stage_token"] - ab["q"]
    assert sum(ab[k] for k in ("block_summary", "label_slab", "gathered_kv", "q", "out_lse", "indices")) == ab["total"]


def test_int8_slab_halves_the_label_bytes_and_adds_the_scales():
    w = W.WORKLOADS["gqa96k_b8_bf16"]
    a0 = bench.algorithmic_bytes(w)
    a8 = bench.algorithmic_bytes(w.with_(slab_bits=8))
    G = 8 * 8
    assert a8["label_slab"] == a0["label_slab"] // 2 + G * 16 * 4
    assert a8["block_summary"] == a0["block_summary"] and a8["gathered_kv"] == a0["gathered_kv"]


def test_latent_workload_reads_no_separate_values():
    w = W.WORKLOADS["mla64k_b4_bf16"]
    ab = bench.algorithmic_bytes(w)
    assert ab["gathered_kv"] == 4 * 1 * 2048 * 576 * 2  # V is the first 512 channels of the latent row


def test_traffic_is_only_reported_for_the_current_kernel_sources(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda files=None: "abc")
    (prof / "traffic.json").write_text(json.dumps({"stage_select": {"bytes_per_launch": 5.0, "source_hash": "abc"}}))
    assert bench.read_traffic("stage_select") == 5.0
    assert bench.read_traffic("stage_attn") is None
    (prof / "traffic.json").write_text(json.dumps({"stage_select": {"bytes_per_launch": 5.0, "source_hash": "old"}}))
    assert bench.read_traffic("stage_select") is None


def test_oracle_baseline_splits_the_step_into_its_groups_without_changing_it():
    """The CPU baseline runs each (sequence, KV head) group as its own oracle
    call on a thread pool; that must be the same computation as the oracle on
    the whole batch."""
    import numpy as np

    from oracle import oracle as O

    w = W.WORKLOADS["gqa48k_bf16"].with_(batch=2, n_kv_heads=2, n_q_heads=8, ctx=1024, k_b=8, k_t=64)
    inp = W.make_decode_inputs(w, seq_lens=[1024, 777])
    st = bench.OracleStep(w, inp, threads=3)
    assert len(st.groups) == 4
    s = O.shape_of(w)
    meta = O.build_meta(s, inp.K, inp.seq_lens)
    bidx, tidx, out, lse = O.decode_step(s, inp.q, inp.K, inp.V, meta, inp.seq_lens, inp.label_idx)
    G = w.group
    for i, gr in enumerate(st.groups):
        b, g = divmod(i, w.n_kv_heads)
        rb, rt, ro, rl = O.decode_step(st.s, np.ascontiguousarray(gr["q"]), gr["K"], gr["V"], gr["meta"], gr["sl"],
                                       gr["label"])
        np.testing.assert_array_equal(rb[0, 0], bidx[b, g])
        np.testing.assert_array_equal(rt[0, 0], tidx[b, g])
        np.testing.assert_array_equal(ro[0], out[b, g * G:(g + 1) * G])
        np.testing.assert_array_equal(rl[0], lse[b, g * G:(g + 1) * G])
    assert st.run() > 0 and st.run(2, threads=False) > 0
