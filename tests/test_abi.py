"""C-ABI checks that need no GPU: the library loads, exports every symbol
declared in include/tls.h, the ctypes struct matches the C layout, and host-side
argument checks return status codes (never abort) before anything is enqueued."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tls.h")


@pytest.fixture(scope="module")
def T():
    from two_level_sparse_quest_b200 import build

    build.build()
    from two_level_sparse_quest_b200 import tls

    return tls


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^TLS_API\s+[\w\s\*]+?\b(tls_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_expected_entry_points():
    syms = declared_symbols()
    for name in ("tls_build_block_meta", "tls_block_score_topk", "tls_token_score_topk", "tls_sparse_attn_decode",
                 "tls_prefetch_diff", "tls_workspace_size", "tls_last_error", "tls_wait_event"):
        assert name in syms


def test_library_exports_every_declared_symbol(T):
    lib = ctypes.CDLL(T.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) == set(T.EXPORTED)


def test_oracle_library_is_separate_and_loads():
    from oracle import oracle as O

    L = O.lib()
    assert L.ora_abi_version() == 1
    assert not hasattr(L, "tls_block_score_topk")


def test_shape_struct_layout_matches_c(T):
    fields = [n for n, _ in T.TlsShape._fields_]
    prog = "#include <stdio.h>\n#include <stddef.h>\n#include \"tls.h\"\nint main(void){\n"
    prog += 'printf("%zu\\n", sizeof(tls_shape));\n'
    for f in fields:
        prog += f'printf("%zu\\n", offsetof(tls_shape, {f}));\n'
    prog += "return 0;}\n"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        open(c, "w").write(prog)
        exe = os.path.join(d, "t")
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe])
        vals = [int(x) for x in subprocess.check_output([exe]).split()]
    assert vals[0] == ctypes.sizeof(T.TlsShape)
    for f, off in zip(fields, vals[1:]):
        assert getattr(T.TlsShape, f).offset == off, f


def good_shape(T, **kw):
    base = dict(batch=1, n_q_heads=32, n_kv_heads=8, d_qk=128, d_v=128, block_size=32, n_label=16, k_b=192,
                k_t=2048, max_ctx=49152, kv_dtype=T.TLS_BF16)
    base.update(kw)
    return T.make_shape(**base)


def call_block(T, s, q=256, meta=256, sl=256, out=256, ws=(256, 1 << 30)):
    return T._lib.tls_block_score_topk(ctypes.byref(s), q, meta, sl, out, None, ws[0], ws[1], None)


def test_version_and_last_error(T):
    assert T.tls_version().startswith("tls ")
    assert T._lib.tls_block_score_topk(None, None, None, None, None, None, None, 0, None) == T.TLS_ERR_INVALID_ARG
    assert "shape is NULL" in T.tls_last_error()


@pytest.mark.parametrize("kw,status", [
    (dict(n_q_heads=30), "TLS_ERR_INVALID_ARG"),
    (dict(d_qk=96, d_v=96), "TLS_ERR_UNSUPPORTED"),
    (dict(n_q_heads=48), "TLS_ERR_UNSUPPORTED"),      # G = 6
    (dict(k_b=0), "TLS_ERR_INVALID_ARG"),
    (dict(k_t=0), "TLS_ERR_INVALID_ARG"),
    (dict(block_size=0), "TLS_ERR_INVALID_ARG"),
    (dict(kv_dtype=7), "TLS_ERR_INVALID_ARG"),
    (dict(n_label=12), "TLS_ERR_UNSUPPORTED"),
    (dict(k_b=1025, block_size=8), "TLS_ERR_UNSUPPORTED"),
    (dict(k_b=600), "TLS_ERR_UNSUPPORTED"),          # 600 * 32 candidates > 16384
    (dict(max_ctx=1 << 20, block_size=32), "TLS_ERR_UNSUPPORTED"),
    # ceil(max_ctx / bs) must not wrap in int: near INT32_MAX it is refused, never a negative count
    (dict(max_ctx=2 ** 31 - 1, block_size=1 << 20), "TLS_ERR_UNSUPPORTED"),
    (dict(max_ctx=2 ** 31 - 16, block_size=32), "TLS_ERR_UNSUPPORTED"),
    (dict(v_is_k_prefix=True, n_q_heads=64, n_kv_heads=1, d_qk=576, d_v=512, kv_dtype=0), "TLS_ERR_UNSUPPORTED"),
])
def test_shape_checks_return_status(T, kw, status):
    s = good_shape(T, **kw)
    assert T.STATUS_NAMES[call_block(T, s)] == status
    assert T.tls_last_error()


def test_pointer_checks(T):
    s = good_shape(T)
    assert call_block(T, s, q=None) == T.TLS_ERR_INVALID_ARG and "q is NULL" in T.tls_last_error()
    assert call_block(T, s, meta=258) == T.TLS_ERR_INVALID_ARG and "aligned" in T.tls_last_error()
    assert call_block(T, s, out=0x1002) == T.TLS_ERR_INVALID_ARG
    st = T._lib.tls_sparse_attn_decode(ctypes.byref(s), 256, 256, None, 256, 256, None, 256, 1 << 30, None)
    assert st == T.TLS_ERR_INVALID_ARG and "V is NULL" in T.tls_last_error()
    st = T._lib.tls_sparse_attn_decode(ctypes.byref(s), 256, 256, 256, 256, 256, None, 256, 8, None)
    assert st == T.TLS_ERR_WORKSPACE


def test_block_aggregation_field_is_checked(T):
    s = good_shape(T)
    s.block_agg = 2
    assert call_block(T, s) == T.TLS_ERR_INVALID_ARG and "block_agg" in T.tls_last_error()
    # the latent shape takes the max-over-heads scores on the tensor cores, which need room for
    # the scores: without block_score_out or a workspace the call is refused before any launch
    mla = good_shape(T, v_is_k_prefix=True, n_q_heads=64, n_kv_heads=1, d_qk=576, d_v=512, n_label=32)
    mla.block_agg = 1
    assert call_block(T, mla, ws=(None, 0)) == T.TLS_ERR_WORKSPACE and "block_score_out" in T.tls_last_error()
    big = good_shape(T, v_is_k_prefix=True, n_q_heads=128, n_kv_heads=1, d_qk=576, d_v=512, n_label=32)
    big.block_agg = 1
    assert call_block(T, big) == T.TLS_ERR_UNSUPPORTED
    f32 = good_shape(T, kv_dtype=T.TLS_F32, n_q_heads=16, n_kv_heads=1, d_qk=64, d_v=64)
    f32.block_agg = 1
    assert call_block(T, f32) == T.TLS_ERR_UNSUPPORTED


def test_group_sizes(T):
    for G in (1, 2, 4, 8, 16, 32, 64):  # host-side plan only: nothing is launched
        assert T.tls_workspace_size(good_shape(T, n_q_heads=G, n_kv_heads=1)) > 0
        assert T.tls_workspace_size(good_shape(T, n_q_heads=G, n_kv_heads=1, d_qk=64, d_v=64)) > 0
    st = call_block(T, good_shape(T, n_q_heads=24, n_kv_heads=1))
    assert st == T.TLS_ERR_UNSUPPORTED and "group size" in T.tls_last_error()
    # max-over-heads with 16 heads per group: the tensor-core path, which needs room for the scores
    mq = good_shape(T, n_q_heads=16, n_kv_heads=1)
    mq.block_agg = 1
    assert call_block(T, mq, ws=(None, 0)) == T.TLS_ERR_WORKSPACE and "16 heads" in T.tls_last_error()


def test_int8_slab_field_and_size(T):
    s = good_shape(T)
    n0 = T.tls_slab_bytes(s)
    assert n0 == s.batch * s.n_kv_heads * s.max_ctx * s.n_label * (2 if s.kv_dtype == T.TLS_BF16 else 4)
    s.slab_bits = 8
    if s.kv_dtype == T.TLS_BF16 and s.n_label >= 16:
        codes = s.batch * s.n_kv_heads * s.max_ctx * s.n_label
        assert T.tls_slab_bytes(s) == -(-codes // 256) * 256 + 4 * s.batch * s.n_kv_heads * s.n_label
    s.slab_bits = 4
    assert call_block(T, s) == T.TLS_ERR_INVALID_ARG and "slab_bits" in T.tls_last_error()
    f32 = good_shape(T, kv_dtype=T.TLS_F32, n_label=16)
    f32.slab_bits = 8
    assert call_block(T, f32) == T.TLS_ERR_UNSUPPORTED and "int8" in T.tls_last_error()
    r8 = good_shape(T, kv_dtype=T.TLS_BF16, n_label=8)
    r8.slab_bits = 8
    assert call_block(T, r8) == T.TLS_ERR_UNSUPPORTED
    with pytest.raises(T.TlsError):
        T.tls_slab_bytes(r8)
    q8 = good_shape(T, kv_dtype=T.TLS_BF16, n_label=16)
    q8.slab_bits = 8
    st = T._lib.tls_append_tokens(ctypes.byref(q8), 256, 256, 256, 4, 256, 256, 256, None)
    assert st == T.TLS_ERR_UNSUPPORTED and "int8" in T.tls_last_error()


def test_select_step_checks_before_launch(T):
    s = good_shape(T)
    st = T._lib.tls_select_step(ctypes.byref(s), 256, 256, None, 256, 256, 256, 256, None, None, None)
    assert st == T.TLS_ERR_INVALID_ARG and "slab is NULL" in T.tls_last_error()
    bad = good_shape(T, k_b=600)
    st = T._lib.tls_select_step(ctypes.byref(bad), 256, 256, 256, 256, 256, 256, 256, None, None, None)
    assert st == T.TLS_ERR_UNSUPPORTED


def test_select_step_ws_checks_before_launch(T):
    s = good_shape(T)
    need = T.tls_workspace_size(s)
    # workspace missing, too small or misaligned: refused before anything else
    for ws, nbytes in ((None, need), (256, need - 1), (0x1010, need)):
        st = T._lib.tls_select_step_ws(ctypes.byref(s), 256, 256, 256, 256, 256, 256, 256, None, None, ws, nbytes,
                                       None)
        assert st == T.TLS_ERR_WORKSPACE and str(need) in T.tls_last_error()
    # then the pointers, as tls_select_step checks them
    st = T._lib.tls_select_step_ws(ctypes.byref(s), 256, 256, None, 256, 256, 256, 256, None, None, 256, need, None)
    assert st == T.TLS_ERR_INVALID_ARG and "slab is NULL" in T.tls_last_error()


def test_append_tokens_checks_before_launch(T):
    s = good_shape(T)
    assert T._lib.tls_append_tokens(ctypes.byref(s), 256, 256, 256, -1, 256, 256, None, None) == T.TLS_ERR_INVALID_ARG
    assert "max_append" in T.tls_last_error()
    assert T._lib.tls_append_tokens(ctypes.byref(s), None, 256, 256, 4, 256, 256, None, None) == T.TLS_ERR_INVALID_ARG
    assert "K is NULL" in T.tls_last_error()
    assert T._lib.tls_append_tokens(ctypes.byref(s), None, None, None, 0, None, None, None, None) == T.TLS_OK


def test_binding_refuses_host_tensors_for_device_arguments(T):
    import torch

    s = good_shape(T)
    cpu = torch.zeros(16, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        T.tls_block_score_topk(s, cpu, cpu, cpu, cpu)
    with pytest.raises(ValueError, match="CUDA tensor"):
        T.tls_select_step(s, 256, 256, 256, 256, 256, 256, cpu)
    with pytest.raises(ValueError, match="CUDA tensor"):
        T.tls_sparse_attn_decode(s, 256, 256, 256, 256, 256, None, ws=cpu)
    with pytest.raises(ValueError, match="pinned"):
        T.tls_prefetch_diff(s, 384, cpu, 256, 256, 256, 256, 256, 256, 256)


def test_device_error_checks_its_argument(T):
    assert T._lib.tls_device_error(None, 0) == T.TLS_ERR_INVALID_ARG
    assert "flags_out is NULL" in T.tls_last_error()


def test_empty_batch_is_a_noop(T):
    s = good_shape(T, batch=0)
    assert T._lib.tls_block_score_topk(ctypes.byref(s), None, None, None, None, None, None, 0, None) == T.TLS_OK
    assert T._lib.tls_sparse_attn_decode(ctypes.byref(s), None, None, None, None, None, None, None, 0, None) == T.TLS_OK


def test_workspace_size_is_positive_for_supported_shapes(T):
    from two_level_sparse_quest_b200 import workloads as W

    for w in W.WORKLOADS.values():
        s = T.shape_from_workload(w)
        n = T.tls_workspace_size(s)
        assert n > 0 and n % 256 == 0
    with pytest.raises(T.TlsError):
        T.tls_workspace_size(good_shape(T, d_qk=96, d_v=96))


def test_offload_checks(T):
    s = good_shape(T)
    assert T._lib.tls_offload_reset(ctypes.byref(s), 0, 256, 256, None) == T.TLS_ERR_INVALID_ARG
    assert T._lib.tls_offload_reset(ctypes.byref(s), 5000, 256, 256, None) == T.TLS_ERR_INVALID_ARG
    sm = good_shape(T, v_is_k_prefix=True, n_q_heads=64, n_kv_heads=1, d_qk=576, d_v=512, block_size=64,
                    n_label=32, k_b=128, max_ctx=65536)
    assert T._lib.tls_offload_reset(ctypes.byref(sm), 256, 256, 256, None) == T.TLS_ERR_UNSUPPORTED
    st = T._lib.tls_prefetch_diff(ctypes.byref(s), 384, None, 256, 256, 256, None, 256, 256, 256, None)
    assert st == T.TLS_ERR_INVALID_ARG and "host_kv" in T.tls_last_error()


def test_wait_event_rejects_null(T):
    assert T._lib.tls_wait_event(None, 10) == T.TLS_ERR_INVALID_ARG
