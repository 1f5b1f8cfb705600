"""The C-ABI library without a GPU: it builds, loads, exports every declared symbol, and its
host-side logic (layout queries, argument validation, status strings) behaves as documented.
No kernel is launched here."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tp_block.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+(tp_[a-z0-9_]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("tp_mlp_fwd", "tp_mlp_bwd", "tp_attn_fwd", "tp_reduce_partials"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    so = lib.load()
    for name in _declared_functions():
        assert hasattr(so, name), name
    assert set(_declared_functions()) == set(lib.EXPORTS)


def test_version_and_status_strings(lib):
    assert lib.tp_version() >= 100
    so = lib.load()
    assert so.tp_status_string(0) == b"TP_OK"
    assert so.tp_status_string(2) == b"TP_ERR_SHAPE"
    assert so.tp_status_string(6) == b"TP_ERR_TIMEOUT"


def test_mlp_layout_sizes(lib):
    # decode MLP shape: T=64, d=8192, d_ff=28672, p=8, SwiGLU, bf16
    d = lib.mlp_desc(64, 8192, 28672, 8, "swiglu", "bf16")
    fs = 28672 // 8
    assert lib.tp_mlp_w1_packed_bytes(d) == 8 * 2 * fs * 8192 * 2
    assert lib.tp_mlp_w2_packed_bytes(d) == 8 * 8192 * fs * 2
    # weights total 1,409,286,144 bytes (3 matrices of 8192 x 28672 bf16)
    assert lib.tp_mlp_w1_packed_bytes(d) + lib.tp_mlp_w2_packed_bytes(d) == 1_409_286_144
    # padding: F_s = 8 pads to 128 per shard
    t = lib.mlp_desc(4, 8, 32, 4, "gelu", "f32")
    assert lib.tp_mlp_w1_packed_bytes(t) == 4 * 128 * 8 * 4
    assert lib.tp_mlp_w2_packed_bytes(t) == 4 * 8 * 128 * 4
    assert lib.tp_mlp_saved_bytes(t) >= (4 * 4 * 128 + 4 * 4 * 128) * 4
    assert lib.tp_mlp_fwd_workspace(t) >= 4 * 4 * 8 * 4
    assert lib.tp_mlp_bwd_workspace(t) >= 4 * 4 * 8 * 4


def test_attn_layout_sizes(lib):
    a = lib.attn_desc(1, 2048, 8192, 64, 8, 128, 8)
    assert lib.tp_attn_wqkv_packed_bytes(a) == 8 * (1024 + 128 + 128) * 8192 * 2
    assert lib.tp_attn_wo_packed_bytes(a) == 8 * 8192 * 1024 * 2
    assert lib.tp_attn_fwd_workspace(a) > 0


@pytest.mark.parametrize("T,d,F,p,status", [
    (4, 8, 30, 4, "TP_ERR_SHAPE"),     # p does not divide d_ff
    (4, 8, 32, 0, "TP_ERR_SHAPE"),     # p < 1
    (-1, 8, 32, 4, "TP_ERR_SHAPE"),    # negative T
    (4, 0, 32, 4, "TP_ERR_SHAPE"),     # d < 1
])
def test_mlp_shape_errors(lib, T, d, F, p, status):
    desc = lib.mlp_desc(T, d, F, p, "gelu", "f32")
    so = lib.load()
    st = so.tp_mlp_fwd(ctypes.byref(desc), None, None, None, None, None, None, None, None, 0, None)
    assert so.tp_status_string(st).decode() == status
    assert lib.tp_mlp_fwd_workspace(desc) == 0
    assert lib.tp_last_error() != ""


def test_mlp_argument_errors(lib):
    so = lib.load()
    desc = lib.mlp_desc(4, 8, 32, 4, "gelu", "f32")
    st = so.tp_mlp_fwd(ctypes.byref(desc), None, None, None, None, None, None, None, None, 0, None)
    assert st == lib.TP_ERR_INVALID_ARG  # null x
    fake = ctypes.c_void_p(0x1000)
    st = so.tp_mlp_fwd(ctypes.byref(desc), fake, fake, fake, None, fake, None, None, fake, 16, None)
    assert st == lib.TP_ERR_WORKSPACE
    bad = lib.mlp_desc(4, 8, 32, 4, 9, "f32")
    assert so.tp_mlp_fwd(ctypes.byref(bad), fake, fake, fake, None, fake, None, None, fake, 1 << 30,
                         None) == lib.TP_ERR_INVALID_ARG
    bad = lib.mlp_desc(4, 8, 32, 4, "gelu", 7)
    assert so.tp_mlp_fwd(ctypes.byref(bad), fake, fake, fake, None, fake, None, None, fake, 1 << 30,
                         None) == lib.TP_ERR_INVALID_ARG
    # SwiGLU needs w_up; the other activations must not get one
    sw = lib.mlp_desc(4, 8, 32, 4, "swiglu", "f32")
    assert so.tp_mlp_pack(ctypes.byref(sw), fake, None, fake, fake, fake, None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_mlp_pack(ctypes.byref(desc), fake, fake, fake, fake, fake, None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_mlp_fwd(ctypes.byref(desc), None, None, None, None, None, None, None, None, 0, None) != 0


def test_attn_shape_errors(lib):
    so = lib.load()
    fake = ctypes.c_void_p(0x1000)

    def st(desc):
        return so.tp_attn_fwd(ctypes.byref(desc), fake, fake, fake, None, None, None, fake, None,
                              fake, 1 << 40, None)
    # "Tensor Parallelism", Notes: with 8 KV heads, p = 16 cannot give every rank a whole KV head
    assert st(lib.attn_desc(1, 4, 64, 16, 8, 8, 16)) == lib.TP_ERR_SHAPE
    assert st(lib.attn_desc(1, 4, 64, 8, 3, 8, 1)) == lib.TP_ERR_SHAPE     # n_kv does not divide n_q
    assert st(lib.attn_desc(1, 4, 64, 8, 8, 12, 1)) == lib.TP_ERR_SHAPE    # head_dim not a multiple of 8
    assert st(lib.attn_desc(1, 2, 64, 8, 8, 8, 1, kv_len=5)) == lib.TP_ERR_SHAPE   # decode needs s=1
    assert st(lib.attn_desc(1, 1, 64, 8, 8, 8, 1, kv_len=5, kv_cap=5)) == lib.TP_ERR_SHAPE


def test_reduce_argument_errors(lib):
    so = lib.load()
    fake = ctypes.c_void_p(0x1000)
    assert so.tp_reduce_partials(fake, 0, 16, 0, None, fake, 0, None) == lib.TP_ERR_SHAPE
    assert so.tp_reduce_partials(fake, 2, -1, 0, None, fake, 0, None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_reduce_partials(None, 2, 16, 0, None, fake, 0, None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_reduce_partials(fake, 2, 16, 5, None, fake, 0, None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_rmsnorm(fake, 0, 2, 0, 1e-5, fake, 0, None) == lib.TP_ERR_SHAPE
    assert so.tp_rmsnorm(fake, 3, 2, 8, 1e-5, fake, 0, None) == lib.TP_ERR_INVALID_ARG
    bad = lib.mlp_desc(4, 8, 32, 4, "gelu", "f32", flags=4)
    assert so.tp_mlp_fwd(ctypes.byref(bad), fake, fake, fake, None, fake, None, None, fake, 1 << 30,
                         None) == lib.TP_ERR_INVALID_ARG
    # the failure-detection self-test checks its limit before enqueueing anything
    assert so.tp_selftest_wait_timeout(0, None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_selftest_wait_timeout(1000001, None) == lib.TP_ERR_INVALID_ARG


def test_empty_batch_counts_one_reduction(lib):
    # T = 0 is a valid, empty call: nothing is launched, the block still has its one reduction
    so = lib.load()
    lib.tp_reset_reduction_count()
    desc = lib.mlp_desc(0, 8, 32, 4, "gelu", "f32")
    assert so.tp_mlp_fwd(ctypes.byref(desc), None, None, None, None, None, None, None, None, 0, None) == 0
    assert lib.tp_reduction_count() == 1
    lib.tp_reset_reduction_count()


def test_sequence_parallel_argument_errors(lib):
    # checked on the host before anything is enqueued
    so = lib.load()
    fake = ctypes.c_void_p(0x1000)
    two = (ctypes.c_void_p * 2)(0x1000, 0x2000)
    one_null = (ctypes.c_void_p * 2)(0x1000, None)
    arr = lambda a: ctypes.cast(a, ctypes.c_void_p)
    # p must divide T
    assert so.tp_reduce_scatter_partials(fake, 2, 5, 8, None, arr(two), 1, None, 1, 1e-5,
                                         None) == lib.TP_ERR_SHAPE
    # every slice pointer must be given
    assert so.tp_reduce_scatter_partials(fake, 2, 4, 8, None, arr(one_null), 1, None, 1, 1e-5,
                                         None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_reduce_scatter_partials(fake, 2, 4, 8, None, None, 1, None, 1, 1e-5,
                                         None) == lib.TP_ERR_INVALID_ARG
    # at most 64 slices
    assert so.tp_reduce_scatter_partials(fake, 65, 65, 8, None, arr(two), 1, None, 1, 1e-5,
                                         None) == lib.TP_ERR_SHAPE
    assert so.tp_all_gather_slices(arr(two), 2, 4, 8, 7, fake, None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_all_gather_slices(arr(one_null), 2, 4, 8, 1, fake, None) == lib.TP_ERR_INVALID_ARG
    # the block calls: p must divide the tokens; the fused reduce has no sequence-parallel form
    d_ok = lib.mlp_desc(8, 64, 256, 2, "swiglu", "bf16")
    d_rag = lib.mlp_desc(9, 64, 256, 2, "swiglu", "bf16")
    d_fused = lib.mlp_desc(8, 64, 256, 2, "swiglu", "bf16", lib.TP_REDUCE_FUSED)
    assert lib.tp_mlp_fwd_sp_workspace(d_ok) > lib.tp_mlp_fwd_workspace(d_ok)
    assert lib.tp_mlp_fwd_sp_workspace(d_rag) == 0
    assert lib.tp_mlp_bwd_sp_workspace(d_fused) == 0
    assert so.tp_mlp_fwd_sp(ctypes.byref(d_rag), arr(two), fake, fake, None, arr(two), None, None,
                            fake, 1 << 30, None) == lib.TP_ERR_SHAPE
    assert so.tp_mlp_fwd_sp(ctypes.byref(d_fused), arr(two), fake, fake, None, arr(two), None,
                            None, fake, 1 << 30, None) == lib.TP_ERR_UNSUPPORTED
    a_rag = lib.attn_desc(1, 9, 64, 4, 2, 16, 2)
    assert lib.tp_attn_fwd_sp_workspace(a_rag) == 0
    a_ok = lib.attn_desc(1, 8, 64, 4, 2, 16, 2)
    assert lib.tp_attn_fwd_sp_workspace(a_ok) > lib.tp_attn_fwd_workspace(a_ok)


def test_moe_layout_and_argument_errors(lib):
    so = lib.load()
    d = lib.moe_desc(64, 256, 512, 256, 16, 2, 2)
    # one expert packs like the dense SwiGLU MLP of the same d, d_ff, p
    md = lib.mlp_desc(64, 256, 512, 2, "swiglu", "bf16")
    assert lib.tp_moe_expert_w1_bytes(d) == lib.tp_mlp_w1_packed_bytes(md)
    assert lib.tp_moe_expert_w2_bytes(d) == lib.tp_mlp_w2_packed_bytes(md)
    md_s = lib.mlp_desc(64, 256, 256, 2, "swiglu", "bf16")
    assert lib.tp_moe_shared_w1_bytes(d) == lib.tp_mlp_w1_packed_bytes(md_s)
    assert lib.tp_moe_shared_w1_bytes(lib.moe_desc(64, 256, 512, 0, 16, 2, 2)) == 0
    assert lib.tp_moe_fwd_workspace(d) > 0
    for bad in (lib.moe_desc(64, 256, 512, 0, 12, 2, 2), lib.moe_desc(64, 256, 512, 0, 16, 0, 2),
                lib.moe_desc(64, 250, 512, 0, 16, 2, 2), lib.moe_desc(64, 256, 512, 100, 16, 2, 8)):
        assert lib.tp_moe_fwd_workspace(bad) == 0
    fake = ctypes.c_void_p(0x1000)
    lib.tp_reset_reduction_count()
    empty = lib.moe_desc(0, 256, 512, 0, 16, 2, 2)
    assert so.tp_moe_fwd(ctypes.byref(empty), None, None, None, None, None, None, None, None, None,
                         None, None, None, 0, None) == 0
    assert lib.tp_reduction_count() == 1
    assert so.tp_moe_fwd(ctypes.byref(d), None, fake, fake, fake, fake, fake, None, None, fake,
                         None, None, fake, 1 << 40, None) == lib.TP_ERR_INVALID_ARG
    lib.tp_reset_reduction_count()
    # the backward: its workspace holds the forward's and more; argument errors before any enqueue
    assert lib.tp_moe_bwd_workspace(d) > lib.tp_moe_fwd_workspace(d)
    assert lib.tp_moe_bwd_workspace(lib.moe_desc(64, 256, 512, 0, 12, 2, 2)) == 0
    args = [fake] * 6 + [fake, fake]          # x, wr, w1p, w2p, w1p_s, w2p_s, dy, dx
    grads = [fake, fake, fake, fake, fake]    # dwr, dw1p, dw2p, dw1p_s, dw2p_s
    assert so.tp_moe_bwd(ctypes.byref(d), *args, None, *grads[1:], fake, 1 << 40,
                         None) == lib.TP_ERR_INVALID_ARG          # dwr null
    assert so.tp_moe_bwd(ctypes.byref(d), *args, *grads[:3], None, fake, fake, 1 << 40,
                         None) == lib.TP_ERR_INVALID_ARG          # the shared expert's dw1p null
    assert so.tp_moe_bwd(ctypes.byref(d), *args, *grads, fake, 64,
                         None) == lib.TP_ERR_WORKSPACE            # workspace too small


def test_moe_pack_and_sp_backward_argument_errors(lib):
    # host-side checks only: nothing is enqueued when they fail
    so = lib.load()
    fake = ctypes.c_void_p(0x1000)
    d = lib.moe_desc(8, 256, 512, 0, 8, 2, 2)
    ok8 = (ctypes.c_void_p * 8)(*([0x1000] * 8))
    arr = lambda a: ctypes.cast(a, ctypes.c_void_p)
    assert so.tp_moe_pack(ctypes.byref(d), None, arr(ok8), arr(ok8), None, None, None, fake, fake,
                          None, None, None) == lib.TP_ERR_INVALID_ARG
    ds = lib.moe_desc(8, 256, 512, 256, 8, 2, 2)   # a shared expert needs its weights
    assert so.tp_moe_fwd(ctypes.byref(ds), fake, fake, fake, fake, None, None, None, None, fake,
                         None, None, fake, 1 << 40, None) == lib.TP_ERR_INVALID_ARG
    # workspace too small
    assert so.tp_moe_fwd(ctypes.byref(d), fake, fake, fake, fake, None, None, None, None, fake,
                         None, None, fake, 16, None) == lib.TP_ERR_WORKSPACE
    two = (ctypes.c_void_p * 2)(0x1000, 0x2000)
    dm = lib.mlp_desc(8, 64, 256, 2, "swiglu", "bf16")
    # the backward needs the forward's saved activations and every slice
    assert so.tp_mlp_bwd_sp(ctypes.byref(dm), arr(two), arr(two), None, fake, fake, arr(two), fake,
                            fake, fake, 1 << 30, None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_mlp_bwd_sp(ctypes.byref(dm), arr(two), None, fake, fake, fake, arr(two), fake,
                            fake, fake, 1 << 30, None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_mlp_bwd_sp(ctypes.byref(dm), arr(two), arr(two), fake, fake, fake, arr(two), fake,
                            fake, fake, 16, None) == lib.TP_ERR_WORKSPACE


def test_product_and_oracle_are_independent():
    # the product package never imports the oracle, and the oracle never imports the product
    # (they share only the seeded input generators, which hold none of the block's arithmetic)
    pkg = os.path.join(ROOT, "tensor_transformer_matmul_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", src, re.M), f
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith(".py"):
            src = open(os.path.join(ROOT, "oracle", f)).read()
            assert "tensor_transformer_matmul_b200" not in src, f
            assert "libtpblock" not in src, f
    # no CUDA source names the oracle
    csrc = os.path.join(pkg, "csrc")
    for f in os.listdir(csrc):
        assert "oracle" not in open(os.path.join(csrc, f)).read().lower(), f


def test_shard_sizes_are_one_pth_of_the_packing(lib):
    # one shard per device: its packed weights are exactly its slice of the p-shard packing
    d = lib.mlp_desc(64, 8192, 28672, 8, "swiglu", "bf16")
    s = lib.tp_mlp_shard_sizes(d, "bf16")
    assert s.col_weight_bytes * 8 == lib.tp_mlp_w1_packed_bytes(d)
    assert s.row_weight_bytes * 8 == lib.tp_mlp_w2_packed_bytes(d)
    assert s.partial_bytes == 64 * 8192 * 2          # the pages' 1 MiB decode all-reduce payload
    assert lib.tp_mlp_shard_sizes(d, "f32").partial_bytes == 64 * 8192 * 4
    a = lib.attn_desc(1, 2048, 8192, 64, 8, 128, 8)
    sa = lib.tp_attn_shard_sizes(a, "f32")
    assert sa.col_weight_bytes * 8 == lib.tp_attn_wqkv_packed_bytes(a)
    assert sa.row_weight_bytes * 8 == lib.tp_attn_wo_packed_bytes(a)
    # per shard Wq 8192x1024, Wk and Wv 8192x128, Wo 1024x8192 (bf16)
    assert sa.col_weight_bytes == 8192 * (1024 + 2 * 128) * 2
    assert sa.row_weight_bytes == 1024 * 8192 * 2
    assert sa.bwd_workspace == 0                      # the attention backward takes bf16 partials
    assert lib.tp_attn_shard_sizes(a, "bf16").bwd_workspace > 0


def test_shard_argument_checks(lib):
    so = lib.load()
    fake = ctypes.c_void_p(0x1000)           # never dereferenced: each call fails its checks first
    d = lib.mlp_desc(8, 64, 256, 4, "swiglu", "bf16")
    for shard in (-1, 4):
        assert so.tp_mlp_fwd_shard(ctypes.byref(d), shard, lib.TP_F32, fake, fake, fake, fake,
                                   None, fake, 1 << 30, None) == lib.TP_ERR_INVALID_ARG
        assert so.tp_mlp_pack_shard(ctypes.byref(d), shard, fake, fake, fake, fake, fake,
                                    None) == lib.TP_ERR_INVALID_ARG
    # a bad partial dtype, and bf16 partials of an fp32 block
    assert so.tp_mlp_fwd_shard(ctypes.byref(d), 0, 7, fake, fake, fake, fake, None, fake,
                               1 << 30, None) == lib.TP_ERR_INVALID_ARG
    with pytest.raises(lib.TpError) as e:
        lib.tp_mlp_shard_sizes(lib.mlp_desc(8, 64, 256, 4, "swiglu", "f32"), "bf16")
    assert e.value.status == lib.TP_ERR_UNSUPPORTED
    with pytest.raises(lib.TpError) as e:     # the partial dtype replaces the flags
        lib.tp_mlp_shard_sizes(lib.mlp_desc(8, 64, 256, 4, "swiglu", "bf16",
                                            flags=lib.TP_FLAG_F32_RESIDUAL), "f32")
    assert e.value.status == lib.TP_ERR_INVALID_ARG
    with pytest.raises(lib.TpError) as e:     # p must divide the heads
        lib.tp_attn_shard_sizes(lib.attn_desc(1, 4, 64, 6, 3, 8, 2), "f32")
    assert e.value.status == lib.TP_ERR_SHAPE
    a = lib.attn_desc(1, 4, 64, 4, 2, 8, 2)
    assert so.tp_attn_fwd_shard(ctypes.byref(a), 2, lib.TP_F32, fake, fake, fake, None, None,
                                fake, fake, 1 << 30, None) == lib.TP_ERR_INVALID_ARG
    assert so.tp_attn_bwd_shard(ctypes.byref(a), -1, fake, fake, fake, fake, fake, fake, fake,
                                fake, 1 << 30, None) == lib.TP_ERR_INVALID_ARG
    # too small a workspace: refused before anything is enqueued
    assert so.tp_mlp_fwd_shard(ctypes.byref(d), 1, lib.TP_F32, fake, fake, fake, fake, None,
                               fake, 16, None) == lib.TP_ERR_WORKSPACE
