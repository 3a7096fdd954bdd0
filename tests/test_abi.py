"""CPU checks of the C ABI: the library loads, exports every function include/had.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "had.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\**\s*(had_[a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    import binarized_qk_sparse_b200 as m
    from binarized_qk_sparse_b200 import _build
    _build.build()
    return m.lib()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for must in ("had_binarize_pack", "had_attention", "had_dense_reference_mode", "had_scores_int",
                 "had_topn_indices", "had_attention_codes_u8", "had_get_device_status", "had_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared_functions():
        assert hasattr(L, name), f"missing export {name}"


def _shape(m, B=1, H=1, n=64, d=64, dtype=1, seqlens=None):
    return m.had_shape(B, H, n, d, dtype, seqlens)


def test_host_validation_rejects_before_launch(L):
    import binarized_qk_sparse_b200 as m
    P = ctypes.c_void_p
    fake = P(0x10000)          # never dereferenced: every case fails validation first
    odd = P(0x10008)           # 8-byte aligned, not 16
    ws = P(0x20000)
    big = 1 << 30

    def att(shape, q=fake, k=fake, v=fake, o=fake, N=0, mode=0, ws_bytes=big, alpha=None, bias=None, wsp=ws):
        return L.had_attention(q, k, v, ctypes.byref(shape), bias, alpha, None, N, mode, o, 1, wsp, ws_bytes, None)

    assert att(_shape(m, d=32)) == m.HAD_ERR_UNSUPPORTED
    assert att(_shape(m, n=16385)) == m.HAD_ERR_UNSUPPORTED
    assert att(_shape(m, H=257)) == m.HAD_ERR_UNSUPPORTED
    assert att(_shape(m, B=0)) == m.HAD_ERR_INVALID
    assert att(_shape(m, n=0)) == m.HAD_ERR_INVALID
    assert att(_shape(m, dtype=7)) == m.HAD_ERR_INVALID
    assert att(_shape(m), N=-1) == m.HAD_ERR_INVALID
    assert att(_shape(m), mode=5) == m.HAD_ERR_INVALID
    assert att(_shape(m), mode=3) == m.HAD_ERR_INVALID
    assert att(_shape(m), q=P(0)) == m.HAD_ERR_INVALID
    assert att(_shape(m), v=odd) == m.HAD_ERR_INVALID
    assert att(_shape(m), o=P(0)) == m.HAD_ERR_INVALID
    assert att(_shape(m), ws_bytes=16) == m.HAD_ERR_INVALID
    assert att(_shape(m), wsp=P(0)) == m.HAD_ERR_INVALID
    assert att(_shape(m, seqlens=0x10002)) == m.HAD_ERR_INVALID
    neg = (ctypes.c_float * 1)(-1.0)
    assert att(_shape(m), alpha=ctypes.cast(neg, P)) == m.HAD_ERR_INVALID
    zero = (ctypes.c_float * 1)(0.0)
    assert att(_shape(m), alpha=ctypes.cast(zero, P)) == m.HAD_ERR_INVALID
    # bias grid must cover the sequence: gh*gw + prefix == n
    bad = m.had_relpos_bias(0x30000, 7, 7, 1)
    assert att(_shape(m), bias=ctypes.byref(bad)) == m.HAD_ERR_INVALID
    # dense comparison mode: bf16 only, dense only
    shp = _shape(m, dtype=0)
    assert L.had_dense_reference_mode(fake, fake, fake, ctypes.byref(shp), None, 0, fake, 1, None, 0, None) \
        == m.HAD_ERR_UNSUPPORTED
    shp = _shape(m)
    assert L.had_dense_reference_mode(fake, fake, fake, ctypes.byref(shp), None, 5, fake, 1, None, 0, None) \
        == m.HAD_ERR_UNSUPPORTED
    # with a bias it needs the workspace for the bias tables
    rb = m.had_relpos_bias(0x30000, 8, 8, 0)
    assert L.had_dense_reference_workspace_size(ctypes.byref(shp), ctypes.byref(rb)) > 0
    assert L.had_dense_reference_workspace_size(ctypes.byref(shp), None) == 0
    assert L.had_dense_reference_mode(fake, fake, fake, ctypes.byref(shp), ctypes.byref(rb), 0, fake, 1, None, 0,
                                      None) == m.HAD_ERR_INVALID
    # exports
    assert L.had_topn_indices(fake, fake, ctypes.byref(shp), None, None, None, 0, fake, ws, big, None) \
        == m.HAD_ERR_INVALID
    assert L.had_attention_codes_u8(fake, fake, fake, ctypes.byref(shp), None, None, None, 0, 5, 5, fake, ws, big,
                                    None) == m.HAD_ERR_INVALID
    assert L.had_binarize_pack(fake, ctypes.byref(shp), None, None, fake, P(0), 0, None) == m.HAD_ERR_INVALID


def test_workspace_size_grows_with_mode_and_bias(L):
    import binarized_qk_sparse_b200 as m
    shp = _shape(m, B=2, H=3, n=197)
    f = L.had_attention_workspace_size(ctypes.byref(shp), 0, 0, None)
    q = L.had_attention_workspace_size(ctypes.byref(shp), 0, 1, None)
    bias = m.had_relpos_bias(0x30000, 14, 14, 1)
    qb = L.had_attention_workspace_size(ctypes.byref(shp), 0, 1, ctypes.byref(bias))
    assert 0 < f < q < qb
    # 4-bit V: half the bytes of the int8 V^T (n_pad = 256 keys -> 128 bytes per channel row)
    q4 = L.had_attention_workspace_size(ctypes.byref(shp), 0, 2, None)
    assert f < q4 < q and q - q4 >= 2 * 3 * 64 * 128
    wide = _shape(m, B=2, H=3, n=197, d=128)   # head dim 128: twice the per-token intermediates
    assert L.had_attention_workspace_size(ctypes.byref(wide), 0, 1, None) > q
    bad = _shape(m, d=96)
    assert L.had_attention_workspace_size(ctypes.byref(bad), 0, 0, None) == 0


def test_four_bit_mode_is_the_output_path_only(L):
    # the index and code exports and the quantizer keep their own modes; the
    # 4-bit quantizer validates like the int8 one
    import binarized_qk_sparse_b200 as m
    P = ctypes.c_void_p
    fake = P(0x10000)
    shp = _shape(m)
    assert L.had_quantize_v4(P(0), ctypes.byref(shp), fake, fake, fake, 1 << 30, None) == m.HAD_ERR_INVALID
    assert L.had_quantize_v4(fake, ctypes.byref(shp), fake, P(0x10002), fake, 1 << 30, None) == m.HAD_ERR_INVALID
    assert L.had_quantize_v4(fake, ctypes.byref(shp), fake, fake, fake, 16, None) == m.HAD_ERR_INVALID
    bad = _shape(m, d=96)
    assert L.had_quantize_v4(fake, ctypes.byref(bad), fake, fake, fake, 1 << 30, None) == m.HAD_ERR_UNSUPPORTED
    assert m._MODES["u8i4"] == m.HAD_MODE_U8I4 == 2


def test_status_strings(L):
    import binarized_qk_sparse_b200 as m
    for st in range(6):
        assert L.had_status_string(st).startswith(b"HAD_")
    assert L.had_version() >= 100


def test_host_entry_point_validates_on_the_host(L):
    # every case fails before a stream or event is created or a byte is copied
    import binarized_qk_sparse_b200 as m
    P = ctypes.c_void_p
    fake = P(0x10000)
    ws = P(0x20000)
    big = 1 << 34

    def host(shape, q=fake, o=fake, N=0, mode=0, odt=1, chunk=0, ws_bytes=big, wsp=ws, alpha=None):
        return L.had_attention_host(q, fake, fake, ctypes.byref(shape), None, alpha, None, N, mode, o, odt, chunk,
                                    wsp, ws_bytes, None)

    shp = _shape(m, B=4, n=64)
    assert host(_shape(m, d=32)) == m.HAD_ERR_UNSUPPORTED
    assert host(shp, q=P(0)) == m.HAD_ERR_INVALID
    assert host(shp, o=P(0)) == m.HAD_ERR_INVALID
    assert host(shp, odt=9) == m.HAD_ERR_INVALID
    assert host(shp, N=-2) == m.HAD_ERR_INVALID
    assert host(shp, mode=3) == m.HAD_ERR_INVALID
    assert host(shp, chunk=-1) == m.HAD_ERR_INVALID
    assert host(shp, ws_bytes=1024) == m.HAD_ERR_INVALID
    assert host(shp, wsp=P(0x20008)) == m.HAD_ERR_INVALID
    neg = (ctypes.c_float * 1)(-1.0)
    assert host(shp, alpha=ctypes.cast(neg, P)) == m.HAD_ERR_INVALID
    # seqlens is a host array here, checked by value
    for bad in ([64, 0, 5, 5], [64, 65, 5, 5], [-1, 1, 1, 1]):
        lens = (ctypes.c_int32 * 4)(*bad)
        s2 = _shape(m, B=4, n=64, seqlens=ctypes.addressof(lens))
        assert host(s2) == m.HAD_ERR_INVALID
    bad_bias = m.had_relpos_bias(0x30000, 7, 7, 1)
    assert L.had_attention_host(fake, fake, fake, ctypes.byref(shp), ctypes.byref(bad_bias), None, None, 0, 0, fake,
                                1, 0, ws, big, None) == m.HAD_ERR_INVALID


def test_host_workspace_grows_with_the_chunk(L):
    import binarized_qk_sparse_b200 as m
    # B=16: four slots of 1 and of 2 sequences, two slots of 8
    shp = _shape(m, B=16, H=3, n=197)
    bias = m.had_relpos_bias(0x30000, 14, 14, 1)
    sizes = [L.had_attention_host_workspace_size(ctypes.byref(shp), 0, 1, ctypes.byref(bias), c) for c in (1, 2, 8)]
    assert 0 < sizes[0] < sizes[1] < sizes[2]
    # a chunk larger than the batch is the whole batch; 0 lets the library choose
    whole = L.had_attention_host_workspace_size(ctypes.byref(shp), 0, 1, ctypes.byref(bias), 16)
    assert L.had_attention_host_workspace_size(ctypes.byref(shp), 0, 1, ctypes.byref(bias), 100) == whole
    assert L.had_attention_host_workspace_size(ctypes.byref(shp), 0, 1, ctypes.byref(bias), 0) > 0
    assert L.had_attention_host_workspace_size(ctypes.byref(shp), 0, 1, ctypes.byref(bias), -1) == 0
    # four slots of one chunk each hold Q, K, V and O at least
    one = 3 * 197 * 64 * 2 + 197 * 64 * 4
    assert sizes[0] >= 4 * one


def test_host_workspace_of_head_groups(L):
    # B2 H8 n16384 bf16: 100 MB of inputs per sequence, more than one chunk holds, so chunk_b = 0 cuts each
    # sequence into groups of 2 heads (at most 16 MiB): four slots of 2 heads against two slots of 8
    import binarized_qk_sparse_b200 as m
    shp = _shape(m, B=2, H=8, n=16384)
    bias = m.had_relpos_bias(0x30000, 128, 128, 0)
    split = L.had_attention_host_workspace_size(ctypes.byref(shp), 0, 0, ctypes.byref(bias), 0)
    whole = L.had_attention_host_workspace_size(ctypes.byref(shp), 0, 0, ctypes.byref(bias), 1)
    head_in = 16384 * 64 * 2
    assert 0 < split < whole
    assert split >= 4 * 2 * (3 * head_in + 2 * head_in)  # Q, K, V and fp32 O of two heads in each of four slots


def test_dense_bias_matrix_validation(L):
    import binarized_qk_sparse_b200 as m
    P = ctypes.c_void_p
    fake = P(0x10000)
    ws = P(0x20000)
    big = 1 << 34

    def att(shape, bias):
        return L.had_attention(fake, fake, fake, ctypes.byref(shape), ctypes.byref(bias), None, None, 0, 0, fake, 1,
                               ws, big, None)

    shp = _shape(m, n=197)
    assert att(shp, m.had_relpos_bias(0x30000, 0, 0, 0, 2)) == m.HAD_ERR_INVALID     # unknown kind
    assert att(shp, m.had_relpos_bias(0x30002, 0, 0, 0, 1)) == m.HAD_ERR_INVALID     # misaligned table
    assert att(_shape(m, n=4097), m.had_relpos_bias(0x30000, 0, 0, 0, 1)) == m.HAD_ERR_UNSUPPORTED
    # the grid fields are ignored for a dense matrix; its tables take n * (n + 2) floats per head
    shp = _shape(m, B=2, H=3, n=197)
    rel = m.had_relpos_bias(0x30000, 14, 14, 1, 0)
    dense = m.had_relpos_bias(0x30000, 7, 7, 1, 1)
    wr = L.had_attention_workspace_size(ctypes.byref(shp), 0, 1, ctypes.byref(rel))
    wd = L.had_attention_workspace_size(ctypes.byref(shp), 0, 1, ctypes.byref(dense))
    assert wd > wr > 0
    assert wd - L.had_attention_workspace_size(ctypes.byref(shp), 0, 1, None) >= 2 * 3 * 197 * 198 * 4


def test_binding_marshals_both_bias_kinds_and_host_arrays(L):
    import torch
    import binarized_qk_sparse_b200 as m
    rel = m.RelPosBias(torch.zeros(3, 27, 27), 14, 14, 1)
    c = m._bias_c(rel)
    assert (c.gh, c.gw, c.prefix, c.dense) == (14, 14, 1, 0) and c.table == rel.table.data_ptr()
    dense = m.DenseBias(torch.zeros(3, 197, 197))
    c = m._bias_c(dense)
    assert (c.dense, c.table) == (1, dense.table.data_ptr())
    Q = torch.zeros(2, 3, 197, 64, dtype=torch.bfloat16)
    # host workspace sizes come from the host (no device needed); the dense tables are larger
    wr = m.had_attention_host_workspace_size(Q, 0, "u8i8", None, rel)
    wd = m.had_attention_host_workspace_size(Q, 0, "u8i8", None, dense)
    assert 0 < wr < wd
    # the host entry point takes contiguous CPU tensors only, checked before any call
    with pytest.raises(ValueError):
        m.had_attention_host(Q.transpose(2, 3), Q, Q)


def test_qkv_prepare_validates_on_the_host(L):
    # the fused projection takes bf16 at head dim 64 and a model width of a multiple of 64
    import binarized_qk_sparse_b200 as m
    P = ctypes.c_void_p
    fake, ws = P(0x10000), P(0x20000)
    big = 1 << 34

    def qkv(shape, Dm=256, x=fake, w=fake, v=fake, mode=0, ws_bytes=big, wsp=ws, N=0):
        return L.had_qkv_prepare(x, w, ctypes.byref(shape), Dm, None, N, mode, v, wsp, ws_bytes, None)

    shp = _shape(m, B=2, H=3, n=197)
    assert qkv(_shape(m, d=128)) == m.HAD_ERR_UNSUPPORTED
    assert qkv(_shape(m, dtype=0)) == m.HAD_ERR_UNSUPPORTED      # fp32 X
    assert qkv(shp, Dm=100) == m.HAD_ERR_INVALID
    assert qkv(shp, Dm=0) == m.HAD_ERR_INVALID
    assert qkv(shp, Dm=16384 + 64) == m.HAD_ERR_UNSUPPORTED
    assert qkv(shp, x=P(0)) == m.HAD_ERR_INVALID
    assert qkv(shp, w=P(0x10008)) == m.HAD_ERR_INVALID
    assert qkv(shp, v=P(0)) == m.HAD_ERR_INVALID
    assert qkv(shp, mode=7) == m.HAD_ERR_INVALID
    assert qkv(shp, N=-1) == m.HAD_ERR_INVALID
    assert qkv(shp, ws_bytes=1024) == m.HAD_ERR_INVALID
    # its workspace holds the attention workspace plus X's token sums and the means
    att = L.had_attention_workspace_size(ctypes.byref(shp), 0, 1, None)
    q = L.had_qkv_workspace_size(ctypes.byref(shp), 256, 0, 1, None)
    assert q >= att + 2 * 256 * 8 + 2 * 2 * 3 * 64 * 4
    assert L.had_qkv_workspace_size(ctypes.byref(_shape(m, d=128)), 256, 0, 1, None) == 0
