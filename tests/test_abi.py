"""The C-ABI library loads on any host and exports every entry point include/hiera.h
declares; host-side argument checks and size queries need no GPU."""

import ctypes

import pytest

from mask_unit_windowed_b200 import binding as hb


def test_library_exports_every_header_symbol():
    names = hb.header_symbols()
    assert len(names) >= 17
    L = hb.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert missing == []


def test_status_strings():
    for code, name in hb.STATUS.items():
        assert hb.status_string(code) == name


def test_null_arguments_rejected_before_any_launch():
    L = hb.lib()
    assert L.hiera_unroll(None, None, 1, 8, 112, 3, hb.HIERA_BF16, None) == 1
    assert L.hiera_linear(None, None, None, None, None, 4, 16, 16, hb.HIERA_BF16, None) == 1
    d = hb.BlockDesc(B=1, tokens=1024, dim_in=112, dim_out=112, heads=2).c()
    assert L.hiera_block_forward(ctypes.byref(d), None, None, None, None, 0, None) == 1


def test_bad_shapes_and_dtypes_rejected():
    L = hb.lib()
    fake = ctypes.c_void_p(1 << 20)
    assert L.hiera_unroll(fake, ctypes.c_void_p(2 << 20), 1, 12, 112, 3, hb.HIERA_BF16, None) == 2
    assert L.hiera_unroll(fake, ctypes.c_void_p(2 << 20), 1, 8, 112, 3, 7, None) == 3
    assert L.hiera_unroll(ctypes.c_void_p((1 << 20) + 8), ctypes.c_void_p(2 << 20), 1, 8, 112, 3,
                          hb.HIERA_BF16, None) == 4
    for bad in (dict(head_dim=64), dict(heads=3), dict(q_stride=2),
                dict(window_tokens=48), dict(dim_in=120)):
        kw = dict(B=1, tokens=1024, dim_in=112, dim_out=112, heads=2)
        kw.update(bad)
        d = hb.BlockDesc(**kw)
        if "heads" in bad:
            d.dim_out = 56 * d.heads
        assert L.hiera_block_workspace_bytes(ctypes.byref(d.c())) == 0, bad


def test_no_gpu_means_device_error_not_fallback():
    """Without an sm_100 device a well-formed call fails with HIERA_ERR_DEVICE."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    L = hb.lib()
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(2 << 20)
    assert L.hiera_unroll(a, b, 1, 8, 112, 3, hb.HIERA_BF16, None) == 8


def test_workspace_and_pack_sizes():
    d = hb.BlockDesc(B=4, tokens=16384, dim_in=112, dim_out=224, heads=4, q_stride=4,
                     window_tokens=64)
    ws = hb.block_workspace_bytes(d)
    offs = hb.block_workspace_layout(d)
    # q [4,256,4,16,64], k/v [4,256,4,64,64] bf16, merged o / r / x1 [4,4096,224], h [4,4096,896]
    q = 4 * 256 * 4 * 16 * 64 * 2
    kv = 4 * 256 * 4 * 64 * 64 * 2
    assert offs[0] == 0 and offs[1] >= q and offs[2] - offs[1] >= kv
    assert offs[4] > 0 and offs[6] > offs[5]
    assert ws >= offs[6] + 4 * 4096 * 896 * 2
    pk = hb.block_packed_bytes(d)
    assert pk >= (4 * 224 * 112 + 224 * 224 + 2 * 896 * 224) * 2
    bb = hb.BackboneDesc(B=1, img=512)
    assert hb.backbone_packed_bytes(bb) > 2 * 69_000_000
    assert hb.backbone_workspace_bytes(bb) > 2 * 16384 * 112 * 2


def test_attention_entry_rejects_bad_arguments_before_any_launch():
    L = hb.lib()
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(2 << 20)
    assert L.hiera_attention(None, a, a, b, 1, 1, 1, 64, 64, None) == 1
    assert L.hiera_attention(a, a, a, b, 0, 1, 1, 64, 64, None) == 1
    assert L.hiera_attention(a, a, a, b, 1, 1, 1, 64, 0, None) == 1
    misaligned = ctypes.c_void_p((1 << 20) + 8)
    assert L.hiera_attention(a, misaligned, a, b, 1, 1, 1, 64, 64, None) == 4
    assert L.hiera_attention(a, a, a, b, 1 << 16, 1 << 10, 8, 64, 64, None) == 2


def test_static_scratch_size_matches_header():
    """The binding reads the scratch size from the library; it must equal the header's
    HIERA_STATIC_SCRATCH_BYTES, so tests of the size limit test the real boundary."""
    import re
    with open(hb.HEADER) as f:
        m = re.search(r"#define HIERA_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", f.read())
    assert m is not None
    assert hb.static_scratch_bytes() == int(m.group(1)) << int(m.group(2))


def test_binding_rejects_mismatched_tensors_before_any_launch():
    """Shapes and dtypes are compared with the descriptor before the C call: a tensor that
    does not match would otherwise be read or written past its end."""
    import torch
    d = hb.BlockDesc(B=2, tokens=256, dim_in=112, dim_out=112, heads=2)
    packed = torch.empty(hb.block_packed_bytes(d), dtype=torch.uint8)
    with pytest.raises(ValueError, match="shape"):
        hb.block_forward(d, packed, torch.empty(2, 128, 112, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="dtype"):
        hb.block_forward(d, packed, torch.empty(2, 256, 112, dtype=torch.float32))
    with pytest.raises(ValueError, match="shape"):
        hb.block_forward_noalloc(d, packed, torch.empty(2, 256, 112, dtype=torch.bfloat16),
                                 out=torch.empty(2, 256, 224, dtype=torch.bfloat16))
    bb = hb.BackboneDesc(B=1, img=64)
    with pytest.raises(ValueError, match="shape"):
        hb.backbone_forward(bb, packed, torch.empty(1, 64, 64, 3, dtype=torch.bfloat16))
    q = torch.empty(1, 4, 2, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="shape"):
        hb.attention(q, torch.empty(1, 4, 2, 64, 56, dtype=torch.bfloat16), q)
    with pytest.raises(ValueError, match="shape"):
        hb.unroll(torch.empty(1, 60, 112, dtype=torch.bfloat16), 8, 3)
    with pytest.raises(ValueError, match="shape"):
        hb.linear(torch.empty(4, 16, dtype=torch.bfloat16),
                  torch.empty(32, 8, dtype=torch.bfloat16))
    # shapes right, but host tensors: still refused before the library is called
    with pytest.raises(ValueError, match="CUDA"):
        hb.block_forward(d, packed, torch.empty(2, 256, 112, dtype=torch.bfloat16))


def test_option_defaults_and_range():
    """Library options are host state: fused MLP, programmatic launch, the fused attention
    half and the split batch default on, the 224-column GEMMs on the eight-warp kernel;
    unknown options and values are rejected."""
    assert [hb.get_option(o) for o in (hb.OPT_FUSED_MLP, hb.OPT_PDL, hb.OPT_FUSED_ATTN,
                                       hb.OPT_GEMM224, hb.OPT_SPLIT_BATCH)] == [1, 1, 1, 0, 1]
    L = hb.lib()
    assert L.hiera_set_option(5, 1) == 1
    assert L.hiera_set_option(hb.OPT_SPLIT_BATCH, 2) == 1
    with hb.split_batch(False):
        assert hb.get_option(hb.OPT_SPLIT_BATCH) == 0
    assert hb.get_option(hb.OPT_SPLIT_BATCH) == 1
    assert L.hiera_set_option(hb.OPT_GEMM224, 3) == 1
    assert L.hiera_set_option(hb.OPT_PDL, 2) == 1
    for mode in (hb.GEMM224_SIXTEEN_WARPS, hb.GEMM224_PAIR):
        with hb.gemm224(mode):
            assert hb.get_option(hb.OPT_GEMM224) == mode
    assert hb.get_option(hb.OPT_GEMM224) == 0
