"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/svg.h declares, sizes its scratch, and rejects bad arguments on the
host before launching anything (the fake device pointers below are never
dereferenced)."""
import ctypes as C
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svg.h")

from sparse_attention_video_svg_b200 import _lib  # noqa: E402

L = _lib.lib
FAKE = 1 << 20          # 16-byte aligned, never dereferenced on the host
FAKE2 = 2 << 20
FAKE3 = 3 << 20
FAKE4 = 4 << 20


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svg_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
        assert n in _lib.SIGNATURES, f"{n} has no ctypes signature"
    assert set(_lib.SIGNATURES) == set(names)


def test_exported_dynamic_symbols_match_header():
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    exported = set(re.findall(r" T (svg_[a-z_0-9]+)", out))
    assert exported == set(declared_functions())


def test_version():
    assert L.svg_version().decode().startswith("svg_b200")


def test_wait_limit_setting_round_trip():
    default = L.svg_get_wait_limit()
    assert default == 1 << 22
    try:
        assert L.svg_set_wait_limit(7) == _lib.SVG_OK
        assert L.svg_get_wait_limit() == 7
    finally:
        assert L.svg_set_wait_limit(0) == _lib.SVG_OK  # 0 restores the default
    assert L.svg_get_wait_limit() == default


def test_workspace_sizes():
    assert L.svg_profile_workspace_size(1, 48, 17550, 64, 64) > 0
    assert L.svg_profile_workspace_size(1, 48, 17550, 64, 64) % 256 == 0
    assert L.svg_profile_workspace_size(1, 48, 17550, 96, 64) == 0
    assert L.svg_block_energy_workspace_size(1, 40, 75600) >= 40 * 75600 * 4
    assert L.svg_calibrated_workspace_size(40, 591, 591) >= 40 * 591 * 19 * 4
    assert L.svg_calibrated_workspace_size(0, 1, 1) == 0


def expect(status, fn, *args, match=None):
    st = getattr(L, fn)(*args)
    assert st == status, (fn, st, L.svg_last_error())
    if match:
        assert match in L.svg_last_error().decode()


INVALID = _lib.SVG_ERR_INVALID_ARG


class TestHostValidation:
    def test_sparse_attn(self):
        base = [FAKE, FAKE2, FAKE3, FAKE4 * 4, 0, 1, 2, 256, 64, FAKE, 3, 2, FAKE, FAKE, 0.0, None,
                None, None]
        expect(_lib.SVG_OK if False else INVALID, "svg_sparse_attn",
               *(base[:8] + [96] + base[9:]), match="d=96")
        expect(INVALID, "svg_sparse_attn", *(base[:11] + [3] + base[12:]), match="n_qblocks")
        expect(INVALID, "svg_sparse_attn", *([FAKE + 8] + base[1:]), match="aligned")
        expect(INVALID, "svg_sparse_attn", *(base[:3] + [FAKE] + base[4:]), match="overlaps")
        expect(INVALID, "svg_sparse_attn", *(base[:4] + [7] + base[5:]), match="dtype")
        expect(INVALID, "svg_sparse_attn", *(base[:14] + [-1.0] + base[15:]), match="scale")
        expect(INVALID, "svg_sparse_attn", *([None] + base[1:]), match="null")

    def test_sparse_attn_fused(self):
        # q k v q_tm k_tm v_tm o dtype B H N d F P mode layout n_lists n_qblocks indptr
        # indices tile_order scale status v_exp stream
        base = [FAKE, FAKE2, FAKE3, None, None, None, FAKE4 * 4, 0, 1, 2, 256, 64, 4, 64, FAKE,
                3, 3, 2, FAKE, FAKE, None, 0.0, None, None, None]
        expect(INVALID, "svg_sparse_attn_fused", *(base[:12] + [5] + base[13:]), match="frames")
        expect(INVALID, "svg_sparse_attn_fused", *(base[:11] + [96] + base[12:]), match="d=96")
        expect(INVALID, "svg_sparse_attn_fused", *(base[:14] + [None] + base[15:]), match="null")
        expect(INVALID, "svg_sparse_attn_fused", *(base[:6] + [FAKE] + base[7:]), match="overlaps")
        expect(INVALID, "svg_sparse_attn_fused", *(base[:15] + [4] + base[16:]), match="layout")
        expect(INVALID, "svg_sparse_attn_fused", *(base[:3] + [FAKE4 * 5] + base[4:]),
               match="all three")
        expect(INVALID, "svg_sparse_attn_fused",
               *(base[:3] + [FAKE4 * 5, FAKE4 * 6, FAKE4 * 7] + base[6:15] + [1] + base[16:]),
               match="exclude")

    def test_qk_norm_rope(self):
        # q k q_out k_out q_tm k_tm dtype B H N d F P ops gamma_q gamma_k eps cos sin stream
        both = _lib.SVG_QK_NORM | _lib.SVG_QK_ROPE
        base = [FAKE, FAKE2, FAKE3, FAKE4, FAKE4 * 2, FAKE4 * 3, 0, 1, 2, 256, 64, 4, 64, both,
                FAKE4 * 4, None, 1e-6, FAKE4 * 5, FAKE4 * 6, None]
        f = "svg_qk_norm_rope"
        expect(INVALID, f, *(base[:13] + [4] + base[14:]), match="bad ops")
        expect(INVALID, f, *(base[:16] + [-1.0] + base[17:]), match="eps")
        expect(INVALID, f, *(base[:17] + [None] + base[18:]), match="cos and sin")
        expect(INVALID, f, *(base[:5] + [None] + base[6:]), match="both token-major")
        expect(INVALID, f, *(base[:11] + [5] + base[12:]), match="frames")
        expect(INVALID, f, *(base[:2] + [FAKE2] + base[3:]), match="overlap")
        expect(INVALID, f, *(base[:4] + [FAKE3 + 4096] + base[5:]), match="token-major outputs")
        expect(INVALID, f, *(base[:14] + [FAKE4 * 4 + 4] + base[15:]), match="aligned")
        expect(INVALID, f, *(base[:10] + [96] + base[11:]), match="d=96")
        expect(INVALID, f, *(base[:6] + [3] + base[7:]), match="dtype")
        expect(INVALID, f, *([None] + base[1:]), match="null")

    def test_repetition(self):
        ws = L.svg_row_similarity_workspace_size(0, 1, 2, 4, 16, 2)
        assert ws > 0
        # q k dtype B H N d frames rows cols eval_frames n_frames sim ws ws_bytes status stream
        base = [FAKE, FAKE2, 0, 1, 2, 256, 64, 4, 4, 16, None, 2, FAKE3, FAKE4 * 2, ws, None, None]
        f = "svg_row_similarity"
        expect(INVALID, f, *(base[:8] + [5] + base[9:]), match="!= N")
        expect(INVALID, f, *(base[:7] + [256, 1, 1] + base[10:]), match="rows=1")
        expect(INVALID, f, *(base[:11] + [5] + base[12:]), match="n_frames")
        expect(INVALID, f, *(base[:14] + [ws - 256] + base[15:]), match="workspace")
        expect(INVALID, f, *(base[:6] + [32] + base[7:]), match="d=32")
        # n_lists nqb indptr indices N frames rows cols anchors list_id repeat n_heads skip
        # out_indptr out_indices capacity list_id_out tile_order_out status stream
        base = [3, 2, FAKE, FAKE2, 256, 4, 4, 16, 5, FAKE3, None, 2, 1, FAKE4, FAKE4 * 2, 100,
                FAKE4 * 3, None, None, None]
        f = "svg_anchor_lists"
        expect(INVALID, f, *(base[:1] + [3] + base[2:]), match="n_qblocks")
        expect(INVALID, f, *(base[:8] + [0] + base[9:]), match="anchors")
        expect(INVALID, f, *(base[:15] + [0] + base[16:]), match="capacity")
        expect(INVALID, f, *(base[:6] + [5] + base[7:]), match="!= N")
        expect(INVALID, f, *(base[:2] + [None] + base[3:]), match="null")
        # list_id given without list_id_out
        expect(INVALID, f, *(base[:16] + [None] + base[17:]), match="null")
        expect(INVALID, "svg_anchor_list_ids", FAKE, None, 0, 3, 1, FAKE2, None, match="sizes")
        expect(INVALID, "svg_anchor_list_ids", FAKE, None, 4, 3, 1, None, None, match="null")
        # o dtype B H N d frames rows cols anchors list_id n_lists stream
        base = [FAKE, 0, 1, 2, 256, 64, 4, 4, 16, 5, FAKE2, 3, None]
        f = "svg_row_broadcast"
        expect(INVALID, f, *(base[:7] + [5] + base[8:]), match="!= N")
        expect(INVALID, f, *(base[:11] + [0] + base[12:]), match="n_lists")
        expect(INVALID, f, *([FAKE + 8] + base[1:]), match="aligned")

    def test_pair_query_tiles(self):
        f = "svg_pair_query_tiles"
        ws = L.svg_pair_query_tiles_workspace_size(2, 5, 5)
        assert ws == 2 * 5 * 1 * 4 and L.svg_pair_query_tiles_workspace_size(0, 5, 5) == 0
        # indptr indices lists rows blocks order status ws ws_bytes stream
        base = [FAKE, FAKE2, 2, 5, 5, FAKE3, None, FAKE4, ws, None]
        expect(INVALID, f, *([None] + base[1:]), match="null")
        expect(INVALID, f, *(base[:3] + [0] + base[4:]), match="bad sizes")
        expect(INVALID, f, *(base[:8] + [ws - 4] + base[9:]), match="workspace")
        expect(INVALID, f, *(base[:3] + [60000, 10 ** 6] + base[5:8]
                             + [L.svg_pair_query_tiles_workspace_size(2, 60000, 10 ** 6)] + base[9:]),
               match="limit")

    def test_permute(self):
        args = [FAKE, FAKE4 * 4, 0, 1, 2, 12, 64, 3, 4, None, None]
        expect(INVALID, "svg_permute_token_major", *(args[:7] + [5] + args[8:]), match="!= N")
        expect(INVALID, "svg_permute_frame_major", *([FAKE, FAKE + 64] + args[2:]), match="overlap")
        expect(INVALID, "svg_permute_token_major", *(args[:6] + [32] + args[7:]), match="d=32")
        # the temporal-only copy needs the modes, and checks shapes like the others
        expect(INVALID, "svg_permute_temporal_heads", *args, match="mode is required")
        expect(INVALID, "svg_permute_temporal_heads", *(args[:7] + [5] + args[8:9] + [FAKE] + args[10:]),
               match="!= N")

    def test_profile(self):
        ws = L.svg_profile_workspace_size(1, 2, 256, 64, 16)
        args = [FAKE, FAKE2, FAKE3, 1, 1, 2, 256, 64, 4, 64, 1, FAKE, 16, None, FAKE4, FAKE4 * 2,
                ws, None]
        expect(INVALID, "svg_profile_heads", *(args[:12] + [65] + args[13:]), match="S=65")
        expect(INVALID, "svg_profile_heads", *(args[:16] + [ws - 256] + args[17:]),
               match="workspace")
        expect(INVALID, "svg_profile_heads", *(args[:10] + [-1] + args[11:]),
               match="spatial_width")

    def test_block_masks(self):
        expect(INVALID, "svg_build_block_mask", 7, 3, 4, 1, 12, FAKE, FAKE2, 1, 0, FAKE3, None,
               None, match="kind")
        expect(INVALID, "svg_build_block_mask", 0, 3, 4, 1, 13, FAKE, FAKE2, 1, 0, FAKE3, None,
               None, match="!= N")
        expect(_lib.SVG_ERR_UNSUPPORTED, "svg_build_block_mask", 0, 3, 4, 1, 12, FAKE, FAKE2, 1,
               0x7fffffff, FAKE3, None, None)
        ws = L.svg_calibrated_workspace_size(2, 3, 3)
        expect(INVALID, "svg_build_block_mask_calibrated", FAKE, 17, 2, 3, 3, C.c_double(0.9),
               C.c_double(0.5), FAKE2, FAKE3, 18, FAKE4, None, FAKE4 * 2, ws, None, match="R=17")
        expect(INVALID, "svg_build_block_mask_calibrated", FAKE, 2, 2, 3, 3, C.c_double(0.9),
               C.c_double(1.5), FAKE2, FAKE3, 18, FAKE4, None, FAKE4 * 2, ws, None, match="rho")
        expect(INVALID, "svg_build_block_mask_calibrated", FAKE, 2, 2, 3, 5000, C.c_double(0.9),
               C.c_double(0.5), FAKE2, FAKE3, 18, FAKE4, None, FAKE4 * 2, ws, None, match="nKB")

    def test_block_energy(self):
        expect(INVALID, "svg_block_energy", FAKE, FAKE2, 0, 1, 2, 256, 64, FAKE3, FAKE4 * 2, 10,
               None, match="workspace")


def test_epsilon_schedule_host_matches_oracle():
    """svg_epsilon_schedule runs on the host: same values as the oracle's
    schedule (libm pow against NumPy's, a few ulp at most)."""
    import ctypes as C

    from oracle import svg_oracle as O
    for n, a, b in ((50, 0.99, 0.84), (1, 0.99, 0.84), (7, 0.95, 0.5), (2, 1.0, 0.9)):
        out = (C.c_double * n)()
        assert L.svg_epsilon_schedule(n, a, b, C.cast(out, C.c_void_p)) == _lib.SVG_OK
        np.testing.assert_allclose(list(out), O.epsilon_schedule(n, a, b), rtol=4e-16)
    out = (C.c_double * 1)()
    assert L.svg_epsilon_schedule(3, 1.5, 0.8, C.cast(out, C.c_void_p)) == INVALID
    assert L.svg_epsilon_schedule(-1, 0.9, 0.8, C.cast(out, C.c_void_p)) == INVALID


def test_encoding_validation():
    expect(INVALID, "svg_lists_to_intervals", 0, 10, FAKE, FAKE2, FAKE3, FAKE4, FAKE4 * 2, 8,
           FAKE4 * 3, None, None, match="bad sizes")
    expect(INVALID, "svg_lists_to_intervals", 3, 10, FAKE, FAKE2, FAKE3, None, None, 8,
           FAKE4 * 3, None, None, match="null starts")
    expect(INVALID, "svg_lists_to_bitmap", 3, 0, FAKE, FAKE2, FAKE3, None, None, match="bad sizes")
    expect(INVALID, "svg_lists_to_bitmap", 3, 10, FAKE, None, FAKE3, None, None, match="null")


def test_layer_argument_checks_before_any_launch():
    # these raise in the binding before anything reaches the library or a GPU
    import torch
    import sparse_attention_video_svg_b200 as svg
    q = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16)
    lists = svg.BlockLists(torch.zeros(3 * 3, dtype=torch.int32),
                           torch.zeros(1, dtype=torch.int32), 3, 2)
    idx = torch.zeros(16, dtype=torch.int32)
    bufs = svg.LayerBuffers(q, 16)
    qk = svg.QKTransform(None, None, 1e-6, None, None)
    with pytest.raises(ValueError, match="qk=True"):
        svg.svg_layer(q, q, q, 4, 64, 1, idx, lists, bufs, qk=qk)
    with pytest.raises(ValueError, match="frame_shape"):
        svg.svg_layer(q, q, q, 4, 64, 1, idx, lists, bufs,
                      repeat=torch.ones(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="frame_shape"):
        svg.svg_layer(q, q, q, 4, 64, 1, idx, lists, bufs,
                      repeat=torch.ones(2, dtype=torch.int32), frame_shape=(8, 9))
