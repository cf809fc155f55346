"""GPU parity: every step of the CUDA path, called through the C ABI, against
the float64 CPU oracle on the same seeded inputs.

Small workloads (seconds of oracle time, several tiles and a ragged tail) are
compared element by element; full-size workloads on sampled query tiles, in
the launch configuration bench.py times.  Integer and data-movement results
are bit-exact; floating-point outputs meet max-abs 2e-2 and rel-RMS 1e-2."""
import numpy as np
import pytest
import torch

import svg_inputs as si
from oracle import svg_oracle as O
from tests.helpers import (MAX_ABS, MODE_MARGIN, assert_close, bits, half_ulp_bf16, to_device,
                           to_float64, workload_tensors)

pytestmark = pytest.mark.gpu

svg = pytest.importorskip("sparse_attention_video_svg_b200")
DEV = "cuda"

SMALL = [si.small(n) for n in si.ORDER]
FULL_BF16 = ["cogvideox", "wan480", "wan720", "hunyuan720"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def head64(x, b, h):
    return si.as_float64(x[b, h])


def tile_rows_kept_keys(q, k, v, t, N, indptr, indices):
    """The oracle's block-sparse rows of query tile t (O8), with the softmax
    taken over the kept key columns only: the columns of the tile's kept key
    tiles are gathered and the oracle's masked attention runs on them with
    every gathered key kept -- the same restricted softmax, without scoring
    the N - |kept| masked keys (thousands of tiles at full size)."""
    rows = O.tile_rows(int(t), N)
    cols = np.concatenate([np.arange(j * 128, min(N, (j + 1) * 128))
                           for j in indices[indptr[t]:indptr[t + 1]]] or [np.zeros(0, np.int64)])
    if cols.size == 0:
        return rows, np.zeros((len(rows), q.shape[1]))
    mask = np.ones((len(rows), cols.size), dtype=bool)
    return rows, O.masked_attention(q[rows], k[cols], v[cols], mask)


# --------------------------------------------------------------------- lists

def gpu_list(kind, F, P, w, N):
    ip, ix, nnz = svg.svg_build_block_mask(kind, F, P, w, N)
    n = int(nnz.item())
    return ip.cpu().numpy(), ix[:n].cpu().numpy()


@pytest.mark.parametrize("F,P,w", [(4, 64, 1), (13, 1350, 1), (21, 1560, 1), (21, 3600, 1),
                                   (33, 3600, 2), (5, 130, 1), (1, 300, 1), (300, 1, 1),
                                   (7, 3, 0), (2, 61, 3), (6, 126, 1)])
def test_geometric_lists_bit_exact(F, P, w):
    N = F * P
    for kind in (O.MODE_SPATIAL, O.MODE_TEMPORAL, O.MODE_DENSE):
        gp, gx = gpu_list(kind, F, P, w, N)
        op, ox = O.geometric_block_lists(kind, F, P, w, N)
        np.testing.assert_array_equal(gp, op)
        np.testing.assert_array_equal(gx, ox)


def test_geometric_lists_shared_buffer_offsets():
    F, P, w = 5, 130, 1
    N = F * P
    nb = svg.n_tiles(N)
    L = svg.geometric_lists(F, P, w, N)
    ip = L.indptr.cpu().numpy().reshape(3, nb + 1)
    ix = L.indices.cpu().numpy()
    for kind in range(3):
        op, ox = O.geometric_block_lists(kind, F, P, w, N)
        np.testing.assert_array_equal(ip[kind] - ip[kind][0], op)
        np.testing.assert_array_equal(ix[ip[kind][0]:ip[kind][-1]], ox)


# --------------------------------------------------------------- permutation

@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_permute_small_bit_exact(wl):
    (q, _, _), (qd, _, _), types = workload_tensors(wl)
    mode = torch.from_numpy(types).to(DEV)
    F, P = wl.F, wl.P
    y = svg.svg_permute_token_major(qd, F, P, mode)
    want = q.copy()
    for b in range(wl.B):
        for h in range(wl.H):
            if types[h] == si.TEMPORAL_TYPE:
                want[b, h] = O.permute_token_major(q[b, h], F, P)
    np.testing.assert_array_equal(bits(y), want.view(np.int16 if q.dtype == np.uint16 else np.int32))
    back = svg.svg_permute_frame_major(y, F, P, mode)
    assert torch.equal(bits_t(back), bits_t(qd))
    yall = svg.svg_permute_token_major(qd, F, P, None)
    np.testing.assert_array_equal(bits(yall), O.permute_token_major(q, F, P).view(bits(yall).dtype))


def bits_t(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_permute_temporal_heads_bit_exact(wl):
    """Temporal heads: the token-major rows; every other head of the output
    keeps what was there (a sentinel pattern), untouched."""
    (q, _, _), (qd, _, _), types = workload_tensors(wl)
    mode = torch.from_numpy(types).to(DEV)
    F, P = wl.F, wl.P
    y = torch.empty_like(qd)
    bits_t(y).fill_(0x5a5a)
    sentinel = bits(y).copy()
    svg.svg_permute_temporal_heads(qd, F, P, mode, out=y)
    yb = bits(y)
    for b in range(wl.B):
        for h in range(wl.H):
            if types[h] == si.TEMPORAL_TYPE:
                want = O.permute_token_major(q[b, h], F, P)
                np.testing.assert_array_equal(yb[b, h], want.view(yb.dtype))
            else:
                np.testing.assert_array_equal(yb[b, h], sentinel[b, h])
    assert (types == si.TEMPORAL_TYPE).any() and (types != si.TEMPORAL_TYPE).any()


@pytest.mark.parametrize("F,P,d,dt", [(1, 77, 64, "bf16"), (77, 1, 128, "bf16"), (3, 5, 128, "fp32"),
                                      (9, 13, 64, "fp32")])
def test_permute_edge_shapes(F, P, d, dt):
    rng = np.random.default_rng(F * 1000 + P)
    N = F * P
    if dt == "bf16":
        x = rng.integers(0, 1 << 16, size=(2, 3, N, d), dtype=np.uint16)
    else:
        x = rng.standard_normal((2, 3, N, d), dtype=np.float32)
    xd = to_device(x)
    y = svg.svg_permute_token_major(xd, F, P)
    np.testing.assert_array_equal(bits(y), O.permute_token_major(x, F, P).view(bits(y).dtype))
    z = svg.svg_permute_frame_major(xd, F, P)
    np.testing.assert_array_equal(bits(z), O.permute_frame_major(x, F, P).view(bits(z).dtype))


@pytest.mark.parametrize("name", FULL_BF16)
def test_permute_full_size_sampled(name):
    wl = si.WORKLOADS[name]
    F, P, N, d = wl.F, wl.P, wl.N, wl.d
    H = 4  # the per-head map is independent of H; 4 heads keep host memory small
    rng = np.random.default_rng(7)
    x = rng.integers(0, 1 << 16, size=(1, H, N, d), dtype=np.uint16)
    xd = to_device(x)
    mode = torch.tensor([1, 0, 1, 1], dtype=torch.int32, device=DEV)
    y = svg.svg_permute_token_major(xd, F, P, mode)
    yb = bits(y)
    src = O.token_major_source(F, P)
    rows = rng.choice(N, size=4096, replace=False)
    for h in range(H):
        s = src[rows] if h != 1 else rows
        np.testing.assert_array_equal(yb[0, h, rows], x[0, h, s].view(np.int16))
    back = svg.svg_permute_frame_major(y, F, P, mode)
    assert torch.equal(bits_t(back), bits_t(xd))


# ------------------------------------------------------------------ profiling

def check_profile(mse_gpu, mode_gpu, mse_ref, mode_ref, what):
    mse_gpu = np.asarray(mse_gpu, np.float64)
    for i in range(len(mode_ref)):
        for c in range(2):
            r = mse_ref[i, c]
            assert abs(mse_gpu[i, c] - r) <= 0.02 * r + 2e-5, (what, i, c, mse_gpu[i], mse_ref[i])
        margin = abs(mse_ref[i, 0] - mse_ref[i, 1]) / max(mse_ref[i].max(), 1e-30)
        if margin > MODE_MARGIN:
            assert mode_gpu[i] == mode_ref[i], (what, i, mse_gpu[i], mse_ref[i])


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_profile_small(wl):
    (q, k, v), (qd, kd, vd), types = workload_tensors(wl)
    idx = si.sample_queries(wl)
    mse, mode = svg.svg_profile_heads(qd, kd, vd, wl.F, wl.P, wl.width,
                                      torch.from_numpy(idx).to(DEV))
    mse_ref, mode_ref = O.profile_heads(si.as_float64(q), si.as_float64(k), si.as_float64(v), idx,
                                        wl.F, wl.P, wl.width)
    check_profile(mse.cpu().numpy(), mode.cpu().numpy(), mse_ref, mode_ref, wl.name)
    np.testing.assert_array_equal(mode.cpu().numpy(), types)


# bf16 profiling shapes at the edges of the tiled pass: padded sample rows
# (S < 64), a single frame, a band wider than the clip (spatial = dense), a
# ragged last tile, keys of a single tile, B > 1, and both head dims
PROFILE_EDGES = [
    si.WORKLOADS["hunyuan720"].scaled("edge-s5", H=2, F=6, ph=5, pw=7, S=5),          # N = 210
    si.WORKLOADS["cogvideox"].scaled("edge-one-frame", H=3, F=1, ph=9, pw=15, S=64),  # N = 135
    si.WORKLOADS["wan480"].scaled("edge-wide-band", H=2, F=3, ph=6, pw=10, width=5),  # N = 180
    si.WORKLOADS["wan480"].scaled("edge-one-tile", H=2, F=4, ph=4, pw=7, S=17),       # N = 112
    si.WORKLOADS["cogvideox"].scaled("edge-b2", B=2, H=2, F=5, ph=7, pw=9, S=33),     # N = 315
]


@pytest.mark.parametrize("wl", PROFILE_EDGES, ids=lambda w: w.name)
def test_profile_edges(wl):
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    idx = si.sample_queries(wl)
    mse, mode = svg.svg_profile_heads(qd, kd, vd, wl.F, wl.P, wl.width,
                                      torch.from_numpy(idx).to(DEV))
    mse_ref, mode_ref = O.profile_heads(si.as_float64(q), si.as_float64(k), si.as_float64(v), idx,
                                        wl.F, wl.P, wl.width)
    check_profile(mse.cpu().numpy(), mode.cpu().numpy(), mse_ref, mode_ref, wl.name)
    if wl.width >= wl.F - 1:
        # every key in the band: the spatial output is the dense one
        assert np.all(mse.cpu().numpy()[:, 0] <= 1e-6)


@pytest.fixture(scope="module")
def full_inputs():
    cache = {}

    def get(name):
        if name not in cache:
            cache.clear()
            wl = si.WORKLOADS[name]
            cache[name] = workload_tensors(wl)
        return cache[name]
    return get


@pytest.mark.parametrize("name", ["cogvideox", "hunyuan720"])
def test_profile_full_size(name, full_inputs):
    wl = si.WORKLOADS[name]
    (q, k, v), (qd, kd, vd), types = full_inputs(name)
    idx = si.sample_queries(wl)
    mse, mode = svg.svg_profile_heads(qd, kd, vd, wl.F, wl.P, wl.width,
                                      torch.from_numpy(idx).to(DEV))
    mse = mse.cpu().numpy()
    mode = mode.cpu().numpy()
    heads = range(wl.H) if wl.H <= 24 else range(0, wl.H, 3)
    for h in heads:
        ms, mt, md = O.profile_head(head64(q, 0, h), head64(k, 0, h), head64(v, 0, h), idx, wl.F,
                                    wl.P, wl.width)
        check_profile(mse[h:h + 1], mode[h:h + 1], np.array([[ms, mt]]), np.array([md]),
                      f"{name} head {h}")


# ---------------------------------------------------------- sparse attention

@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("kind", [O.MODE_SPATIAL, O.MODE_TEMPORAL, O.MODE_DENSE])
def test_sparse_attn_small(wl, kind):
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    list_id = torch.full((wl.B * wl.H,), kind, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_sparse_attn(qd, kd, vd, list_id, lists, status=status)
    got = to_float64(o)
    ip, ix = O.geometric_block_lists(kind, wl.F, wl.P, wl.width, wl.N)
    for b in range(wl.B):
        for h in range(wl.H):
            ref = O.block_sparse_attention(head64(q, b, h), head64(k, b, h), head64(v, b, h), ip, ix)
            assert_close(got[b, h], ref, f"{wl.name} kind {kind} head {h}",
                         bf16=wl.dtype == "bf16")
    assert status.item() == 0


@pytest.mark.parametrize("name", FULL_BF16[:1] + ["wan480", "hunyuan720"])
def test_sparse_attn_full_size_sampled(name, full_inputs):
    wl = si.WORKLOADS[name]
    (q, k, v), (qd, kd, vd), types = full_inputs(name)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    # spatial-type heads on the spatial list, temporal-type heads on the
    # temporal list (run on frame-major data: the list is applied as given)
    list_id = torch.from_numpy(types).to(DEV)
    o = svg.svg_sparse_attn(qd, kd, vd, list_id, lists)
    ob = o.view(torch.int16)
    rng = np.random.default_rng(11)
    nb = svg.n_tiles(wl.N)
    heads = rng.choice(wl.H, size=6, replace=False)
    for h in heads:
        kind = int(types[h])
        ip, ix = O.geometric_block_lists(kind, wl.F, wl.P, wl.width, wl.N)
        tiles = np.r_[rng.choice(nb - 1, size=3, replace=False), nb - 1]  # incl. ragged tail
        qh, kh, vh = head64(q, 0, h), head64(k, 0, h), head64(v, 0, h)
        for t in tiles:
            rows = O.tile_rows(int(t), wl.N)
            ref = O.block_sparse_rows(qh, kh, vh, rows, ip, ix)
            got = to_float64(o[0, h, rows[0]:rows[-1] + 1])
            assert_close(got, ref, f"{name} head {h} tile {t}")


def test_sparse_attn_empty_and_invalid_lists():
    wl = si.small("wan480")
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    N, nb = wl.N, svg.n_tiles(wl.N)
    # list 0: row 0 empty, row 1 = [nb-1], row 2 = [-3 (bad), 0], others = [i]
    rows = [[]] + [[nb - 1]] + [[-3, 0]] + [[i] for i in range(3, nb)]
    ip = np.cumsum([0] + [len(r) for r in rows]).astype(np.int32)
    ix = np.array([j for r in rows for j in r], dtype=np.int32)
    lists = svg.BlockLists(torch.from_numpy(ip).to(DEV), torch.from_numpy(ix).to(DEV), 1, nb)
    list_id = torch.tensor([0, 0, 5, 0], dtype=torch.int32, device=DEV)  # head 2: bad id
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = to_float64(svg.svg_sparse_attn(qd, kd, vd, list_id, lists, status=status))
    st = status.item()
    assert st & svg._lib.SVG_DEVICE_BAD_LIST_ID and st & svg._lib.SVG_DEVICE_BAD_INDEX
    assert (o[0, 2] == 0).all()
    assert (o[0, 0, :128] == 0).all()
    okp = np.cumsum([0] + [len([j for j in r if 0 <= j < nb]) for r in rows]).astype(np.int32)
    okx = np.array([j for r in rows for j in r if 0 <= j < nb], dtype=np.int32)
    for h in (0, 1, 3):
        ref = O.block_sparse_attention(head64(q, 0, h), head64(k, 0, h), head64(v, 0, h), okp, okx)
        assert_close(o[0, h], ref, f"head {h}")


@pytest.mark.parametrize("name", ["wan480", "cogvideox", "tiny"])
def test_sparse_attn_repeated_and_descending_entries(name):
    """A row is a set of key blocks: an entry that repeats or falls below the
    row's previous used entry is skipped and flagged (SVG_DEVICE_BAD_INDEX),
    so no block is attended twice.  Checked against the oracle on the rows'
    strictly ascending parts, for both members of a work item."""
    wl = si.small(name)
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    N, nb = wl.N, svg.n_tiles(wl.N)
    rows = [[0, 0, 2], [2, 1, 2, nb - 1], [1, 1, 1], [nb - 1, 0]] + \
        [[i, i] for i in range(4, nb)]
    rows = rows[:nb]
    ip = np.cumsum([0] + [len(r) for r in rows]).astype(np.int32)
    ix = np.array([j for r in rows for j in r], dtype=np.int32)
    lists = svg.BlockLists(torch.from_numpy(ip).to(DEV), torch.from_numpy(ix).to(DEV), 1, nb)
    list_id = torch.zeros(wl.B * wl.H, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = to_float64(svg.svg_sparse_attn(qd, kd, vd, list_id, lists, status=status))
    assert status.item() & svg._lib.SVG_DEVICE_BAD_INDEX

    def used(r):
        out, last = [], -1
        for j in r:
            if 0 <= j < nb and j > last:
                out.append(j)
                last = j
        return out
    clean = [used(r) for r in rows]
    if nb >= 4:
        assert clean[:4] == [[0, 2], [2, nb - 1], [1], [nb - 1]]
    okp = np.cumsum([0] + [len(r) for r in clean]).astype(np.int32)
    okx = np.array([j for r in clean for j in r], dtype=np.int32)
    for h in range(wl.H):
        ref = O.block_sparse_attention(head64(q, 0, h), head64(k, 0, h), head64(v, 0, h), okp, okx)
        assert_close(o[0, h], ref, f"{name} head {h}", bf16=wl.dtype == "bf16")


@pytest.mark.parametrize("name", ["wan480", "cogvideox"])
def test_wait_timeout_returns_and_context_survives(name):
    """With the poll limit of the pipeline waits cut to one, a wait runs out
    at once: the call returns, the device status word carries
    SVG_DEVICE_TIMEOUT, and the next call (default limit) is again bit-exact
    with the first, so the kernel drained its copies and MMAs, freed its
    tensor memory and left the context usable.  No fault, no trap."""
    wl = si.small(name)
    (q, k, v), (qd, kd, vd), types = workload_tensors(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    list_id = torch.full((wl.B * wl.H,), O.MODE_DENSE, dtype=torch.int32, device=DEV)
    ref = bits(svg.svg_sparse_attn(qd, kd, vd, list_id, lists))
    lib = svg._lib.lib
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    try:
        assert lib.svg_set_wait_limit(1) == svg._lib.SVG_OK
        svg.svg_sparse_attn(qd, kd, vd, list_id, lists, status=status)
        torch.cuda.synchronize()
    finally:
        lib.svg_set_wait_limit(0)
    assert status.item() & svg._lib.SVG_DEVICE_TIMEOUT
    assert lib.svg_get_wait_limit() == 1 << 22
    status.zero_()
    again = svg.svg_sparse_attn(qd, kd, vd, list_id, lists, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    np.testing.assert_array_equal(bits(again), ref)


@pytest.mark.parametrize("N,d", [(100, 64), (128, 128), (129, 64), (383, 128)])
def test_sparse_attn_ragged_dense(N, d):
    rng = np.random.default_rng(N + d)
    x = [si.to_bf16_bits(rng.standard_normal((2, 1, N, d), dtype=np.float32) * 2) for _ in range(3)]
    qd, kd, vd = (to_device(t) for t in x)
    lists = svg.geometric_lists(1, N, 0, N)
    list_id = torch.full((2,), O.MODE_DENSE, dtype=torch.int32, device=DEV)
    o = to_float64(svg.svg_sparse_attn(qd, kd, vd, list_id, lists))
    for b in range(2):
        ref = O.dense_attention(*(si.as_float64(t[b, 0]) for t in x))
        assert_close(o[b, 0], ref, f"N={N} d={d} b={b}")


# ------------------------------------------------- fused layout transformation

def _unfused(qd, kd, vd, F, P, mode, lists):
    perm = [svg.svg_permute_token_major(x, F, P, mode) for x in (qd, kd, vd)]
    op = svg.svg_sparse_attn(*perm, mode, lists)
    return svg.svg_permute_frame_major(op, F, P, mode)


FUSE_IN, FUSE_OUT = 1, 2


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_sparse_attn_fused_small(wl):
    """Every fused layout == permute -> attention -> permute back, bit for
    bit, and element-wise against the oracle, with mixed modes (incl. dense)."""
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    modes = np.array([(O.MODE_TEMPORAL, O.MODE_SPATIAL, O.MODE_DENSE, O.MODE_TEMPORAL)[h % 4]
                      for h in range(wl.B * wl.H)], dtype=np.int32)
    mode = torch.from_numpy(modes).to(DEV)
    ref_bits = bits(_unfused(qd, kd, vd, wl.F, wl.P, mode, lists))
    perm = [svg.svg_permute_token_major(x, wl.F, wl.P, mode) for x in (qd, kd, vd)]
    for layout in (FUSE_IN, FUSE_OUT, FUSE_IN | FUSE_OUT):
        ins = (qd, kd, vd) if layout & FUSE_IN else perm
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        o = svg.svg_sparse_attn_fused(*ins, wl.F, wl.P, mode, lists, layout=layout, status=status)
        assert status.item() == 0
        if not layout & FUSE_OUT:
            o = svg.svg_permute_frame_major(o, wl.F, wl.P, mode)
        np.testing.assert_array_equal(bits(o), ref_bits, err_msg=f"layout {layout}")
    got = to_float64(o)
    for h in range(wl.H):
        md = int(modes[h])
        ip, ix = O.geometric_block_lists(md, wl.F, wl.P, wl.width, wl.N)
        qh, kh, vh = head64(q, 0, h), head64(k, 0, h), head64(v, 0, h)
        if md == O.MODE_TEMPORAL:
            qh, kh, vh = (O.permute_token_major(t, wl.F, wl.P) for t in (qh, kh, vh))
        ref = O.block_sparse_attention(qh, kh, vh, ip, ix)
        if md == O.MODE_TEMPORAL:
            ref = O.permute_frame_major(ref, wl.F, wl.P)
        assert_close(got[0, h], ref, f"{wl.name} mode {md} head {h}", bf16=wl.dtype == "bf16")


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_sparse_attn_fused_with_copies(wl):
    """Temporal heads read token-major copies of every head, the others the
    frame-major inputs: same bits as the unfused composition."""
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    modes = np.array([(O.MODE_SPATIAL, O.MODE_TEMPORAL)[h % 2] for h in range(wl.H)], np.int32)
    mode = torch.from_numpy(modes).to(DEV)
    copies = tuple(svg.svg_permute_token_major(x, wl.F, wl.P, None) for x in (qd, kd, vd))
    ref = bits(_unfused(qd, kd, vd, wl.F, wl.P, mode, lists))
    for layout in (0, FUSE_OUT):
        o = svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, mode, lists, layout=layout,
                                      copies=copies)
        if not layout & FUSE_OUT:
            o = svg.svg_permute_frame_major(o, wl.F, wl.P, mode)
        np.testing.assert_array_equal(bits(o), ref, err_msg=f"layout {layout}")


@pytest.mark.parametrize("name", ["wan480", "hunyuan720"])
def test_sparse_attn_fused_full_size_sampled(name, full_inputs):
    """Token-major gathers at the full sizes (F = 21 and 33 frames)."""
    wl = si.WORKLOADS[name]
    (q, k, v), (qd, kd, vd), types = full_inputs(name)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    mode = torch.from_numpy(types).to(DEV)
    o = svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, mode, lists)
    src = O.token_major_source(wl.F, wl.P)
    rng = np.random.default_rng(13)
    nb = svg.n_tiles(wl.N)
    temporal = np.flatnonzero(types == O.MODE_TEMPORAL)
    for h in list(rng.choice(temporal, size=3, replace=False)) + [int(np.flatnonzero(types == 0)[0])]:
        md = int(types[h])
        ip, ix = O.geometric_block_lists(md, wl.F, wl.P, wl.width, wl.N)
        qh, kh, vh = head64(q, 0, h), head64(k, 0, h), head64(v, 0, h)
        if md == O.MODE_TEMPORAL:
            qh, kh, vh = (O.permute_token_major(t, wl.F, wl.P) for t in (qh, kh, vh))
        for t in np.r_[rng.choice(nb - 1, size=2, replace=False), nb - 1]:
            rows = O.tile_rows(int(t), wl.N)
            ref = O.block_sparse_rows(qh, kh, vh, rows, ip, ix)
            out_rows = src[rows] if md == O.MODE_TEMPORAL else rows
            got = to_float64(o[0, h][torch.from_numpy(out_rows).to(DEV)])
            assert_close(got, ref, f"{name} fused head {h} tile {t}")


def test_sparse_attn_fused_bad_mode():
    wl = si.small("cogvideox")
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    mode = torch.tensor([1, 7, 0, 1], dtype=torch.int32, device=DEV)  # head 1: not a list
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, mode, lists, status=status)
    assert status.item() & svg._lib.SVG_DEVICE_BAD_LIST_ID
    assert (to_float64(o[0, 1]) == 0).all()
    good = torch.tensor([1, 0, 0, 1], dtype=torch.int32, device=DEV)
    ref = svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, good, lists)
    for h in (0, 2, 3):
        np.testing.assert_array_equal(bits(o[0, h]), bits(ref[0, h]))


@pytest.mark.parametrize("value,flagged", [(65280.0, False), (-65280.0, False), (65536.0, True),
                                           (-1.0e6, True), (float("inf"), True),
                                           (float("nan"), True)])
def test_sparse_attn_v_range_flag(value, flagged):
    """bf16 -> fp16 conversion of V on chip: the largest bf16 below the fp16
    limit 65504 passes; larger magnitudes, inf and NaN set SVG_DEVICE_RANGE."""
    wl = si.small("cogvideox")
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    dense = torch.full((wl.B * wl.H,), O.MODE_DENSE, dtype=torch.int32, device=DEV)
    vd = vd.clone()
    vd[0, 1, wl.N - 1, 5] = value  # last (ragged) key tile of head 1
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_sparse_attn(qd, kd, vd, dense, lists, status=status)
    torch.cuda.synchronize()
    assert bool(status.item() & svg._lib.SVG_DEVICE_RANGE) == flagged
    if not flagged:
        # the value is exact in fp16, so head 1 matches the oracle; with |v|
        # this large the fp16 rounding of P (2^-12 relative per term, and as
        # much again through the row sum) is no longer below the bf16 output
        # rounding, so the bound adds 2^-11 |o| to half a bf16 ulp
        vh = head64(v, 0, 1)
        vh[wl.N - 1, 5] = value
        ip, ix = O.geometric_block_lists(O.MODE_DENSE, wl.F, wl.P, wl.width, wl.N)
        rows = np.arange(wl.N)
        want = O.block_sparse_rows(head64(q, 0, 1), head64(k, 0, 1), vh, rows, ip, ix)
        got = to_float64(o[0, 1])
        bound = np.maximum(MAX_ABS, half_ulp_bf16(want) + 1e-3 + 2.0 ** -11 * np.abs(want))
        err = np.abs(got - want)
        assert (err <= bound).all(), f"v = {value}: worst excess {(err - bound).max():.4g}"


def _v_exponents_ref(vbits):
    """Oracle-free reference of svg_v_exponents from the bf16 bits: the
    smallest e >= 0 with max|v| * 2^-e <= 65504 (255 for inf / NaN)."""
    B, H = vbits.shape[:2]
    out = np.zeros(B * H, np.int64)
    for b in range(B):
        for h in range(H):
            m = int((vbits[b, h].astype(np.uint32) & 0x7fff).max())
            if m >= 0x7f80:
                out[b * H + h] = 255
                continue
            mx = float(si.bf16_bits_to_f32(np.array([m], np.uint16))[0])
            e = 0
            while mx * 2.0 ** -e > 65504.0:
                e += 1
            out[b * H + h] = e
    return out


@pytest.mark.parametrize("name", ["wan480", "cogvideox"])
def test_v_exponents_scale_v_into_fp16_range(name):
    """V beyond the fp16 range gives the correct output when the call takes
    svg_v_exponents' per-head exponents: head 0 holds one outlier (checked
    against the oracle), head 1 is the whole head times 2^20 (its output is
    exactly 2^20 times the unscaled head's, bit for bit), head 2 an inf
    (exponent 255, flagged), head 3 is untouched (exponent 0, bits equal to
    the call without exponents)."""
    wl = si.small(name)
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    dense = torch.full((wl.B * wl.H,), O.MODE_DENSE, dtype=torch.int32, device=DEV)
    plain = svg.svg_sparse_attn(qd, kd, vd, dense, lists)
    v2 = vd.clone()
    v2[0, 0, 7, 3] = 3.0e5
    v2[0, 1] = vd[0, 1] * 2.0 ** 20
    v2[0, 2, 9, 1] = float("inf")
    vbits = v2.view(torch.int16).cpu().numpy().view(np.uint16)
    exps = svg.svg_v_exponents(v2)
    np.testing.assert_array_equal(exps.cpu().numpy(), _v_exponents_ref(vbits))
    assert exps[0].item() > 0 and exps[1].item() > 0 and exps[2].item() == 255
    assert exps[3].item() == 0
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = svg.svg_sparse_attn(qd, kd, v2, dense, lists, v_exp=exps, status=status)
    torch.cuda.synchronize()
    assert status.item() & svg._lib.SVG_DEVICE_RANGE  # head 2's inf
    # head 0: the outlier, against the oracle (as in the range-flag test)
    vh = head64(v, 0, 0)
    vh[7, 3] = float(v2[0, 0, 7, 3].item())
    ip, ix = O.geometric_block_lists(O.MODE_DENSE, wl.F, wl.P, wl.width, wl.N)
    want = O.block_sparse_rows(head64(q, 0, 0), head64(k, 0, 0), vh, np.arange(wl.N), ip, ix)
    got = to_float64(o[0, 0])
    bound = np.maximum(MAX_ABS, half_ulp_bf16(want) + 1e-3 + 2.0 ** -11 * np.abs(want))
    assert (np.abs(got - want) <= bound).all()
    # head 1: 2^20 times the unscaled head (the scaled head converts v * 2^12
    # to fp16, exact, so the products only move by a power of two; a value
    # below the fp16 normal range may keep more bits there than unscaled,
    # hence one bf16 ulp of slack)
    g1, w1 = to_float64(o[0, 1]), to_float64(plain[0, 1]) * 2.0 ** 20
    assert (np.abs(g1 - w1) <= 2 * half_ulp_bf16(w1)).all()
    assert (g1 == w1).mean() > 0.999
    # head 3: the same bits as without exponents
    np.testing.assert_array_equal(bits(o[0, 3]), bits(plain[0, 3]))
    # without exponents head 1 overflows fp16: flagged
    status.zero_()
    svg.svg_sparse_attn(qd, kd, v2, dense, lists, status=status)
    torch.cuda.synchronize()
    assert status.item() & svg._lib.SVG_DEVICE_RANGE


# ---------------------------------------------------------------- the layer

@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_layer_small(wl):
    (q, k, v), (qd, kd, vd), types = workload_tensors(wl)
    idx = si.sample_queries(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    o, mode, mse = svg.svg_layer(qd, kd, vd, wl.F, wl.P, wl.width,
                                 torch.from_numpy(idx).to(DEV), lists)
    o_ref, mode_ref, mse_ref = O.svg_layer(si.as_float64(q), si.as_float64(k), si.as_float64(v),
                                           idx, wl.F, wl.P, wl.width)
    check_profile(mse.cpu().numpy(), mode.cpu().numpy(), mse_ref, mode_ref, wl.name)
    np.testing.assert_array_equal(mode.cpu().numpy(), mode_ref)
    got = to_float64(o)
    for h in range(wl.H):
        assert_close(got[0, h], o_ref[0, h], f"{wl.name} head {h}", bf16=wl.dtype == "bf16")


@pytest.mark.parametrize("wl", SMALL[:3], ids=lambda w: w.name)
def test_layer_small_layouts_agree(wl):
    """The layer gives the same bits whichever side of the reordering is
    fused into the attention kernel."""
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    idx = torch.from_numpy(si.sample_queries(wl)).to(DEV)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    outs = []
    for layout, overlap in ((0, False), (0, True), (FUSE_IN, False), (FUSE_OUT, False),
                            (FUSE_OUT, True), (FUSE_IN | FUSE_OUT, False)):
        bufs = svg.LayerBuffers(qd, idx.numel(), layout=layout)
        o, m, _ = svg.svg_layer(qd, kd, vd, wl.F, wl.P, wl.width, idx, lists, bufs, layout=layout,
                                overlap=overlap)
        torch.cuda.synchronize()
        outs.append((bits(o), m.cpu().numpy()))
    for o, m in outs[1:]:
        np.testing.assert_array_equal(m, outs[0][1])
        np.testing.assert_array_equal(o, outs[0][0])


@pytest.mark.parametrize("wl", [w for w in SMALL if w.dtype == "bf16" and w.kind == "profiled"],
                         ids=lambda w: w.name)
def test_layer_from_host_matches_device_layer(wl):
    """The host-streamed layer (chunks of heads through two device slots, copies
    overlapped with compute) gives the device layer's bits, for one chunk per
    head, two heads per chunk and all heads in one chunk; repeated calls reuse
    the slots."""
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    idx = torch.from_numpy(si.sample_queries(wl)).to(DEV)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    o_ref, m_ref, _ = svg.svg_layer(qd, kd, vd, wl.F, wl.P, wl.width, idx, lists)
    torch.cuda.synchronize()
    o_ref, m_ref = bits(o_ref), m_ref.cpu().numpy()
    host = [x.cpu().pin_memory() for x in (qd, kd, vd)]
    BH = wl.B * wl.H
    for hc in (1, 2, BH):
        if BH % hc:
            continue
        bufs = svg.HostLayerBuffers(hc, wl.N, wl.d, idx.numel())
        for call in range(3):  # own buffers, then the same slots twice
            out, mode = svg.svg_layer_from_host(*host, wl.F, wl.P, wl.width, idx, lists,
                                                heads_per_chunk=hc,
                                                buffers=None if call == 0 else bufs)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(mode.numpy(), m_ref)
            np.testing.assert_array_equal(bits(out), o_ref)
    with pytest.raises(ValueError):
        svg.svg_layer_from_host(*host, wl.F, wl.P, wl.width, idx, lists, heads_per_chunk=BH + 1)


def test_layer_full_size_hunyuan_every_head(full_inputs):
    """The HunyuanVideo 720p layer (B=1, H=24, N=118800, d=128, band 2) as the
    bench runs it (profiling, token-major copies of the temporal heads,
    attention writing frame-major rows): the modes, and 64 query tiles of
    every head (the ragged tail among them) against the oracle."""
    name = "hunyuan720"
    wl = si.WORKLOADS[name]
    (q, k, v), (qd, kd, vd), types = full_inputs(name)
    idx = si.sample_queries(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    o, mode, _ = svg.svg_layer(qd, kd, vd, wl.F, wl.P, wl.width, torch.from_numpy(idx).to(DEV),
                               lists)
    mode = mode.cpu().numpy()
    np.testing.assert_array_equal(mode, types)
    src = O.token_major_source(wl.F, wl.P)
    rng = np.random.default_rng(118800)
    nb = svg.n_tiles(wl.N)
    geo = {md: O.geometric_block_lists(md, wl.F, wl.P, wl.width, wl.N) for md in (0, 1)}
    for h in range(wl.H):
        md = int(mode[h])
        ip, ix = geo[md]
        qh, kh, vh = head64(q, 0, h), head64(k, 0, h), head64(v, 0, h)
        if md == O.MODE_TEMPORAL:
            qh, kh, vh = (O.permute_token_major(t, wl.F, wl.P) for t in (qh, kh, vh))
        for t in np.r_[rng.choice(nb - 1, size=63, replace=False), nb - 1]:
            rows, ref = tile_rows_kept_keys(qh, kh, vh, int(t), wl.N, ip, ix)
            out_rows = src[rows] if md == O.MODE_TEMPORAL else rows
            got = to_float64(o[0, h][torch.from_numpy(out_rows).to(DEV)])
            assert_close(got, ref, f"layer head {h} tile {t}")


def test_layer_full_size_cogvideox_sampled(full_inputs):
    name = "cogvideox"
    wl = si.WORKLOADS[name]
    (q, k, v), (qd, kd, vd), types = full_inputs(name)
    idx = si.sample_queries(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    o, mode, mse = svg.svg_layer(qd, kd, vd, wl.F, wl.P, wl.width,
                                 torch.from_numpy(idx).to(DEV), lists)
    mode = mode.cpu().numpy()
    np.testing.assert_array_equal(mode, types)
    src = O.token_major_source(wl.F, wl.P)
    rng = np.random.default_rng(5)
    nb = svg.n_tiles(wl.N)
    for h in rng.choice(wl.H, size=6, replace=False):
        md = int(mode[h])
        ip, ix = O.geometric_block_lists(md, wl.F, wl.P, wl.width, wl.N)
        qh, kh, vh = head64(q, 0, h), head64(k, 0, h), head64(v, 0, h)
        if md == O.MODE_TEMPORAL:
            qh, kh, vh = (O.permute_token_major(t, wl.F, wl.P) for t in (qh, kh, vh))
        for t in np.r_[rng.choice(nb - 1, size=2, replace=False), nb - 1]:
            rows = O.tile_rows(int(t), wl.N)
            ref = O.block_sparse_rows(qh, kh, vh, rows, ip, ix)
            out_rows = src[rows] if md == O.MODE_TEMPORAL else rows
            got = to_float64(o[0, h][torch.from_numpy(out_rows).to(DEV)])
            assert_close(got, ref, f"layer head {h} tile {t}")


# ------------------------------------------------------ energy and calibration

@pytest.mark.parametrize("name", ["tiny", "wan720", "cogvideox"])
def test_block_energy_small(name):
    wl = si.small(name)
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    E = svg.svg_block_energy(qd, kd).cpu().numpy().astype(np.float64)
    for h in range(wl.H):
        ref = O.block_energy(head64(q, 0, h), head64(k, 0, h))
        np.testing.assert_allclose(E[h], ref, rtol=2e-3, atol=2e-5, err_msg=f"{name} head {h}")
        np.testing.assert_allclose(E[h].sum(1), 1.0, atol=1e-4)


def test_calibrated_lists_bit_exact_given_energies():
    rng = np.random.default_rng(21)
    R, L, nq, nk = 4, 3, 9, 37
    E = rng.dirichlet(np.ones(nk) * 0.3, size=(R, L, nq)).astype(np.float32)
    E[0, 0, 0] = 0.0
    E[0, 0, 0, :4] = 0.25                        # exact ties
    E[:, 1, 2] = np.float32(1.0 / nk)            # all ties, every input
    E[1, 2, 3] = np.eye(nk, dtype=np.float32)[5]
    for eps, rho in [(0.9, 0.5), (0.5, 1.0), (0.99, 0.25), (0.3, 0.75)]:
        lists = svg.svg_build_block_mask_calibrated(torch.from_numpy(E).to(DEV), eps, rho)
        ip = lists.indptr.cpu().numpy().reshape(L, nq + 1)
        ix = lists.indices.cpu().numpy()
        for l in range(L):
            op, ox = O.calibrate_lists([E[r, l].astype(np.float64) for r in range(R)], eps, rho)
            np.testing.assert_array_equal(ip[l] - ip[l][0], op, err_msg=f"eps {eps} rho {rho}")
            np.testing.assert_array_equal(ix[ip[l][0]:ip[l][-1]], ox)


@pytest.mark.parametrize("R,L,nq,nk", [(4, 5, 600, 600), (3, 2, 1100, 929), (4, 40, 64, 591)])
def test_calibrated_lists_bit_exact_given_energies_large(R, L, nq, nk):
    """Rows wider than 512 key blocks (the 1024-entry sort) and more rows
    than one scan chunk (L * nQB > 1024, carried across chunks)."""
    rng = np.random.default_rng(1000 + nk)
    E = rng.dirichlet(np.ones(nk) * 0.05, size=(R, L, nq)).astype(np.float32)
    E[0, 0, 1] = np.float32(1.0 / nk)            # all ties
    for eps, rho in [(0.9, 0.5), (0.97, 0.75)]:
        lists = svg.svg_build_block_mask_calibrated(torch.from_numpy(E).to(DEV), eps, rho)
        ip = lists.indptr.cpu().numpy().reshape(L, nq + 1)
        ix = lists.indices.cpu().numpy()
        assert ip[0][0] == 0 and (np.diff(ip.reshape(-1)[:-1]) >= 0).all()
        for l in sorted({0, L // 2, L - 1}):
            op, ox = O.calibrate_lists([E[r, l].astype(np.float64) for r in range(R)], eps, rho)
            np.testing.assert_array_equal(ip[l] - ip[l][0], op, err_msg=f"list {l} eps {eps}")
            np.testing.assert_array_equal(ix[ip[l][0]:ip[l][-1]], ox)
        # every list starts where the previous one ends (one shared indices array)
        np.testing.assert_array_equal(ip[1:, 0], ip[:-1, -1])


def cut_margin(e_row, eps):
    order = O.energy_order(e_row)
    cum = np.cumsum(np.asarray(e_row, np.float64)[order])
    kk = int(np.searchsorted(cum, eps))  # first index with cum >= eps
    prev = cum[kk - 1] if kk > 0 else 0.0
    nxt = cum[kk] if kk < len(cum) else 1.0
    gap = (e_row[order[kk]] - e_row[order[kk + 1]]) if kk + 1 < len(order) else 1.0
    return min(eps - prev, nxt - eps, gap)


def test_calibration_end_to_end_small():
    wl = si.small("wan720")
    types_seed = wl.calib_seeds[0]
    Es_gpu, Es_ref = [], []
    for s in wl.calib_seeds:
        (q, k, v), (qd, kd, vd), _ = workload_tensors(wl, seed=s, types_seed=types_seed)
        Es_gpu.append(svg.svg_block_energy(qd, kd))
        Es_ref.append([O.block_energy(head64(q, 0, h), head64(k, 0, h)) for h in range(wl.H)])
    E = torch.stack(Es_gpu)  # [R, L, nq, nk]
    lists = svg.svg_build_block_mask_calibrated(E.contiguous(), wl.eps, wl.rho)
    nq = svg.n_tiles(wl.N)
    ip = lists.indptr.cpu().numpy().reshape(wl.H, nq + 1)
    ix = lists.indices.cpu().numpy()
    compared = 0
    for h in range(wl.H):
        op, ox = O.calibrate_lists([Es_ref[r][h] for r in range(len(wl.calib_seeds))], wl.eps,
                                   wl.rho)
        for r in range(nq):
            if min(cut_margin(Es_ref[s][h][r], wl.eps) for s in range(len(wl.calib_seeds))) <= 1e-3:
                continue
            compared += 1
            np.testing.assert_array_equal(ix[ip[h][r]:ip[h][r + 1]], ox[op[r]:op[r + 1]])
    assert compared > 0
    # and attention on the calibrated lists for the timed input
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl, seed=wl.seed, types_seed=types_seed)
    list_id = torch.arange(wl.H, dtype=torch.int32, device=DEV)
    o = to_float64(svg.svg_sparse_attn(qd, kd, vd, list_id, lists))
    for h in range(wl.H):
        hp = ip[h] - ip[h][0]
        hx = ix[ip[h][0]:ip[h][-1]]
        ref = O.block_sparse_attention(head64(q, 0, h), head64(k, 0, h), head64(v, 0, h), hp, hx)
        assert_close(o[0, h], ref, f"calibrated head {h}")


def test_calibration_full_size_sampled():
    """The calibrated Wan 2.1 720p layer at full size (B=1, H=40, N=75600,
    d=128): GPU block energies of the four calibration inputs, the 40
    per-head lists built from them, and attention on the timed input with
    list_id = h.  The oracle computes energy rows of sampled query blocks
    (float64, full N keys) for sampled heads; a list row is compared where
    every input's cut margin exceeds 1e-3.  Attention is compared on sampled
    query tiles of sampled heads, element by element, on the lists the GPU
    built."""
    wl = si.WORKLOADS["wan720"]
    rng = np.random.default_rng(720)
    heads = sorted(rng.choice(wl.H, 4, replace=False).tolist())
    nb = svg.n_tiles(wl.N)
    blocks = sorted(rng.choice(nb - 1, 5, replace=False).tolist()) + [nb - 1]  # + ragged tail
    types_seed = wl.calib_seeds[0]
    Es = []
    ref_E = {h: [] for h in heads}
    for s in wl.calib_seeds:
        q, k, _, _ = si.generate(wl, seed=s, types_seed=types_seed)
        qd, kd = to_device(q), to_device(k)
        Es.append(svg.svg_block_energy(qd, kd))
        del qd, kd
        for h in heads:
            ref_E[h].append(O.block_energy(head64(q, 0, h), head64(k, 0, h), row_blocks=blocks))
        del q, k
    E = torch.stack(Es).contiguous()  # [R, 40, 591, 591]
    del Es
    Eh = E.cpu().numpy()
    for h in heads:  # the GPU energies of the sampled rows, against float64
        for s in range(len(wl.calib_seeds)):
            np.testing.assert_allclose(Eh[s, h][blocks], ref_E[h][s], rtol=2e-3, atol=2e-5)
    lists = svg.svg_build_block_mask_calibrated(E, wl.eps, wl.rho)
    del E
    ip = lists.indptr.cpu().numpy().reshape(wl.H, nb + 1)
    ix = lists.indices.cpu().numpy()
    R = len(wl.calib_seeds)
    compared = 0
    for h in heads:
        # the builder at full size (1024-entry sorts, 23640 rows over many
        # scan chunks) is bit-exact given the energies it was handed ...
        Eg = [Eh[s, h][blocks].astype(np.float64) for s in range(R)]
        gp, gx = O.calibrate_lists(Eg, wl.eps, wl.rho)
        # ... and end to end it equals the float64 pipeline on every row whose
        # per-input eps-cuts come out the same from the GPU's fp32 energies
        # as from the oracle's (near-ties of 591 small energies can flip)
        op, ox = O.calibrate_lists(ref_E[h], wl.eps, wl.rho)
        for n, r in enumerate(blocks):
            got = ix[ip[h][r]:ip[h][r + 1]]
            np.testing.assert_array_equal(got, gx[gp[n]:gp[n + 1]], err_msg=f"head {h} block {r}")
            if all(O.minimal_energy_set(Eg[s][n], wl.eps) ==
                   O.minimal_energy_set(ref_E[h][s][n], wl.eps) for s in range(R)):
                compared += 1
                np.testing.assert_array_equal(got, ox[op[n]:op[n + 1]],
                                              err_msg=f"head {h} block {r}")
    assert compared >= 1
    kept = (ip[:, -1] - ip[:, 0]).sum() / float(wl.H * nb * nb)
    assert 0.0 < kept < 1.0
    # attention on the timed input as the bench runs it (V exponents, every
    # head on its own list, query tiles paired by svg_pair_query_tiles): 64
    # query tiles of every head, the ragged tail among them
    q, k, v, _ = si.generate(wl, seed=wl.seed, types_seed=types_seed)
    qd, kd, vd = (to_device(x) for x in (q, k, v))
    list_id = torch.arange(wl.H, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    paired = svg.svg_pair_query_tiles(lists, status=status)
    o = svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, list_id, paired, layout=0,
                                  v_exp=svg.svg_v_exponents(vd), status=status)
    assert int(status.item()) == 0
    del qd, kd, vd
    for h in range(wl.H):
        hp = ip[h] - ip[h][0]
        hx = ix[ip[h][0]:ip[h][-1]]
        qh, kh, vh = head64(q, 0, h), head64(k, 0, h), head64(v, 0, h)
        for t in np.r_[rng.choice(nb - 1, size=63, replace=False), nb - 1]:
            rows, ref = tile_rows_kept_keys(qh, kh, vh, int(t), wl.N, hp, hx)
            got = to_float64(o[0, h, rows[0]:rows[-1] + 1])
            assert_close(got, ref, f"calibrated head {h} tile {t}")


# ------------------------------------------------ mask encodings (skip list, bitmap)

def _rand_csr(rows, n_cols, seed, dup=False):
    rng = np.random.default_rng(seed)
    ip, ix = [0], []
    for _ in range(rows):
        k = int(rng.integers(0, min(n_cols, 80) + 1))
        r = sorted(rng.choice(n_cols, size=k, replace=False).tolist())
        if dup and r:
            r = sorted(r + rng.choice(r, size=min(3, len(r))).tolist())
        ix.extend(r)
        ip.append(len(ix))
    return np.asarray(ip, np.int32), np.asarray(ix, np.int32)


def _check_encodings(ip, ix, n_cols, what):
    ipd = torch.from_numpy(ip).to(DEV)
    ixd = torch.from_numpy(ix if ix.size else np.zeros(1, np.int32)).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    iptr, st, en = svg.svg_lists_to_intervals(ipd, ixd, n_cols, status=status)
    bm = svg.svg_lists_to_bitmap(ipd, ixd, n_cols, status=status)
    assert status.item() == 0, what
    r_iptr, r_st, r_en = O.lists_to_intervals(ip, ix)
    np.testing.assert_array_equal(iptr.cpu().numpy(), r_iptr, err_msg=what)
    np.testing.assert_array_equal(st.cpu().numpy(), r_st, err_msg=what)
    np.testing.assert_array_equal(en.cpu().numpy(), r_en, err_msg=what)
    np.testing.assert_array_equal(bm.cpu().numpy().view(np.uint32),
                                  O.lists_to_bitmap(ip, ix, n_cols), err_msg=what)


@pytest.mark.parametrize("n_cols", [1, 31, 32, 33, 138, 929, 2000])
def test_encodings_random(n_cols):
    ip, ix = _rand_csr(300, n_cols, n_cols)
    _check_encodings(ip, ix, n_cols, f"random n_cols={n_cols}")
    ip, ix = _rand_csr(57, n_cols, n_cols + 1, dup=True)  # duplicates merge into runs
    _check_encodings(ip, ix, n_cols, f"duplicates n_cols={n_cols}")


@pytest.mark.parametrize("name", si.ORDER)
def test_encodings_geometric_lists(name):
    wl = si.WORKLOADS[name]
    nb = svg.n_tiles(wl.N)
    for kind in (O.MODE_SPATIAL, O.MODE_TEMPORAL, O.MODE_DENSE):
        ip, ix = O.geometric_block_lists(kind, wl.F, wl.P, wl.width, wl.N)
        _check_encodings(ip, ix, nb, f"{name} kind {kind}")


def test_encodings_capacity_and_bad_index():
    ip, ix = _rand_csr(40, 100, 3)
    ipd, ixd = torch.from_numpy(ip).to(DEV), torch.from_numpy(ix).to(DEV)
    n_runs = len(O.lists_to_intervals(ip, ix)[1])
    iptr = torch.empty(41, dtype=torch.int32, device=DEV)
    starts = torch.full((n_runs - 1,), -7, dtype=torch.int32, device=DEV)
    ends = torch.full((n_runs - 1,), -7, dtype=torch.int32, device=DEV)
    n = torch.zeros(1, dtype=torch.int64, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    svg._lib.call("svg_lists_to_intervals", 40, 100, ipd.data_ptr(), ixd.data_ptr(),
                  iptr.data_ptr(), starts.data_ptr(), ends.data_ptr(), n_runs - 1, n.data_ptr(),
                  status.data_ptr(), None)
    assert status.item() & svg._lib.SVG_DEVICE_CAPACITY and n.item() == n_runs
    _, r_st, r_en = O.lists_to_intervals(ip, ix)
    np.testing.assert_array_equal(starts.cpu().numpy(), r_st[:n_runs - 1])
    np.testing.assert_array_equal(ends.cpu().numpy(), r_en[:n_runs - 1])
    bad = ix.copy()
    bad[5] = 100  # outside [0, n_cols)
    status.zero_()
    bm = svg.svg_lists_to_bitmap(ipd, torch.from_numpy(bad).to(DEV), 100, status=status)
    assert status.item() & svg._lib.SVG_DEVICE_BAD_INDEX
    good = np.delete(bad, 5)
    ip2 = ip.copy()
    ip2[np.searchsorted(ip, 5, side="right"):] -= 1
    np.testing.assert_array_equal(bm.cpu().numpy().view(np.uint32), O.lists_to_bitmap(ip2, good, 100))


# ------------------------------------------------------- QK-Norm + RoPE (f2)

def qk_inputs(wl):
    (q, k, _), (qd, kd, _), _ = workload_tensors(wl)
    gq, gk = si.qk_norm_weights(wl)
    cos, sin = si.rope_tables(wl)
    dev = lambda a: torch.from_numpy(a).to(DEV)
    qk = svg.QKTransform(dev(gq), dev(gk), 1e-6, dev(cos), dev(sin))
    return (q, k), (qd, kd), (gq, gk, cos, sin), qk


def check_qk(got, x64, gamma, eps, cos, sin, bf16, what, norm=True, rope=True):
    """got vs the float64 oracle.  Bound per element: fp32 arithmetic (a few
    2^-24 of the rotated magnitudes |a c| + |b s|, with margin 2^-17) plus,
    for bf16 results, half a bf16 ulp of the rounding."""
    ref = O.qk_norm_rope(x64, gamma, eps, cos, sin, norm=norm, rope=rope)
    pre = np.abs(O.qk_rms_norm(x64, gamma, eps) if norm else x64)
    if rope:
        c, s = np.abs(cos), np.abs(sin)
        mag = np.empty_like(pre)
        mag[..., 0::2] = pre[..., 0::2] * c + pre[..., 1::2] * s
        mag[..., 1::2] = pre[..., 0::2] * s + pre[..., 1::2] * c
    else:
        mag = pre
    slack = 2.0 ** -17 * mag + 1e-30
    bound = slack + (half_ulp_bf16(np.abs(ref) + slack) if bf16 else 0.0)
    err = np.abs(got - ref)
    assert (err <= bound).all(), f"{what}: worst excess {(err - bound).max():.3g}"


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_qk_norm_rope_small(wl):
    (q, k), (qd, kd), (gq, gk, cos, sin), qk = qk_inputs(wl)
    q_tm, k_tm = torch.empty_like(qd), torch.empty_like(kd)
    qo, ko = svg.svg_qk_norm_rope(qd, kd, qk, tm_out=(q_tm, k_tm), frames=wl.F,
                                  tokens_per_frame=wl.P)
    bf16 = wl.dtype == "bf16"
    for x, g, got in ((q, gq, qo), (k, gk, ko)):
        check_qk(to_float64(got), si.as_float64(x), g, 1e-6, cos, sin, bf16, wl.name)
    # the token-major copies hold the same bits, reordered m = s F + f <- n = f P + s
    src = O.token_major_source(wl.F, wl.P)
    for fm, tm in ((qo, q_tm), (ko, k_tm)):
        np.testing.assert_array_equal(bits(tm), bits(fm)[:, :, src])


@pytest.mark.parametrize("which", ["norm", "rope", "copy", "unit_weight"])
def test_qk_norm_rope_ops(which):
    wl = si.small("wan480")
    (q, k), (qd, kd), (gq, gk, cos, sin), qk = qk_inputs(wl)
    norm, rope = which in ("norm", "unit_weight"), which == "rope"
    if which == "unit_weight":
        qk = qk._replace(gamma_q=None, gamma_k=None)
        gq = gk = None
    qk = qk._replace(norm=norm, cos=qk.cos if rope else None, sin=qk.sin if rope else None)
    qo, ko = svg.svg_qk_norm_rope(qd, kd, qk)
    if which == "copy":
        np.testing.assert_array_equal(bits(qo), bits(qd))
        np.testing.assert_array_equal(bits(ko), bits(kd))
        return
    for x, g, got in ((q, gq, qo), (k, gk, ko)):
        check_qk(to_float64(got), si.as_float64(x), g, 1e-6, cos, sin, True, which,
                 norm=norm, rope=rope)


def test_qk_norm_rope_in_place():
    wl = si.small("cogvideox")
    _, (qd, kd), _, qk = qk_inputs(wl)
    want = svg.svg_qk_norm_rope(qd, kd, qk)
    qi, ki = qd.clone(), kd.clone()
    svg.svg_qk_norm_rope(qi, ki, qk, out=(qi, ki))
    np.testing.assert_array_equal(bits(qi), bits(want[0]))
    np.testing.assert_array_equal(bits(ki), bits(want[1]))


@pytest.mark.parametrize("name", ["cogvideox", "hunyuan720"])
def test_qk_norm_rope_full_sampled(name, full_inputs):
    wl = si.WORKLOADS[name]
    (q, k, _), (qd, kd, _), _ = full_inputs(name)
    gq, gk = si.qk_norm_weights(wl)
    cos, sin = si.rope_tables(wl)
    dev = lambda a: torch.from_numpy(a).to(DEV)
    qk = svg.QKTransform(dev(gq), dev(gk), 1e-6, dev(cos), dev(sin))
    q_tm, k_tm = torch.empty_like(qd), torch.empty_like(kd)
    qo, ko = svg.svg_qk_norm_rope(qd, kd, qk, tm_out=(q_tm, k_tm), frames=wl.F,
                                  tokens_per_frame=wl.P)
    rng = np.random.default_rng(17)
    heads = rng.choice(wl.H, size=4, replace=False)
    rows = np.r_[rng.choice(wl.N - 1, size=509, replace=False), wl.N - 1]
    src = O.token_major_source(wl.F, wl.P)
    inv = np.empty_like(src)
    inv[src] = np.arange(wl.N)  # token-major row of token n
    rows_d = torch.from_numpy(rows).to(DEV)
    inv_d = torch.from_numpy(inv[rows]).to(DEV)
    for h in heads:
        for x, g, got, tm in ((q, gq, qo, q_tm), (k, gk, ko, k_tm)):
            sel = got[0, h][rows_d]
            check_qk(to_float64(sel), si.as_float64(x[0, h][rows]), g, 1e-6, cos[rows],
                     sin[rows], True, f"{name} head {h}")
            np.testing.assert_array_equal(bits(tm[0, h][inv_d]), bits(sel))


@pytest.mark.parametrize("overlap", [True, False])
@pytest.mark.parametrize("name", ["cogvideox", "wan480"])
def test_layer_small_with_qk_norm_rope(name, overlap):
    wl = si.small(name)
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    gq, gk = si.qk_norm_weights(wl)
    cos, sin = si.rope_tables(wl)
    dev = lambda a: torch.from_numpy(a).to(DEV)
    qk = svg.QKTransform(dev(gq), dev(gk), 1e-6, dev(cos), dev(sin))
    idx = si.sample_queries(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    o, mode, mse = svg.svg_layer(qd, kd, vd, wl.F, wl.P, wl.width,
                                 torch.from_numpy(idx).to(DEV), lists, overlap=overlap, qk=qk)
    o_ref, mode_ref, mse_ref = O.svg_layer(si.as_float64(q), si.as_float64(k), si.as_float64(v),
                                           idx, wl.F, wl.P, wl.width,
                                           qk=(gq, gk, 1e-6, cos, sin),
                                           qk_bf16=wl.dtype == "bf16")
    check_profile(mse.cpu().numpy(), mode.cpu().numpy(), mse_ref, mode_ref, wl.name)
    m = mode.cpu().numpy()
    for bh in range(wl.B * wl.H):
        if m[bh] != mode_ref[bh]:
            continue  # a near-tie decided the other way (checked above)
        b, h = divmod(bh, wl.H)
        assert_close(to_float64(o[b, h]), o_ref[b, h], f"{wl.name} head {h}")


# ------------------------------------------- spatial-repetition heads (f4)

def sim_tol(wl):
    # probabilities are rounded to fp16 (2^-11 relative) before the Gram
    # products: every G entry within 2^-10 relative, a cosine within 2e-3
    return 2e-3 if wl.dtype == "bf16" else 1e-5


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_row_similarity_small(wl):
    (q, k, _), (qd, kd, _), _ = workload_tensors(wl)
    sim = svg.svg_row_similarity(qd, kd, wl.F, wl.ph, wl.pw).cpu().numpy()
    pick = [wl.F - 1, 1]
    sub = torch.tensor(pick, dtype=torch.int32, device=DEV)
    sim_sub = svg.svg_row_similarity(qd, kd, wl.F, wl.ph, wl.pw, sub).cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            q64, k64 = head64(q, b, h), head64(k, b, h)
            want = O.row_similarity(q64, k64, wl.F, wl.ph, wl.pw)
            want_sub = O.row_similarity(q64, k64, wl.F, wl.ph, wl.pw, pick)
            i = b * wl.H + h
            assert abs(sim[i] - want) <= sim_tol(wl), (wl.name, h, sim[i], want)
            assert abs(sim_sub[i] - want_sub) <= sim_tol(wl), (wl.name, h, sim_sub[i], want_sub)


def test_row_similarity_identical_rows():
    # queries that depend on (frame, column) only: every row attends alike
    wl = si.small("wan480")
    (q, k, _), _, _ = workload_tensors(wl)
    qr = q.reshape(wl.B, wl.H, wl.F, wl.ph, wl.pw, wl.d)
    qr = np.ascontiguousarray(np.broadcast_to(qr[:, :, :, :1], qr.shape)).reshape(q.shape)
    sim = svg.svg_row_similarity(to_device(qr), to_device(k), wl.F, wl.ph, wl.pw).cpu().numpy()
    assert (np.abs(sim - 1.0) <= sim_tol(wl)).all(), sim
    assert (sim > 0.87).all()
    want = O.row_similarity(head64(qr, 0, 0), head64(k, 0, 0), wl.F, wl.ph, wl.pw)
    assert want == pytest.approx(1.0, abs=1e-12)


def test_row_similarity_full_sampled(full_inputs):
    name = "cogvideox"
    wl = si.WORKLOADS[name]
    (q, k, _), (qd, kd, _), types = full_inputs(name)
    frames = torch.tensor([6], dtype=torch.int32, device=DEV)
    sim = svg.svg_row_similarity(qd, kd, wl.F, wl.ph, wl.pw, frames).cpu().numpy()
    for h in (0, int(np.flatnonzero(types == 1)[0]), wl.H - 1):
        want = O.row_similarity(head64(q, 0, h), head64(k, 0, h), wl.F, wl.ph, wl.pw, [6])
        assert abs(sim[h] - want) <= sim_tol(wl), (h, sim[h], want)


def test_anchor_lists_bit_exact():
    wl = si.small("cogvideox")
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    nb = svg.n_tiles(wl.N)
    rng = np.random.default_rng(5)
    H = 12
    lid = rng.integers(0, 3, size=H).astype(np.int32)
    rep = rng.integers(0, 2, size=H).astype(np.int32)
    alists, ids = svg.svg_anchor_lists(lists, wl.N, wl.F, wl.ph, wl.pw,
                                       torch.from_numpy(lid).to(DEV),
                                       torch.from_numpy(rep).to(DEV), skip_list=1)
    ip = alists.indptr.cpu().numpy().reshape(6, nb + 1)
    ix = alists.indices.cpu().numpy()
    for c in range(6):
        kind = c % 3
        op, ox = O.geometric_block_lists(kind, wl.F, wl.P, wl.width, wl.N)
        if c >= 3:
            op, ox = O.anchor_tile_lists(op, ox, wl.F, wl.ph, wl.pw, 5)
        np.testing.assert_array_equal(ip[c] - ip[c][0], op)
        np.testing.assert_array_equal(ix[ip[c][0]:ip[c][-1]], ox)
    want = np.where((rep != 0) & (lid != 1), lid + 3, lid)
    np.testing.assert_array_equal(ids.cpu().numpy(), want)
    # lists alone, then the ids alone, give the same
    only, none = svg.svg_anchor_lists(lists, wl.N, wl.F, wl.ph, wl.pw)
    assert none is None
    np.testing.assert_array_equal(only.indptr.cpu().numpy(), alists.indptr.cpu().numpy())
    n_used = int(ip[-1][-1])
    np.testing.assert_array_equal(only.indices.cpu().numpy()[:n_used], ix[:n_used])
    np.testing.assert_array_equal(only.tile_order.cpu().numpy(), alists.tile_order.cpu().numpy())
    ids2 = svg.svg_anchor_list_ids(torch.from_numpy(lid).to(DEV), torch.from_numpy(rep).to(DEV),
                                   3, skip_list=1)
    np.testing.assert_array_equal(ids2.cpu().numpy(), want)
    # pairing order: index order for the plain copies, tiles holding anchor
    # rows first for the anchor copies
    order = alists.tile_order.cpu().numpy().reshape(6, nb)
    on = O.anchor_token_mask(wl.F, wl.ph, wl.pw, 5)
    live = [i for i in range(nb) if on[O.tile_rows(i, wl.N)].any()]
    idle = [i for i in range(nb) if i not in live]
    for c in range(6):
        assert order[c].tolist() == (list(range(nb)) if c < 3 else live + idle)


def test_tile_order_changes_no_result():
    # the pairing order is scheduling only: outputs are bit-identical with and
    # without it, and an out-of-range entry is flagged, not faulted
    wl = si.small("wan480")
    (_, _, _), (qd, kd, vd), types = workload_tensors(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    mode = torch.from_numpy(types).to(DEV)
    rep = torch.ones(wl.H, dtype=torch.int32, device=DEV)
    alists, ids = svg.svg_anchor_lists(lists, wl.N, wl.F, wl.ph, wl.pw, mode, rep, skip_list=1)
    a = svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, ids, alists)
    b = svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, ids, alists._replace(tile_order=None))
    np.testing.assert_array_equal(bits(a), bits(b))
    rev = torch.flip(alists.tile_order.view(6, -1), dims=[1]).contiguous().view(-1)
    c = svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, ids, alists._replace(tile_order=rev))
    np.testing.assert_array_equal(bits(c), bits(b))
    bad = alists.tile_order.clone()
    bad[3 * svg.n_tiles(wl.N)] = 10 ** 6  # first slot of anchor list 3
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, ids, alists._replace(tile_order=bad),
                              status=status)
    assert status.item() & svg._lib.SVG_DEVICE_BAD_INDEX


def _greedy_pairing(rows, nq):
    """The pairing rule restated: the smallest unpaired tile takes the unpaired
    tile with the most key blocks in common (ties: the smaller index)."""
    taken = [False] * nq
    order = []
    for a in range(nq):
        if taken[a]:
            continue
        taken[a] = True
        order.append(a)
        best, best_c = -1, -1
        for c in range(nq):
            if not taken[c]:
                ov = len(rows[a] & rows[c])
                if ov > best:
                    best, best_c = ov, c
        if best_c >= 0:
            taken[best_c] = True
            order.append(best_c)
    return order


def test_pair_query_tiles_on_calibrated_lists():
    """svg_pair_query_tiles: each row a permutation equal to the greedy rule,
    more shared key blocks per work item than index pairs on the heads that
    attend along time, and attention results bit-identical with the order."""
    wl = si.small("wan720")
    types_seed = wl.calib_seeds[0]
    E = []
    for s in wl.calib_seeds:
        (_, _, _), (qd, kd, _), _ = workload_tensors(wl, seed=s, types_seed=types_seed)
        E.append(svg.svg_block_energy(qd, kd))
    lists = svg.svg_build_block_mask_calibrated(torch.stack(E).contiguous(), wl.eps, wl.rho)
    nq = svg.n_tiles(wl.N)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    paired = svg.svg_pair_query_tiles(lists, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    order = paired.tile_order.cpu().numpy().reshape(wl.H, nq)
    ip = lists.indptr.cpu().numpy().reshape(wl.H, nq + 1)
    ix = lists.indices.cpu().numpy()
    shared_idx = shared_paired = 0
    for h in range(wl.H):
        assert sorted(order[h].tolist()) == list(range(nq))
        rows = [set(ix[ip[h][r]:ip[h][r + 1]].tolist()) for r in range(nq)]
        assert order[h].tolist() == _greedy_pairing(rows, nq)
        for i in range(0, nq - 1, 2):
            shared_idx += len(rows[i] & rows[i + 1])
            shared_paired += len(rows[order[h][i]] & rows[order[h][i + 1]])
    assert shared_paired >= shared_idx
    (_, _, _), (qd, kd, vd), _ = workload_tensors(wl, seed=wl.seed, types_seed=types_seed)
    list_id = torch.arange(wl.H, dtype=torch.int32, device=DEV)
    a = svg.svg_sparse_attn(qd, kd, vd, list_id, lists)
    b = svg.svg_sparse_attn_fused(qd, kd, vd, wl.F, wl.P, list_id, paired, layout=0)
    np.testing.assert_array_equal(bits(a), bits(b))


def test_attention_from_host_matches_device_call():
    """The host-streamed attention (chunks of heads, copies overlapped) gives
    the device call's bits, with and without a pairing order."""
    wl = si.small("wan720")
    (_, _, _), (qd, kd, vd), _ = workload_tensors(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    list_id = torch.tensor([h % 3 for h in range(wl.H)], dtype=torch.int32, device=DEV)
    vexp = svg.svg_v_exponents(vd)
    ref = bits(svg.svg_sparse_attn(qd, kd, vd, list_id, lists, v_exp=vexp))
    host = [x.cpu().pin_memory() for x in (qd, kd, vd)]
    for ls in (lists, svg.svg_pair_query_tiles(lists)):
        for hc in (1, 2, wl.H):
            out = svg.svg_attention_from_host(*host, list_id, ls, heads_per_chunk=hc)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(bits(out), ref)


def test_pair_query_tiles_edges():
    """One tile; an odd count; empty rows; a row set shared by far-apart tiles;
    an out-of-range index is skipped and flagged."""
    def run(rows, nk):
        nq = len(rows)
        indptr = np.zeros(nq + 1, np.int32)
        indptr[1:] = np.cumsum([len(r) for r in rows])
        flat = [c for r in rows for c in r] or [0]
        lists = svg.BlockLists(torch.from_numpy(indptr).to(DEV),
                               torch.tensor(flat, dtype=torch.int32, device=DEV), 1, nq)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        out = svg.svg_pair_query_tiles(lists, nk, status=status)
        torch.cuda.synchronize()
        return out.tile_order.cpu().numpy().tolist(), status.item()
    assert run([[0, 1]], 2) == ([0], 0)
    assert run([[0], [1], [2]], 3) == ([0, 1, 2], 0)
    assert run([[], [], [], []], 1) == ([0, 1, 2, 3], 0)
    # tile 0 and tile 3 keep the same blocks, as do 1 and 2
    assert run([[0, 5, 9], [2, 3], [2, 3], [0, 5, 9]], 10) == ([0, 3, 1, 2], 0)
    order, st = run([[0, 40], [1], [0]], 8)
    assert sorted(order) == [0, 1, 2] and st & svg._lib.SVG_DEVICE_BAD_INDEX


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_row_broadcast_bit_exact(dtype):
    wl = si.small("hunyuan720")
    g = torch.Generator().manual_seed(3)
    o = torch.randn(wl.B, wl.H, wl.N, wl.d, generator=g).to(dtype).to(DEV)
    ids = torch.tensor([0, 4, 2, 5], dtype=torch.int32, device=DEV)  # heads 1, 3 repeat
    want = o.clone()
    svg.svg_row_broadcast(o, wl.F, wl.ph, wl.pw, ids, 3)
    got, ref = bits(o), bits(want)
    for h in range(wl.H):
        exp = ref[0, h]
        if h in (1, 3):
            exp = O.broadcast_rows(exp, wl.F, wl.ph, wl.pw, 5)
        np.testing.assert_array_equal(got[0, h], exp)


@pytest.mark.parametrize("wl", [si.small(n) for n in ("tiny", "cogvideox", "wan720")],
                         ids=lambda w: w.name)
def test_repeat_attention_small(wl):
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    lid = np.resize(np.array([0, 2, 0, 0], dtype=np.int32), wl.H)   # spatial / dense lists
    rep = np.resize(np.array([1, 1, 0, 1], dtype=np.int32), wl.H)
    o = svg.svg_repeat_attention(qd, kd, vd, wl.F, wl.ph, wl.pw, torch.from_numpy(lid).to(DEV),
                                 lists, torch.from_numpy(rep).to(DEV))
    for h in range(wl.H):
        ip, ix = O.geometric_block_lists(int(lid[h]), wl.F, wl.P, wl.width, wl.N)
        q64, k64, v64 = head64(q, 0, h), head64(k, 0, h), head64(v, 0, h)
        if rep[h]:
            ref = O.repeat_head_attention(q64, k64, v64, ip, ix, wl.F, wl.ph, wl.pw, 5)
        else:
            ref = O.block_sparse_attention(q64, k64, v64, ip, ix)
        assert_close(to_float64(o[0, h]), ref, f"{wl.name} head {h}", bf16=wl.dtype == "bf16")


@pytest.mark.parametrize("overlap", [True, False])
def test_layer_small_with_repeat(overlap):
    wl = si.small("cogvideox")
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    idx = si.sample_queries(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    rep = np.array([1, 1, 0, 1], dtype=np.int32)
    o, mode, mse = svg.svg_layer(qd, kd, vd, wl.F, wl.P, wl.width, torch.from_numpy(idx).to(DEV),
                                 lists, overlap=overlap, repeat=torch.from_numpy(rep).to(DEV),
                                 frame_shape=(wl.ph, wl.pw))
    o_ref, mode_ref, mse_ref = O.svg_layer(si.as_float64(q), si.as_float64(k), si.as_float64(v),
                                           idx, wl.F, wl.P, wl.width)
    np.testing.assert_array_equal(mode.cpu().numpy(), mode_ref)
    for h in range(wl.H):
        ref = o_ref[0, h]
        if rep[h] and mode_ref[h] != O.MODE_TEMPORAL:
            ref = O.broadcast_rows(ref, wl.F, wl.ph, wl.pw, 5)
        assert_close(to_float64(o[0, h]), ref, f"layer head {h}")


def test_layer_small_with_qk_norm_rope_and_repeat():
    wl = si.small("wan480")
    (q, k, v), (qd, kd, vd), _ = workload_tensors(wl)
    gq, gk = si.qk_norm_weights(wl)
    cos, sin = si.rope_tables(wl)
    dev = lambda a: torch.from_numpy(a).to(DEV)
    qk = svg.QKTransform(dev(gq), dev(gk), 1e-6, dev(cos), dev(sin))
    idx = si.sample_queries(wl)
    lists = svg.geometric_lists(wl.F, wl.P, wl.width, wl.N)
    rep = np.array([1, 0, 1, 1], dtype=np.int32)
    o, mode, mse = svg.svg_layer(qd, kd, vd, wl.F, wl.P, wl.width, torch.from_numpy(idx).to(DEV),
                                 lists, qk=qk, repeat=dev(rep), frame_shape=(wl.ph, wl.pw))
    o_ref, mode_ref, mse_ref = O.svg_layer(si.as_float64(q), si.as_float64(k), si.as_float64(v),
                                           idx, wl.F, wl.P, wl.width, qk=(gq, gk, 1e-6, cos, sin),
                                           qk_bf16=True)
    check_profile(mse.cpu().numpy(), mode.cpu().numpy(), mse_ref, mode_ref, wl.name)
    m = mode.cpu().numpy()
    for h in range(wl.H):
        if m[h] != mode_ref[h]:
            continue  # a near tie decided the other way (checked above)
        ref = o_ref[0, h]
        if rep[h] and m[h] != O.MODE_TEMPORAL:
            ref = O.broadcast_rows(ref, wl.F, wl.ph, wl.pw, 5)
        assert_close(to_float64(o[0, h]), ref, f"head {h}")
