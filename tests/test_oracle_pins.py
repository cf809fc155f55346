"""Pins of the float64 oracle to things other than itself: library routines
(torch scaled_dot_product_attention in float64), closed forms, invariants,
brute force on tiny inputs and hand-worked examples under tests/golden/.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, index or axis, a transposed operand, '>' for '>=') fails it."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import svg_inputs as si
from oracle import svg_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def sdpa64(q, k, v, mask=None, scale=None):
    """torch's own attention in float64 (library cross-check)."""
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))[None, None]
    m = None if mask is None else torch.from_numpy(np.asarray(mask, bool))[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m,
                                                         scale=scale)
    return o[0, 0].numpy()


def rand(shape, seed=0, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------- O1 / O2

class TestDenseAttention:
    def test_matches_torch_sdpa(self):
        q, k, v = rand((37, 64), 1, 2.0), rand((91, 64), 2, 2.0), rand((91, 64), 3)
        np.testing.assert_allclose(O.dense_attention(q, k, v), sdpa64(q, k, v), atol=1e-12)

    def test_non_square_head_dim_and_scale(self):
        q, k, v = rand((5, 128), 4), rand((300, 128), 5), rand((300, 128), 6)
        np.testing.assert_allclose(O.dense_attention(q, k, v, scale=0.3),
                                   sdpa64(q, k, v, scale=0.3), atol=1e-12)

    def test_default_scale_is_inverse_sqrt_d(self):
        assert O.softmax_scale(64) == 0.125
        q, k, v = rand((3, 16), 7), rand((20, 16), 8), rand((20, 16), 9)
        np.testing.assert_allclose(O.dense_attention(q, k, v),
                                   O.dense_attention(q, k, v, scale=0.25), atol=0)

    def test_zero_query_gives_mean_of_values(self):
        k, v = rand((50, 32), 10), rand((50, 32), 11)
        o = O.dense_attention(np.zeros((4, 32)), k, v)
        np.testing.assert_allclose(o, np.broadcast_to(v.mean(0), o.shape), atol=1e-13)

    def test_constant_values_pass_through(self):
        q, k = rand((6, 32), 12, 3.0), rand((40, 32), 13, 3.0)
        v = np.tile(rand((1, 32), 14), (40, 1))
        np.testing.assert_allclose(O.dense_attention(q, k, v), np.tile(v[:1], (6, 1)), atol=1e-12)

    def test_two_key_closed_form(self):
        q = np.array([[1.0, 0.0]])
        k = np.array([[1.0, 0.0], [0.0, 1.0]])
        v = np.array([[2.0, -1.0], [4.0, 3.0]])
        p0 = math.e / (math.e + 1.0)
        want = p0 * v[0] + (1 - p0) * v[1]
        np.testing.assert_allclose(O.dense_attention(q, k, v, scale=1.0)[0], want, atol=1e-15)

    def test_probabilities_rows_sum_to_one_and_large_logits(self):
        q, k = rand((8, 64), 15, 30.0), rand((70, 64), 16, 30.0)
        p = O.attention_probs(q, k, 0.125)
        assert np.isfinite(p).all()
        np.testing.assert_allclose(p.sum(1), 1.0, atol=1e-13)


class TestMaskedAttention:
    def test_all_true_equals_dense(self):
        q, k, v = rand((9, 64), 20), rand((33, 64), 21), rand((33, 64), 22)
        np.testing.assert_allclose(O.masked_attention(q, k, v, np.ones((9, 33), bool)),
                                   O.dense_attention(q, k, v), atol=1e-13)

    def test_matches_torch_sdpa_bool_mask(self):
        q, k, v = rand((16, 64), 23, 2), rand((64, 64), 24, 2), rand((64, 64), 25)
        mask = np.random.default_rng(26).random((16, 64)) < 0.3
        mask[:, 0] = True
        np.testing.assert_allclose(O.masked_attention(q, k, v, mask), sdpa64(q, k, v, mask),
                                   atol=1e-12)

    def test_single_key_returns_that_value(self):
        q, k, v = rand((3, 8), 27), rand((10, 8), 28), rand((10, 8), 29)
        mask = np.zeros((3, 10), bool)
        mask[0, 4] = mask[1, 7] = mask[2, 0] = True
        o = O.masked_attention(q, k, v, mask)
        np.testing.assert_allclose(o, v[[4, 7, 0]], atol=0)

    def test_empty_row_is_zero(self):
        q, k, v = rand((2, 8), 30), rand((5, 8), 31), rand((5, 8), 32)
        mask = np.zeros((2, 5), bool)
        mask[1, 2] = True
        o = O.masked_attention(q, k, v, mask)
        assert (o[0] == 0).all()
        np.testing.assert_allclose(o[1], v[2], atol=0)


# ---------------------------------------------------------------- O3

class TestTokenMasks:
    def test_golden_F3_P2(self):
        g = golden("token_masks_F3_P2.json")
        n = np.arange(g["F"] * g["P"])
        np.testing.assert_array_equal(O.spatial_mask(n, n, g["P"], g["width"]),
                                      np.array(g["spatial"], bool))
        np.testing.assert_array_equal(O.temporal_mask_frame_major(n, n, g["P"]),
                                      np.array(g["temporal_frame_major"], bool))

    @pytest.mark.parametrize("F,P", [(4, 3), (5, 7), (1, 6), (6, 1)])
    def test_temporal_mask_commutes_with_permutation(self, F, P):
        # the token-major temporal mask is the frame-major one read through the map
        src = O.token_major_source(F, P)
        m = np.arange(F * P)
        np.testing.assert_array_equal(O.temporal_mask_token_major(m, m, F),
                                      O.temporal_mask_frame_major(src, src, P))

    def test_spatial_width_covers_everything(self):
        n = np.arange(4 * 5)
        assert O.spatial_mask(n, n, 5, 3).all()
        assert not O.spatial_mask(n, n, 5, 2).all()


# ---------------------------------------------------------------- O5

class TestPermutation:
    def test_golden_F3_P4(self):
        g = golden("permutation_F3_P4.json")
        np.testing.assert_array_equal(O.token_major_source(g["F"], g["P"]),
                                      g["token_major_source"])
        x = np.arange(12, dtype=np.float64).reshape(12, 1)
        np.testing.assert_array_equal(O.permute_token_major(x, 3, 4)[:, 0],
                                      g["token_major_source"])

    @pytest.mark.parametrize("F,P", [(13, 7), (4, 64), (1, 9), (9, 1), (21, 5)])
    def test_bijection_inverse_and_closed_form(self, F, P):
        N = F * P
        src = O.token_major_source(F, P)
        np.testing.assert_array_equal(np.sort(src), np.arange(N))
        m = np.arange(N)
        np.testing.assert_array_equal(src, (m % F) * P + m // F)
        x = np.random.default_rng(F * 100 + P).standard_normal((2, 3, N, 4))
        y = O.permute_token_major(x, F, P)
        np.testing.assert_array_equal(y, x[..., src, :])
        np.testing.assert_array_equal(O.permute_frame_major(y, F, P), x)
        np.testing.assert_array_equal(O.permute_token_major(O.permute_frame_major(x, F, P), F, P), x)

    def test_identity_cases(self):
        x = rand((10, 3), 40)
        np.testing.assert_array_equal(O.permute_token_major(x, 1, 10), x)
        np.testing.assert_array_equal(O.permute_token_major(x, 10, 1), x)

    def test_temporal_stripes_become_contiguous(self):
        # after the transform, the keys a temporal row sees are one contiguous run
        F, P = 6, 11
        src = O.token_major_source(F, P)
        for m in range(F * P):
            cols = np.nonzero(O.temporal_mask_frame_major(src[m:m + 1], src, P)[0])[0]
            assert cols[-1] - cols[0] + 1 == len(cols) == F


# ---------------------------------------------------------------- O7

def brute_lists(mask, N, T):
    nb = (N + T - 1) // T
    indptr, indices = [0], []
    for i in range(nb):
        for j in range(nb):
            if mask[i * T:(i + 1) * T, j * T:(j + 1) * T].any():
                indices.append(j)
        indptr.append(len(indices))
    return np.array(indptr), np.array(indices)


def closed_form_lists(kind, F, P, w, N, T):
    """Interval overlap: rows of tile i span frames (or positions) [a_i, b_i]."""
    nb = (N + T - 1) // T
    div = P if kind == O.MODE_SPATIAL else F
    lo = [i * T // div for i in range(nb)]
    hi = [(min(N, (i + 1) * T) - 1) // div for i in range(nb)]
    ww = w if kind == O.MODE_SPATIAL else 0
    indptr, indices = [0], []
    for i in range(nb):
        for j in range(nb):
            if kind == O.MODE_DENSE or (lo[j] <= hi[i] + ww and hi[j] >= lo[i] - ww):
                indices.append(j)
        indptr.append(len(indices))
    return np.array(indptr), np.array(indices)


class TestGeometricLists:
    def test_golden_small_tile(self):
        g = golden("block_lists_F3_P5_T4.json")
        F, P, N, T = g["F"], g["P"], g["N"], g["T"]
        for key, kind, w in [("spatial_w0", O.MODE_SPATIAL, 0), ("spatial_w1", O.MODE_SPATIAL, 1),
                             ("temporal", O.MODE_TEMPORAL, 0)]:
            ip, ix = O.geometric_block_lists(kind, F, P, w, N, T)
            np.testing.assert_array_equal(ip, g[key]["indptr"])
            np.testing.assert_array_equal(ix, g[key]["indices"])

    @pytest.mark.parametrize("F,P,w,T", [(3, 5, 1, 4), (4, 7, 1, 8), (5, 9, 2, 16), (7, 3, 0, 5),
                                         (2, 40, 1, 32), (13, 11, 1, 128), (6, 50, 1, 128)])
    def test_brute_force_and_closed_form(self, F, P, w, T):
        N = F * P
        n = np.arange(N)
        src = O.token_major_source(F, P)
        masks = {O.MODE_SPATIAL: O.spatial_mask(n, n, P, w),
                 O.MODE_TEMPORAL: O.temporal_mask_frame_major(src, src, P),
                 O.MODE_DENSE: np.ones((N, N), bool)}
        for kind, M in masks.items():
            ip, ix = O.geometric_block_lists(kind, F, P, w, N, T)
            bp, bx = brute_lists(M, N, T)
            np.testing.assert_array_equal(ip, bp)
            np.testing.assert_array_equal(ix, bx)
            cp, cx = closed_form_lists(kind, F, P, w, N, T)
            np.testing.assert_array_equal(ip, cp)
            np.testing.assert_array_equal(ix, cx)

    @pytest.mark.parametrize("F,P,w", [(13, 1350, 1), (21, 1560, 1), (33, 3600, 2)])
    def test_closed_form_at_workload_shapes(self, F, P, w):
        N = F * P
        for kind in (O.MODE_SPATIAL, O.MODE_TEMPORAL):
            ip, ix = O.geometric_block_lists(kind, F, P, w, N)
            cp, cx = closed_form_lists(kind, F, P, w, N, 128)
            np.testing.assert_array_equal(ip, cp)
            np.testing.assert_array_equal(ix, cx)

    def test_wide_band_keeps_everything_and_diagonal_always_kept(self):
        F, P = 5, 33
        N = F * P
        ip, ix = O.geometric_block_lists(O.MODE_SPATIAL, F, P, F - 1, N, 16)
        dp, dx = O.geometric_block_lists(O.MODE_DENSE, F, P, 0, N, 16)
        np.testing.assert_array_equal(ip, dp)
        np.testing.assert_array_equal(ix, dx)
        for kind in (O.MODE_SPATIAL, O.MODE_TEMPORAL):
            ip, ix = O.geometric_block_lists(kind, F, P, 0, N, 16)
            for i in range(len(ip) - 1):
                assert i in ix[ip[i]:ip[i + 1]]
                assert (np.diff(ix[ip[i]:ip[i + 1]]) > 0).all()

    def test_block_mask_contains_token_mask(self):
        F, P, w, T = 4, 37, 1, 32
        N = F * P
        n = np.arange(N)
        ip, ix = O.geometric_block_lists(O.MODE_SPATIAL, F, P, w, N, T)
        MB = O.block_mask_from_lists(ip, ix, N, T)
        assert (MB | ~O.spatial_mask(n, n, P, w)).all()


# ---------------------------------------------------------------- O8

def kron_mask(indptr, indices, N, T):
    nb = len(indptr) - 1
    tiles = np.zeros((nb, nb), bool)
    for i in range(nb):
        tiles[i, indices[indptr[i]:indptr[i + 1]]] = True
    return np.kron(tiles, np.ones((T, T), bool))[:N, :N]


class TestBlockSparseAttention:
    def test_all_kept_equals_dense(self):
        N, T = 300, 64
        q, k, v = rand((N, 64), 50, 2), rand((N, 64), 51, 2), rand((N, 64), 52)
        ip, ix = O.geometric_block_lists(O.MODE_DENSE, 1, N, 0, N, T)
        np.testing.assert_allclose(O.block_sparse_attention(q, k, v, ip, ix, T), sdpa64(q, k, v),
                                   atol=1e-12)

    def test_geometric_lists_match_sdpa_with_tile_mask(self):
        F, P, w, T = 5, 41, 1, 32
        N = F * P
        q, k, v = rand((N, 32), 53, 2), rand((N, 32), 54, 2), rand((N, 32), 55)
        ip, ix = O.geometric_block_lists(O.MODE_SPATIAL, F, P, w, N, T)
        np.testing.assert_allclose(O.block_sparse_attention(q, k, v, ip, ix, T),
                                   sdpa64(q, k, v, kron_mask(ip, ix, N, T)), atol=1e-12)
        rows = np.array([0, 31, 32, 150, N - 1])
        np.testing.assert_allclose(O.block_sparse_rows(q, k, v, rows, ip, ix, T),
                                   sdpa64(q, k, v, kron_mask(ip, ix, N, T))[rows], atol=1e-12)

    def test_empty_list_gives_zero_rows_and_ragged_tail(self):
        N, T = 70, 32                       # tiles of 32, 32, 6 rows
        q, k, v = rand((N, 16), 56), rand((N, 16), 57), rand((N, 16), 58)
        ip = np.array([0, 1, 1, 3])
        ix = np.array([2, 0, 2])
        o = O.block_sparse_attention(q, k, v, ip, ix, T)
        assert (o[32:64] == 0).all()
        # tile 0 sees only the 6 keys of the ragged last tile
        np.testing.assert_allclose(o[:32], O.dense_attention(q[:32], k[64:], v[64:]), atol=1e-13)
        keys = np.r_[0:32, 64:70]
        np.testing.assert_allclose(o[64:], O.dense_attention(q[64:], k[keys], v[keys]), atol=1e-13)


# ---------------------------------------------------------------- O4

def brute_profile(q, k, v, idx, P, w):
    """Full N x N attention for each mask through torch, then the sampled rows."""
    N = q.shape[0]
    sp = np.zeros((N, N), bool)
    tp = np.zeros((N, N), bool)
    for i in range(N):
        for j in range(N):
            sp[i, j] = abs(i // P - j // P) <= w
            tp[i, j] = (i % P) == (j % P)
    od = sdpa64(q, k, v)[idx]
    os_ = sdpa64(q, k, v, sp)[idx]
    ot = sdpa64(q, k, v, tp)[idx]
    return ((os_ - od) ** 2).mean(), ((ot - od) ** 2).mean()


class TestProfiling:
    def test_brute_force_on_tiny_workload(self):
        wl = si.WORKLOADS["tiny"]
        q, k, v, types = si.generate(wl)
        idx = si.sample_queries(wl)
        for h in range(wl.H):
            qh, kh, vh = (si.as_float64(t[0, h]) for t in (q, k, v))
            ms, mt, mode = O.profile_head(qh, kh, vh, idx, wl.F, wl.P, wl.width)
            bs, bt = brute_profile(qh, kh, vh, idx, wl.P, wl.width)
            assert ms == pytest.approx(bs, rel=1e-10, abs=1e-15)
            assert mt == pytest.approx(bt, rel=1e-10, abs=1e-15)

    def test_designed_labels_with_margin(self):
        wl = si.WORKLOADS["tiny"]
        q, k, v, types = si.generate(wl)
        idx = si.sample_queries(wl)
        mse, mode = O.profile_heads(*(si.as_float64(t) for t in (q, k, v)), idx, wl.F, wl.P,
                                    wl.width)
        assert list(types) == [si.SPATIAL_TYPE, si.TEMPORAL_TYPE]
        assert list(mode) == [O.MODE_SPATIAL, O.MODE_TEMPORAL]
        assert mse[0, 1] > 10 * mse[0, 0]
        assert mse[1, 0] > 10 * mse[1, 1]

    def test_tie_goes_to_spatial_and_constant_v(self):
        N, P, F = 24, 6, 4
        q, k = rand((N, 8), 60), rand((N, 8), 61)
        ms, mt, mode = O.profile_head(q, k, np.zeros((N, 8)), np.array([0, 5, 13]), F, P, 1)
        assert ms == 0 and mt == 0 and mode == O.MODE_SPATIAL
        ms, mt, mode = O.profile_head(q, k, np.ones((N, 8)), np.array([0, 5, 13]), F, P, 1)
        assert ms < 1e-28 and mt < 1e-28

    def test_designed_labels_small_workloads(self):
        for name in ("cogvideox", "wan480", "hunyuan720"):
            wl = si.small(name)
            q, k, v, types = si.generate(wl)
            idx = si.sample_queries(wl)
            mse, mode = O.profile_heads(*(si.as_float64(t) for t in (q, k, v)), idx, wl.F,
                                        wl.P, wl.width)
            np.testing.assert_array_equal(mode, types)


# ---------------------------------------------------------------- O9

class TestCalibration:
    def test_golden_minimal_sets(self):
        for case in golden("calibration_examples.json")["minimal_set"]:
            assert O.minimal_energy_set(case["energy"], case["eps"]) == case["kept"]

    def test_golden_votes(self):
        for case in golden("calibration_examples.json")["vote"]:
            E = [np.array([row]) for row in case["energies"]]
            ip, ix = O.calibrate_lists(E, case["eps"], case["rho"])
            np.testing.assert_array_equal(ip, [0, len(case["kept"])])
            np.testing.assert_array_equal(ix, case["kept"])

    def test_minimality_against_exhaustive_search(self):
        rng = np.random.default_rng(70)
        for trial in range(60):
            nb = int(rng.integers(1, 9))
            e = rng.dirichlet(np.ones(nb) * 0.5)
            eps = float(rng.uniform(0.3, 0.99))
            kept = O.minimal_energy_set(e, eps)
            assert e[kept].sum() >= eps or len(kept) == nb
            best = min(len(s) for r in range(1, nb + 1)
                       for s in itertools.combinations(range(nb), r) if e[list(s)].sum() >= eps)
            assert len(kept) == best
            # dropping the smallest kept block falls below eps
            if len(kept) > 1:
                assert e[kept].sum() - e[kept].min() < eps

    def test_single_input_returns_its_sets_and_eps_one_keeps_all_nonzero(self):
        rng = np.random.default_rng(71)
        E = rng.dirichlet(np.ones(7), size=5)
        ip, ix = O.calibrate_lists([E], 0.8, 0.5)
        for r in range(5):
            assert list(ix[ip[r]:ip[r + 1]]) == O.minimal_energy_set(E[r], 0.8)
        E[:, 3] = 0.0
        E = E / E.sum(1, keepdims=True)
        ip, ix = O.calibrate_lists([E], 1.0 - 1e-12, 0.5)
        for r in range(5):
            assert list(ix[ip[r]:ip[r + 1]]) == [0, 1, 2, 4, 5, 6]

    def test_energy_matches_torch_softmax_and_rows_sum_to_one(self):
        N, T, d = 200, 64, 32
        q, k = rand((N, d), 72, 2), rand((N, d), 73, 2)
        E = O.block_energy(q, k, T)
        p = torch.softmax(torch.from_numpy(q @ k.T) / math.sqrt(d), dim=-1).numpy()
        nb = 4
        pad = np.zeros((nb * T, nb * T))
        pad[:N, :N] = p
        sums = pad.reshape(nb, T, nb, T).sum(axis=(1, 3))
        counts = np.array([64, 64, 64, 8])[:, None]
        np.testing.assert_allclose(E, sums / counts, atol=1e-13)
        np.testing.assert_allclose(E.sum(1), 1.0, atol=1e-13)
        # a subset of query blocks, in the order asked for
        Er = O.block_energy(q, k, T, row_blocks=[3, 0])
        np.testing.assert_allclose(Er, (sums / counts)[[3, 0]], atol=1e-13)

    def test_energy_uniform_for_zero_queries(self):
        N, T = 150, 64
        E = O.block_energy(np.zeros((N, 8)), rand((N, 8), 74), T)
        np.testing.assert_allclose(E, np.tile(np.array([64, 64, 22]) / N, (3, 1)), atol=1e-14)


# ---------------------------------------------------------------- whole layer

def test_layer_composes_steps_on_tiny():
    wl = si.WORKLOADS["tiny"]
    q, k, v, _ = (si.generate(wl)[i] for i in range(4))
    q64, k64, v64 = (si.as_float64(t) for t in (q, k, v))
    idx = si.sample_queries(wl)
    o, mode, mse = O.svg_layer(q64, k64, v64, idx, wl.F, wl.P, wl.width)
    # head 0 is spatial: N = 256 is two tiles spanning frames {0,1} and {2,3},
    # so the band |f - f'| <= 1 touches both tiles and the head is dense
    np.testing.assert_allclose(o[0, 0], sdpa64(q64[0, 0], k64[0, 0], v64[0, 0]), atol=1e-12)
    # head 1 is temporal: token-major tiles of 128 rows hold positions 0-31 and
    # 32-63, each tile sees only itself, i.e. keys of the same half of positions
    P = wl.P
    n = np.arange(wl.N)
    half = (n % P) // 32
    M = half[:, None] == half[None, :]
    np.testing.assert_allclose(o[0, 1], sdpa64(q64[0, 1], k64[0, 1], v64[0, 1], M), atol=1e-12)


# ------------------------------------------- eps(t) schedule and mask encodings

def random_lists(rows, n_cols, seed):
    rng = np.random.default_rng(seed)
    ip, ix = [0], []
    for _ in range(rows):
        k = int(rng.integers(0, n_cols + 1))
        ix.extend(sorted(rng.choice(n_cols, size=k, replace=False).tolist()))
        ip.append(len(ix))
    return np.asarray(ip, np.int32), np.asarray(ix, np.int32)


class TestScheduleAndEncodings:
    def test_schedule_end_values_and_exponential_shape(self):
        e = O.epsilon_schedule(50)
        assert e[0] == pytest.approx(0.99, abs=1e-15) and e[-1] == pytest.approx(0.84, abs=1e-15)
        assert (np.diff(e) < 0).all()
        # exponential decay: constant ratio between consecutive steps, and the
        # log is linear in the step index
        r = e[1:] / e[:-1]
        np.testing.assert_allclose(r, (0.84 / 0.99) ** (1 / 49), rtol=1e-13)
        np.testing.assert_allclose(np.diff(np.log(e), 2), 0.0, atol=1e-13)
        assert O.epsilon_schedule(1).tolist() == [0.99]
        assert O.epsilon_schedule(0).size == 0
        np.testing.assert_allclose(O.epsilon_schedule(3, 0.9, 0.9), 0.9, rtol=1e-15)

    def test_golden_intervals_and_bitmap(self):
        g = golden("mask_encodings.json")
        ip, ix = np.asarray(g["indptr"]), np.asarray(g["indices"])
        iptr, st, en = O.lists_to_intervals(ip, ix)
        assert iptr.tolist() == g["intervals"]["iptr"]
        assert st.tolist() == g["intervals"]["starts"]
        assert en.tolist() == g["intervals"]["ends"]
        bm = O.lists_to_bitmap(ip, ix, g["n_cols"])
        assert [[f"0x{int(w):08x}" for w in row] for row in bm] == g["bitmap_hex"]

    def test_round_trips_on_random_sets(self):
        for seed in range(20):
            n_cols = [1, 31, 32, 33, 64, 138, 591][seed % 7]
            ip, ix = random_lists(9, n_cols, seed)
            iptr, st, en = O.lists_to_intervals(ip, ix)
            ip2, ix2 = O.intervals_to_lists(iptr, st, en)
            assert ip2.tolist() == ip.tolist() and ix2.tolist() == ix.tolist()
            # maximal runs: no two intervals of a row touch
            for r in range(len(iptr) - 1):
                for t in range(iptr[r] + 1, iptr[r + 1]):
                    assert st[t] > en[t - 1]
            bm = O.lists_to_bitmap(ip, ix, n_cols)
            ip3, ix3 = O.bitmap_to_lists(bm, n_cols)
            assert ip3.tolist() == ip.tolist() and ix3.tolist() == ix.tolist()
            # popcount of the bitmap = number of kept blocks
            assert sum(bin(int(w)).count("1") for w in bm.ravel()) == len(ix)

    def test_bitmap_is_32x_smaller_than_an_int32_mask(self):
        # [CAL] 3.3: bitmap storage of the mask takes 32x less memory than one
        # 32-bit value per (query block, key block)
        for n_cols in (32, 64, 640):
            ip, ix = random_lists(5, n_cols, n_cols)
            bm = O.lists_to_bitmap(ip, ix, n_cols)
            assert bm.nbytes * 32 == 5 * n_cols * 4

    def test_duplicates_and_unsorted_rows_become_sets(self):
        iptr, st, en = O.lists_to_intervals(np.array([0, 5]), np.array([4, 2, 3, 3, 9]))
        assert st.tolist() == [2, 9] and en.tolist() == [5, 10]


# ------------------------------------------------------- QK-Norm and RoPE

class TestQkNormRope:
    def test_rms_norm_matches_torch(self):
        x = rand((7, 64), 1, 3.0)
        g = 1.0 + 0.3 * rand(64, 2)
        for eps in (0.0, 1e-6, 0.5):
            want = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,),
                                                weight=torch.from_numpy(g), eps=eps).numpy()
            np.testing.assert_allclose(O.qk_rms_norm(x, g, eps), want, rtol=1e-13, atol=1e-14)

    def test_rms_norm_closed_forms(self):
        x = rand((5, 128), 3, 7.0)
        y = O.qk_rms_norm(x, None, 0.0)
        np.testing.assert_allclose(np.mean(y * y, axis=1), 1.0, rtol=1e-13)
        # scale invariance without epsilon, and a constant row a -> a / sqrt(a^2 + eps)
        np.testing.assert_allclose(O.qk_rms_norm(4.5 * x, None, 0.0), y, rtol=1e-12)
        c = O.qk_rms_norm(np.full((1, 8), 3.0), None, 0.25)
        np.testing.assert_allclose(c, 3.0 / math.sqrt(9.25), rtol=1e-15)
        # the weight scales channel c alone
        g = np.arange(1, 129, dtype=np.float64)
        np.testing.assert_allclose(O.qk_rms_norm(x, g, 0.0), y * g, rtol=1e-13)

    def test_rope_matches_complex_multiplication(self):
        x = rand((9, 64), 4)
        ang = rand((9, 32), 5, 2.0)
        z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * ang)
        want = np.empty_like(x)
        want[:, 0::2], want[:, 1::2] = z.real, z.imag
        np.testing.assert_allclose(O.rope_rotate(x, np.cos(ang), np.sin(ang)), want,
                                   rtol=1e-12, atol=1e-13)

    def test_rope_closed_forms(self):
        x = rand((4, 16), 6)
        zero = np.zeros((4, 8))
        np.testing.assert_array_equal(O.rope_rotate(x, np.cos(zero), np.sin(zero)), x)
        a, b = rand((4, 8), 7), rand((4, 8), 8)
        y = O.rope_rotate(O.rope_rotate(x, np.cos(a), np.sin(a)), np.cos(b), np.sin(b))
        np.testing.assert_allclose(y, O.rope_rotate(x, np.cos(a + b), np.sin(a + b)),
                                   rtol=1e-12, atol=1e-13)
        # every pair keeps its length
        r = O.rope_rotate(x, np.cos(a), np.sin(a))
        np.testing.assert_allclose(r[:, 0::2] ** 2 + r[:, 1::2] ** 2,
                                   x[:, 0::2] ** 2 + x[:, 1::2] ** 2, rtol=1e-12)

    def test_rope_relative_position(self):
        # angles pos * freq: the score of a rotated query and key depends on
        # the position difference only
        d = 32
        freq = 10000.0 ** (-np.arange(d // 2) / (d // 2))
        tab = lambda pos: (np.cos(pos * freq)[None], np.sin(pos * freq)[None])
        q, k = rand((1, d), 9), rand((1, d), 10)
        s = lambda m, n: float((O.rope_rotate(q, *tab(m)) @ O.rope_rotate(k, *tab(n)).T)[0, 0])
        for m, n, t in ((3, 1, 5), (0, 7, 11), (20, 20, 3)):
            assert s(m, n) == pytest.approx(s(m + t, n + t), rel=1e-11)
        assert s(0, 0) == pytest.approx(float((q @ k.T)[0, 0]), rel=1e-12)

    def test_worked_example(self):
        # x = (1, 2, 3, 4): rms = sqrt(30 / 4); pair 0 turned by pi/2 maps
        # (a, b) -> (-b, a); pair 1 turned by pi maps (a, b) -> (-a, -b)
        x = np.array([[1.0, 2.0, 3.0, 4.0]])
        ang = np.array([[math.pi / 2, math.pi]])
        y = O.qk_norm_rope(x, None, 0.0, np.cos(ang), np.sin(ang))
        np.testing.assert_allclose(y, np.array([[-2.0, 1.0, -3.0, -4.0]]) / math.sqrt(7.5),
                                   rtol=1e-14, atol=1e-15)

    def test_norm_commutes_with_rope_at_unit_weight(self):
        # the rotation keeps every row's sum of squares, so with gamma = 1 the
        # two orders agree (up to cos^2 + sin^2 = 1 in the float32 tables);
        # with a non-uniform weight they do not
        wl = si.small("cogvideox")
        cos, sin = si.rope_tables(wl)
        x = rand((wl.N, wl.d), 11, 2.0)
        a = O.qk_norm_rope(x, None, 1e-6, cos, sin)
        b = O.qk_rms_norm(O.rope_rotate(x, cos, sin), None, 1e-6)
        np.testing.assert_allclose(a, b, rtol=1e-6, atol=1e-6)
        g = si.qk_norm_weights(wl)[0]
        a = O.qk_norm_rope(x, g, 1e-6, cos, sin)
        b = O.qk_rms_norm(O.rope_rotate(x, cos, sin), g, 1e-6)
        assert np.abs(a - b).max() > 1e-3

    def test_layer_with_unit_transform_is_the_plain_layer(self):
        wl = si.WORKLOADS["tiny"]
        q, k, v, _ = si.generate(wl)
        q, k, v = (si.as_float64(t) for t in (q, k, v))
        idx = si.sample_queries(wl)
        ones = np.ones((wl.N, wl.d // 2))
        zeros = np.zeros((wl.N, wl.d // 2))
        o1, m1, e1 = O.svg_layer(q, k, v, idx, wl.F, wl.P, wl.width,
                                 qk=(None, None, 0.0, ones, zeros))
        nrm = lambda t: torch.nn.functional.rms_norm(torch.from_numpy(t), (wl.d,)).numpy()
        o2, m2, e2 = O.svg_layer(nrm(q), nrm(k), v, idx, wl.F, wl.P, wl.width)
        np.testing.assert_array_equal(m1, m2)
        np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)

    def test_round_bf16(self):
        # library cross-check: torch's float32 -> bf16 cast (round to nearest
        # even) on float32 values, where no double rounding can occur
        x = (rand(4000, 12, 3.0) * np.exp(rand(4000, 13, 4.0))).astype(np.float32)
        want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
        np.testing.assert_array_equal(O.round_bf16(x.astype(np.float64)), want)
        # ties go to even; just above a tie goes up; sign symmetry; exact values stay
        u = 2.0 ** -8
        assert O.round_bf16(1 + u) == 1.0 and O.round_bf16(1 + 3 * u) == 1 + 4 * u
        assert O.round_bf16(1 + u * (1 + 2.0 ** -30)) == 1 + 2 * u
        assert O.round_bf16(-(1 + 3 * u)) == -(1 + 4 * u)
        assert O.round_bf16(0.0) == 0.0 and O.round_bf16(-40.0) == -40.0
        np.testing.assert_array_equal(O.round_bf16(O.round_bf16(x.astype(np.float64))),
                                      O.round_bf16(x.astype(np.float64)))

    def test_rope_tables_input(self):
        wl = si.small("wan480")
        cos, sin = si.rope_tables(wl)
        assert cos.shape == (wl.N, wl.d // 2) and cos.dtype == np.float32
        np.testing.assert_allclose(cos.astype(np.float64) ** 2 + sin.astype(np.float64) ** 2,
                                   1.0, atol=1e-6)
        np.testing.assert_array_equal(cos[0], 1.0)  # token 0 sits at the origin
        np.testing.assert_array_equal(sin[0], 0.0)


# ------------------------------------------------- spatial repetition ([CAL] 3.2)

class TestSpatialRepetition:
    def brute_similarity(self, q, k, F, ph, pw, frames):
        # explicit loops over row pairs, columns and keys; probabilities from
        # torch's softmax in float64
        P, N = ph * pw, k.shape[0]
        s = torch.from_numpy(q @ k.T / math.sqrt(q.shape[1]))
        p = torch.softmax(s, dim=1).numpy()
        vals = []
        for f in frames:
            pairs = []
            for y in range(ph):
                for y2 in range(y + 1, ph):
                    num = na = nb = 0.0
                    for x in range(pw):
                        a = p[f * P + y * pw + x]
                        b = p[f * P + y2 * pw + x]
                        for j in range(N):
                            num += a[j] * b[j]
                            na += a[j] * a[j]
                            nb += b[j] * b[j]
                    pairs.append(num / math.sqrt(na * nb))
            vals.append(sum(pairs) / len(pairs))
        return sum(vals) / len(vals)

    def test_similarity_brute_force(self):
        F, ph, pw, d = 2, 3, 4, 8
        N = F * ph * pw
        q, k = rand((N, d), 20, 1.5), rand((N, d), 21, 1.5)
        for frames in ([0, 1], [1]):
            want = self.brute_similarity(q, k, F, ph, pw, frames)
            assert O.row_similarity(q, k, F, ph, pw, frames) == pytest.approx(want, rel=1e-12)

    def test_identical_rows_give_one(self):
        # queries that depend on (frame, column) only: every row of a frame
        # has the same pattern
        F, ph, pw, d = 3, 5, 4, 16
        base = rand((F, 1, pw, d), 22)
        q = np.broadcast_to(base, (F, ph, pw, d)).reshape(-1, d)
        k = rand((F * ph * pw, d), 23)
        assert O.row_similarity(q, k, F, ph, pw) == pytest.approx(1.0, abs=1e-12)
        assert O.is_repetitive(O.row_similarity(q, k, F, ph, pw))

    def test_key_order_and_frame_mean(self):
        F, ph, pw, d = 3, 4, 5, 8
        N = F * ph * pw
        q, k = rand((N, d), 24, 2.0), rand((N, d), 25, 2.0)
        perm = np.random.default_rng(26).permutation(N)
        a = O.row_similarity(q, k, F, ph, pw)
        assert O.row_similarity(q, k[perm], F, ph, pw) == pytest.approx(a, rel=1e-12)
        per = [O.row_similarity(q, k, F, ph, pw, [f]) for f in range(F)]
        assert a == pytest.approx(np.mean(per), rel=1e-12)
        assert 0.0 < a < 1.0

    def test_threshold_is_strict(self):
        assert not O.is_repetitive(0.87)
        assert O.is_repetitive(0.87 + 1e-9)
        assert not O.is_repetitive(0.5)

    def test_anchor_rows(self):
        assert O.anchor_rows(30, 5).tolist() == [3, 9, 15, 21, 27]
        assert O.anchor_rows(45, 5).tolist() == [4, 13, 22, 31, 40]
        assert O.anchor_rows(4, 5).tolist() == [0, 1, 2, 3]
        assert O.anchor_rows(6, 5).tolist() == [1, 2, 3, 4, 5]  # bands [0,2) [2] [3] [4] [5]
        assert O.anchor_rows(7, 2).tolist() == [2, 5]           # bands [0,4) [4,7)
        for ph in range(1, 50):
            for k in (1, 2, 5, 7):
                a, src = O.anchor_rows(ph, k), O.row_anchor(ph, k)
                assert len(a) == min(k, ph) and (np.diff(a) > 0).all()
                assert (src[a] == a).all()          # an anchor takes itself
                assert set(src.tolist()) == set(a.tolist())
                assert (np.diff(src) >= 0).all()    # bands are contiguous
                # every row takes the anchor of its own band floor(y k / ph)
                for y in range(ph):
                    if k < ph:
                        assert (src[y] * k) // ph == (y * k) // ph
                    assert abs(y - src[y]) <= (ph + k - 1) // k

    def test_broadcast_rows(self):
        F, ph, pw, d = 2, 7, 3, 2
        o = np.arange(F * ph * pw * d, dtype=np.float64).reshape(-1, d)
        b = O.broadcast_rows(o, F, ph, pw, 3)
        src = O.row_anchor(ph, 3)
        for f in range(F):
            for y in range(ph):
                for x in range(pw):
                    n, m = f * ph * pw + y * pw + x, f * ph * pw + src[y] * pw + x
                    assert (b[n] == o[m]).all()
        np.testing.assert_array_equal(O.broadcast_rows(o, F, ph, pw, ph), o)

    def test_anchor_tile_lists_brute_force(self):
        F, ph, pw, T = 3, 20, 13, 16
        N = F * ph * pw
        ip, ix = O.geometric_block_lists(O.MODE_SPATIAL, F, ph * pw, 1, N, T)
        aip, aix = O.anchor_tile_lists(ip, ix, F, ph, pw, 5, T)
        anchors = set(O.anchor_rows(ph, 5).tolist())
        for i in range(len(ip) - 1):
            has = any(((n % (ph * pw)) // pw) in anchors for n in range(i * T, min(N, i * T + T)))
            got = aix[aip[i]:aip[i + 1]].tolist()
            assert got == (ix[ip[i]:ip[i + 1]].tolist() if has else [])
        assert aip[-1] < ip[-1]  # some tiles hold no anchor row

    def test_repeat_head_is_broadcast_of_full_attention(self):
        F, ph, pw, d, T = 3, 6, 10, 8, 16
        N = F * ph * pw
        q, k, v = rand((N, d), 27), rand((N, d), 28), rand((N, d), 29)
        ip, ix = O.geometric_block_lists(O.MODE_SPATIAL, F, ph * pw, 1, N, T)
        full = O.block_sparse_attention(q, k, v, ip, ix, T)
        got = O.repeat_head_attention(q, k, v, ip, ix, F, ph, pw, 2, T)
        np.testing.assert_allclose(got, O.broadcast_rows(full, F, ph, pw, 2), rtol=1e-13,
                                   atol=1e-14)
        # anchor rows are exactly the full layer's rows
        on = O.anchor_token_mask(F, ph, pw, 2)
        np.testing.assert_allclose(got[on], full[on], rtol=1e-13, atol=1e-14)
