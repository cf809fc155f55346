"""Float64 CPU oracle for sparse spatial/temporal video attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA library (no kernels, headers, tables or helpers); the only
module both sides use is the seeded input generator in ``svg_inputs``.

Every function is the plain definition of one step of the path, written in
float64 with explicit boolean element masks and no blocking, fusion or
reordering beyond what the definition states.  Sources:

* [SVG]  Sparse VideoGen article, m.jxzklqfsx.com/article/815093.html:
  sections "Spatial Head", "Temporal Head", "動態自適應的稀疏策略" (online
  profiling, steps 1-3) and "Layout Transformation + Kernel 加速".
* [CAL]  CalibAtt article, lpnh.cn/news/568491: section 2.2 (128x128 block
  granularity), section 3.1 (energy threshold and cross-prompt aggregation),
  section 3.3 (per-block skip list).
* [SURV] video-diffusion acceleration survey, wmrh.cn/news/48564: section 2.1
  (softmax(QK^T / sqrt(d_k)) V).

Readings of points the pages leave open (each is also listed in the design
notes):
* profiling chooses between the spatial and the temporal mask only; dense is
  the yardstick.  The error is the mean squared difference over the S x d
  sampled outputs; an exact tie goes to SPATIAL;
* masks are token-level for profiling; block lists keep a whole 128x128 tile
  when the token mask touches it, and a kept tile is attended in full;
* a query row whose kept key set is empty gets o = 0;
* block energy E(r, c) is the softmax mass of the rows of query block r that
  falls in key block c, divided by the row count of r (each row of E sums
  to 1); the kept set is the shortest prefix, in descending energy with ties
  to the smaller block index, whose sum reaches eps; a block survives the
  cross-input vote when its keep frequency is >= rho; an empty voted row keeps
  the block of largest summed energy;
* QK-Norm is an RMS normalisation over the head dimension with a per-channel
  weight and an epsilon inside the square root; RoPE rotates interleaved
  channel pairs (2i, 2i+1) by caller-supplied per-token angles (cos / sin
  tables); QK-Norm runs first;
* spatial repetition ([CAL] 3.2): a row's attention pattern is the block of
  dense probabilities of its pw query tokens over all keys; the head score
  is the mean pairwise cosine over the rows of each evaluated frame; anchors
  are the middle rows of k equal bands and each row copies the anchor of its
  band; anchor rows attend exactly as in the full layer (query tiles with no
  anchor row are skipped);
* the energy threshold decays exponentially in the denoising-step index from
  0.99 (first step) to 0.84 (last step); the skip list holds each row's
  maximal runs of consecutive kept blocks; the bitmap holds one bit per
  (query block, key block) in 32-bit words.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(library cross-checks, closed forms, invariants, brute force, and worked
examples under ``tests/golden/``).
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

MODE_SPATIAL = 0
MODE_TEMPORAL = 1
MODE_DENSE = 2


# ---------------------------------------------------------------------------
# O1 / O2: dense and masked attention   ([SURV] 2.1)
# ---------------------------------------------------------------------------

def softmax_scale(d: int) -> float:
    """tau = 1 / sqrt(d_k)  ([SURV] 2.1)."""
    return 1.0 / math.sqrt(d)


def attention_probs(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """p[i, j] = exp(tau q_i.k_j - m_i) / sum_j' exp(tau q_i.k_j' - m_i),
    m_i = max_j tau q_i.k_j.  q [n, d], k [N, d] -> p [n, N]."""
    s = (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T) * scale
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=1, keepdims=True)


def dense_attention(q, k, v, scale=None) -> np.ndarray:
    """o = softmax(tau Q K^T) V over all keys  ([SURV] 2.1)."""
    q = np.asarray(q, np.float64)
    scale = softmax_scale(q.shape[-1]) if scale is None else scale
    return attention_probs(q, k, scale) @ np.asarray(v, np.float64)


def masked_attention(q, k, v, mask, scale=None) -> np.ndarray:
    """Softmax restricted to {j : mask[i, j]}; a row with no kept key gives
    o_i = 0.  q [n, d], k/v [N, d], mask bool [n, N]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    mask = np.asarray(mask, bool)
    scale = softmax_scale(q.shape[-1]) if scale is None else scale
    s = (q @ k.T) * scale
    s = np.where(mask, s, -np.inf)
    has = mask.any(axis=1)
    m = np.where(has, s.max(axis=1, initial=-np.inf), 0.0)[:, None]
    e = np.where(mask, np.exp(s - m), 0.0)
    den = e.sum(axis=1, keepdims=True)
    den = np.where(den > 0, den, 1.0)
    return (e / den) @ v


# ---------------------------------------------------------------------------
# O3: token masks   ([SVG] "Spatial Head", "Temporal Head")
# ---------------------------------------------------------------------------

def spatial_mask(rows, cols, P: int, width: int) -> np.ndarray:
    """Spatial head, frame-major tokens n = f P + s: query row i sees key j iff
    their frames differ by at most ``width`` (same and adjacent frames)."""
    fr = np.asarray(rows) // P
    fc = np.asarray(cols) // P
    return np.abs(fr[:, None] - fc[None, :]) <= width


def temporal_mask_frame_major(rows, cols, P: int) -> np.ndarray:
    """Temporal head, frame-major tokens: i sees j iff they are the same
    spatial position s = n mod P (in any frame)."""
    return (np.asarray(rows)[:, None] % P) == (np.asarray(cols)[None, :] % P)


def temporal_mask_token_major(rows, cols, F: int) -> np.ndarray:
    """The temporal mask in token-major indices m = s F + f: same s = m div F."""
    return (np.asarray(rows)[:, None] // F) == (np.asarray(cols)[None, :] // F)


# ---------------------------------------------------------------------------
# O4: online head profiling   ([SVG] "動態自適應的稀疏策略", steps 1-3)
# ---------------------------------------------------------------------------

def profile_head(q, k, v, idx, F: int, P: int, width: int, scale=None):
    """For the sampled rows ``idx`` (frame-major), compute the dense output and
    the outputs under the spatial and temporal masks over all N keys; the
    error of a mask is mean((o_mask - o_dense)^2) over the S x d outputs; the
    head takes the mask of smaller error (an exact tie goes to SPATIAL).

    Returns (mse_spatial, mse_temporal, mode)."""
    q = np.asarray(q, np.float64)
    N = k.shape[0]
    idx = np.asarray(idx)
    cols = np.arange(N)
    qs = q[idx]
    o_d = dense_attention(qs, k, v, scale)
    o_s = masked_attention(qs, k, v, spatial_mask(idx, cols, P, width), scale)
    o_t = masked_attention(qs, k, v, temporal_mask_frame_major(idx, cols, P), scale)
    n = o_d.size
    mse_s = float(((o_s - o_d) ** 2).sum() / n)
    mse_t = float(((o_t - o_d) ** 2).sum() / n)
    mode = MODE_TEMPORAL if mse_t < mse_s else MODE_SPATIAL
    return mse_s, mse_t, mode


def profile_heads(q, k, v, idx, F: int, P: int, width: int):
    """profile_head over every (b, h) of [B, H, N, d] inputs.
    Returns mse [B*H, 2] (spatial, temporal) and mode [B*H]."""
    B, H = q.shape[:2]
    mse = np.zeros((B * H, 2))
    mode = np.zeros(B * H, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            ms, mt, md = profile_head(q[b, h], k[b, h], v[b, h], idx, F, P, width)
            mse[b * H + h] = (ms, mt)
            mode[b * H + h] = md
    return mse, mode


# ---------------------------------------------------------------------------
# O5: frame-major <-> token-major permutation
#     ([SVG] "Layout Transformation + Kernel 加速")
# ---------------------------------------------------------------------------

def token_major_source(F: int, P: int) -> np.ndarray:
    """src[m] = frame-major index of token-major position m, from
    y[s F + f] = x[f P + s]."""
    src = np.empty(F * P, dtype=np.int64)
    for f in range(F):
        for s in range(P):
            src[s * F + f] = f * P + s
    return src


def permute_token_major(x: np.ndarray, F: int, P: int) -> np.ndarray:
    """y[..., s F + f, :] = x[..., f P + s, :] along the token axis (-2)."""
    y = np.empty_like(x)
    for f in range(F):
        for s in range(P):
            y[..., s * F + f, :] = x[..., f * P + s, :]
    return y


def permute_frame_major(y: np.ndarray, F: int, P: int) -> np.ndarray:
    """The inverse map: x[..., f P + s, :] = y[..., s F + f, :]."""
    x = np.empty_like(y)
    for f in range(F):
        for s in range(P):
            x[..., f * P + s, :] = y[..., s * F + f, :]
    return x


# ---------------------------------------------------------------------------
# O6 / O7: 128-row tiles and geometric key-block lists   ([CAL] 2.2)
# ---------------------------------------------------------------------------

def tile_rows(i: int, N: int, T: int = 128) -> np.ndarray:
    """Tile i holds rows [i T, min(N, (i + 1) T))."""
    return np.arange(i * T, min(N, (i + 1) * T))


def n_tiles(N: int, T: int = 128) -> int:
    return (N + T - 1) // T


def _row_mask(kind: int, r: int, N: int, F: int, P: int, width: int) -> np.ndarray:
    cols = np.arange(N)
    rr = np.array([r])
    if kind == MODE_SPATIAL:
        return spatial_mask(rr, cols, P, width)[0]
    if kind == MODE_TEMPORAL:
        return temporal_mask_token_major(rr, cols, F)[0]
    return np.ones(N, dtype=bool)


def geometric_block_lists(kind: int, F: int, P: int, width: int, N: int,
                          T: int = 128) -> Tuple[np.ndarray, np.ndarray]:
    """Keep tile pair (i, j) iff some query row of tile i and key column of
    tile j satisfy the token mask: the spatial mask in frame-major indices,
    the temporal mask in token-major indices (the layout temporal heads run
    in), all pairs for dense.  Brute force over the element masks; rows with
    the same frame (spatial) or the same position (temporal) have the same mask
    row, so each distinct row is evaluated once.  Returns CSR (indptr
    [nB + 1], indices ascending)."""
    nb = n_tiles(N, T)
    indptr = [0]
    indices: List[int] = []
    for i in range(nb):
        rows = tile_rows(i, N, T)
        if kind == MODE_SPATIAL:
            cls = rows // P
        elif kind == MODE_TEMPORAL:
            cls = rows // F
        else:
            cls = np.zeros_like(rows)
        seen = {}
        for r, c in zip(rows, cls):
            if c not in seen:
                seen[c] = r
        keymask = np.zeros(N, dtype=bool)
        for r in seen.values():
            keymask |= _row_mask(kind, int(r), N, F, P, width)
        for j in range(nb):
            if keymask[j * T: min(N, (j + 1) * T)].any():
                indices.append(j)
        indptr.append(len(indices))
    return np.asarray(indptr, np.int32), np.asarray(indices, np.int32)


def block_mask_from_lists(indptr, indices, N: int, T: int = 128) -> np.ndarray:
    """Element mask M_B [N, N]: M_B[r, c] = (tile(c) is in the list of tile(r))."""
    M = np.zeros((N, N), dtype=bool)
    for i in range(len(indptr) - 1):
        rows = tile_rows(i, N, T)
        for j in indices[indptr[i]:indptr[i + 1]]:
            M[rows[0]:rows[-1] + 1, j * T: min(N, (j + 1) * T)] = True
    return M


# ---------------------------------------------------------------------------
# O8: block-sparse attention   ([CAL] 2.2, 3.3; [SURV] 2.1)
# ---------------------------------------------------------------------------

def block_sparse_rows(q, k, v, rows, indptr, indices, T: int = 128, scale=None):
    """o for the given query rows: softmax over the key columns of the kept
    tiles of the row's query tile (the whole tile, clipped at N)."""
    N = k.shape[0]
    rows = np.asarray(rows)
    mask = np.zeros((len(rows), N), dtype=bool)
    for a, r in enumerate(rows):
        i = int(r) // T
        for j in indices[indptr[i]:indptr[i + 1]]:
            mask[a, j * T: min(N, (j + 1) * T)] = True
    return masked_attention(np.asarray(q, np.float64)[rows], k, v, mask, scale)


def block_sparse_attention(q, k, v, indptr, indices, T: int = 128, scale=None):
    """O8 for every query row of one head: [N, d] -> [N, d]."""
    N = q.shape[0]
    out = np.zeros((N, q.shape[1]))
    for i in range(n_tiles(N, T)):
        rows = tile_rows(i, N, T)
        out[rows] = block_sparse_rows(q, k, v, rows, indptr, indices, T, scale)
    return out


# ---------------------------------------------------------------------------
# O9: energy-threshold calibration with cross-input vote   ([CAL] 3.1)
# ---------------------------------------------------------------------------

def block_energy(q, k, T: int = 128, scale=None, row_blocks=None) -> np.ndarray:
    """E[r, c] = sum_{i in block r, j in block c} p_ij / |block r|, p the dense
    softmax of one head.  q, k [N, d] -> E [nB, nB].  row_blocks (a sequence
    of query-block indices) computes only those rows of E, in that order
    (each row depends on its own query block alone)."""
    q = np.asarray(q, np.float64)
    N = q.shape[0]
    scale = softmax_scale(q.shape[1]) if scale is None else scale
    nb = n_tiles(N, T)
    row_blocks = range(nb) if row_blocks is None else row_blocks
    E = np.zeros((len(row_blocks), nb))
    for out_r, r in enumerate(row_blocks):
        rows = tile_rows(r, N, T)
        p = attention_probs(q[rows], k, scale)
        for c in range(nb):
            E[out_r, c] = p[:, c * T: min(N, (c + 1) * T)].sum() / len(rows)
    return E


def energy_order(e_row: Sequence[float]) -> List[int]:
    """Key blocks by descending energy; equal energies by ascending index."""
    return sorted(range(len(e_row)), key=lambda c: (-float(e_row[c]), c))


def minimal_energy_set(e_row: Sequence[float], eps: float) -> List[int]:
    """S(r): the shortest prefix of the descending-energy order whose running
    sum (float64, in that order) reaches eps.  If no prefix reaches eps, all
    blocks are kept."""
    order = energy_order(e_row)
    acc = 0.0
    kept = []
    for c in order:
        kept.append(c)
        acc += float(e_row[c])
        if acc >= eps:
            break
    return sorted(kept)


def calibrate_lists(E_list: Sequence[np.ndarray], eps: float, rho: float):
    """Cross-input vote: E_list holds R energy maps [nQB, nKB] of one head.
    freq(r, c) = #{s : c in S_s(r)} / R; keep (r, c) iff freq >= rho; an
    empty row keeps argmax_c sum_s E_s(r, c) (smallest index on ties).
    Returns CSR (indptr, indices ascending)."""
    R = len(E_list)
    nq, nk = E_list[0].shape
    indptr = [0]
    indices: List[int] = []
    for r in range(nq):
        count = np.zeros(nk, dtype=np.int64)
        for E in E_list:
            for c in minimal_energy_set(E[r], eps):
                count[c] += 1
        kept = [c for c in range(nk) if count[c] / R >= rho]
        if not kept:
            tot = np.zeros(nk)
            for E in E_list:
                tot = tot + np.asarray(E[r], np.float64)
            kept = [int(np.argmax(tot))]
        indices.extend(kept)
        indptr.append(len(indices))
    return np.asarray(indptr, np.int32), np.asarray(indices, np.int32)


# ---------------------------------------------------------------------------
# O10: timestep schedule of the energy threshold and mask encodings
#      ([CAL] 3.1: eps(t) decays exponentially, about 0.99 early and 0.84
#      late; 3.3: the mask as a skip list of contiguous block intervals and
#      as a bitmap, 32x smaller)
# ---------------------------------------------------------------------------

def epsilon_schedule(n_steps: int, eps_first: float = 0.99, eps_last: float = 0.84) -> np.ndarray:
    """eps at denoising steps 0 .. n_steps-1, decaying exponentially in the
    step index from eps_first to eps_last: eps_i = eps_first *
    (eps_last / eps_first) ** (i / (n_steps - 1)); a single step uses
    eps_first.  (The pages give the two end values and the decay shape, not
    the formula; this is the plainest exponential between them.)"""
    if n_steps <= 0:
        return np.zeros(0)
    if n_steps == 1:
        return np.array([float(eps_first)])
    i = np.arange(n_steps, dtype=np.float64)
    return float(eps_first) * (float(eps_last) / float(eps_first)) ** (i / (n_steps - 1))


def lists_to_intervals(indptr, indices):
    """Skip list: each row's set of kept key blocks as maximal runs of
    consecutive blocks [start, end), ascending.  Returns (iptr [rows + 1],
    starts, ends)."""
    iptr = [0]
    starts: List[int] = []
    ends: List[int] = []
    for r in range(len(indptr) - 1):
        kept = sorted(set(int(c) for c in indices[indptr[r]:indptr[r + 1]]))
        run_start = None
        prev = None
        for c in kept:
            if run_start is None:
                run_start = c
            elif c != prev + 1:
                starts.append(run_start)
                ends.append(prev + 1)
                run_start = c
            prev = c
        if run_start is not None:
            starts.append(run_start)
            ends.append(prev + 1)
        iptr.append(len(starts))
    return (np.asarray(iptr, np.int32), np.asarray(starts, np.int32), np.asarray(ends, np.int32))


def intervals_to_lists(iptr, starts, ends):
    """Inverse of lists_to_intervals: CSR with ascending indices."""
    indptr = [0]
    indices: List[int] = []
    for r in range(len(iptr) - 1):
        for t in range(iptr[r], iptr[r + 1]):
            indices.extend(range(int(starts[t]), int(ends[t])))
        indptr.append(len(indices))
    return np.asarray(indptr, np.int32), np.asarray(indices, np.int32)


def lists_to_bitmap(indptr, indices, n_cols: int) -> np.ndarray:
    """Bitmap of the kept blocks: uint32 words [rows][ceil(n_cols / 32)],
    block c of row r is bit (c mod 32) of word (c div 32)."""
    rows = len(indptr) - 1
    words = (n_cols + 31) // 32
    bm = np.zeros((rows, words), dtype=np.uint32)
    for r in range(rows):
        for c in indices[indptr[r]:indptr[r + 1]]:
            c = int(c)
            bm[r, c // 32] |= np.uint32(1) << np.uint32(c % 32)
    return bm


def bitmap_to_lists(bm: np.ndarray, n_cols: int):
    """Inverse of lists_to_bitmap: CSR with ascending indices."""
    indptr = [0]
    indices: List[int] = []
    for r in range(bm.shape[0]):
        for c in range(n_cols):
            if (int(bm[r, c // 32]) >> (c % 32)) & 1:
                indices.append(c)
        indptr.append(len(indices))
    return np.asarray(indptr, np.int32), np.asarray(indices, np.int32)


# ---------------------------------------------------------------------------
# QK-Norm and rotary position embedding before attention
#   ([SVG] "Layout Transformation + Kernel 加速": the method ships its own
#   QK-Norm and RoPE kernels next to the attention kernels)
# ---------------------------------------------------------------------------

def qk_rms_norm(x, gamma=None, eps: float = 1e-6) -> np.ndarray:
    """RMS normalisation of every row over the head dimension:
    x_hat = x / sqrt(mean_c x_c^2 + eps) * gamma (gamma = 1 when None)."""
    x = np.asarray(x, np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, np.float64)
    return y


def rope_rotate(x, cos, sin) -> np.ndarray:
    """Rotary embedding on interleaved channel pairs: pair i of row n,
    (a, b) = (x[n, 2i], x[n, 2i+1]), becomes (a cos - b sin, a sin + b cos)
    with cos = cos[n, i], sin = sin[n, i].  x [..., N, d], tables [N, d/2]."""
    x = np.asarray(x, np.float64)
    c = np.asarray(cos, np.float64)
    s = np.asarray(sin, np.float64)
    a = x[..., 0::2]
    b = x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = a * c - b * s
    y[..., 1::2] = a * s + b * c
    return y


def round_bf16(x) -> np.ndarray:
    """x rounded to the nearest bf16 value (8 significant bits, ties to
    even), kept in float64: with x = m 2^e, 0.5 <= |m| < 1, the result is
    round_half_even(m 2^8) 2^(e-8).  Models a bf16 tensor holding a
    result; no overflow or subnormal handling (not reached here)."""
    m, e = np.frexp(np.asarray(x, np.float64))
    return np.ldexp(np.round(m * 256.0), e - 8)


def qk_norm_rope(x, gamma=None, eps: float = 1e-6, cos=None, sin=None,
                 norm: bool = True, rope: bool = True) -> np.ndarray:
    """The pre-attention transform of q or k: QK-Norm first, then RoPE
    (either may be switched off)."""
    y = np.asarray(x, np.float64)
    if norm:
        y = qk_rms_norm(y, gamma, eps)
    if rope:
        y = rope_rotate(y, cos, sin)
    return y


# ---------------------------------------------------------------------------
# Spatial-repetition heads   ([CAL] 3.2)
#   Some heads attend almost identically from every image row of a frame:
#   they are found by the mean cosine similarity of the rows' attention
#   patterns (> gamma = 0.87), and for them only k = 5 equally spaced anchor
#   rows per frame are computed; every other row takes its anchor's output.
# ---------------------------------------------------------------------------

def row_similarity(q, k, F: int, ph: int, pw: int, frames=None, scale=None) -> float:
    """Mean cosine similarity between the attention patterns of the image
    rows of a frame.  The pattern of row y of frame f is the pw x N block of
    dense attention probabilities of its query tokens n = f P + y pw + x
    (x < pw) over all N keys; the cosine of rows y, y' is the Frobenius inner
    product of their blocks over the product of their Frobenius norms.  The
    mean runs over all pairs y < y' of a frame, then over the evaluated
    frames (all when None).  Needs ph >= 2."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    P = ph * pw
    N = k.shape[0]
    scale = softmax_scale(q.shape[-1]) if scale is None else scale
    frames = range(F) if frames is None else frames
    iu = np.triu_indices(ph, 1)
    per_frame = []
    for f in frames:
        p = attention_probs(q[f * P:(f + 1) * P], k, scale)   # rows in order y pw + x
        A = p.reshape(ph, pw * N)                             # row y -> its flattened block
        G = A @ A.T
        nrm = np.sqrt(np.diag(G))
        per_frame.append(np.mean((G / np.outer(nrm, nrm))[iu]))
    return float(np.mean(per_frame))


def is_repetitive(similarity, gamma: float = 0.87):
    """A head repeats spatially when its mean row similarity exceeds gamma."""
    return np.asarray(similarity) > gamma


def anchor_rows(ph: int, k: int = 5) -> np.ndarray:
    """k equally spaced anchor rows: the ph rows fall into k equal bands
    (band j = the rows y with floor(y k / ph) = j, i.e. y in
    [ceil(j ph / k), ceil((j+1) ph / k))) and each band's anchor is its
    middle row (the upper one of two); every row when k >= ph."""
    if k >= ph:
        return np.arange(ph)
    out = []
    for j in range(k):
        lo = -(-j * ph // k)
        hi = -(-(j + 1) * ph // k)
        out.append(lo + (hi - lo) // 2)
    return np.array(out)


def row_anchor(ph: int, k: int = 5) -> np.ndarray:
    """The anchor row each row y takes its output from: the anchor of band
    floor(y k / ph)."""
    if k >= ph:
        return np.arange(ph)
    a = anchor_rows(ph, k)
    return np.array([a[(y * k) // ph] for y in range(ph)])


def anchor_token_mask(F: int, ph: int, pw: int, k: int = 5) -> np.ndarray:
    """Boolean [N]: frame-major tokens that lie on an anchor row."""
    rows = np.zeros(ph, dtype=bool)
    rows[anchor_rows(ph, k)] = True
    return np.tile(np.repeat(rows, pw), F)


def anchor_tile_lists(indptr, indices, F: int, ph: int, pw: int, k: int = 5, T: int = 128):
    """The lists of the query tiles that hold an anchor-row token; the other
    tiles get empty lists (their rows are all filled by the broadcast)."""
    N = F * ph * pw
    on = anchor_token_mask(F, ph, pw, k)
    keep = [bool(on[tile_rows(i, N, T)].any()) for i in range(len(indptr) - 1)]
    ip, ix = [0], []
    for i, kp in enumerate(keep):
        if kp:
            ix.extend(indices[indptr[i]:indptr[i + 1]])
        ip.append(len(ix))
    return np.array(ip, dtype=np.int64), np.array(ix, dtype=np.int64)


def broadcast_rows(o, F: int, ph: int, pw: int, k: int = 5) -> np.ndarray:
    """o'[f, y, x] = o[f, anchor(y), x] for [N, d] frame-major rows."""
    o = np.asarray(o)
    src = row_anchor(ph, k)
    y = o.reshape(F, ph, pw, -1)[:, src]
    return y.reshape(o.shape).copy()


def repeat_head_attention(q, k, v, indptr, indices, F: int, ph: int, pw: int, kk: int = 5,
                          T: int = 128, scale=None) -> np.ndarray:
    """Attention of a spatially repeating head: block-sparse attention over
    the anchor-tile lists, then every row takes its anchor's output."""
    ip, ix = anchor_tile_lists(indptr, indices, F, ph, pw, kk, T)
    o = block_sparse_attention(q, k, v, ip, ix, T, scale)
    return broadcast_rows(o, F, ph, pw, kk)


# ---------------------------------------------------------------------------
# The whole layer: profile -> permute temporal heads -> block-sparse -> back
# ---------------------------------------------------------------------------

def svg_layer(q, k, v, idx, F: int, P: int, width: int, T: int = 128, qk=None,
              qk_bf16: bool = False):
    """One attention layer of the method for [B, H, N, d] inputs: profile each
    head, run spatial heads on their frame-major lists, temporal heads in
    token-major order on their lists, and map temporal outputs back.
    qk = (gamma_q, gamma_k, eps, cos, sin) first applies QK-Norm + RoPE to q
    and k; qk_bf16 stores that result as bf16 (the tensor type of a bf16
    layer) before attention reads it.
    Returns (o [B, H, N, d], mode [B*H], mse [B*H, 2])."""
    B, H, N, d = q.shape
    if qk is not None:
        gq, gk, eps, cos, sin = qk
        q = qk_norm_rope(q, gq, eps, cos, sin)
        k = qk_norm_rope(k, gk, eps, cos, sin)
        if qk_bf16:
            q, k = round_bf16(q), round_bf16(k)
    mse, mode = profile_heads(q, k, v, idx, F, P, width)
    lists = {MODE_SPATIAL: geometric_block_lists(MODE_SPATIAL, F, P, width, N, T),
             MODE_TEMPORAL: geometric_block_lists(MODE_TEMPORAL, F, P, width, N, T)}
    o = np.zeros((B, H, N, d))
    for b in range(B):
        for h in range(H):
            md = int(mode[b * H + h])
            ip, ix = lists[md]
            if md == MODE_TEMPORAL:
                qt, kt, vt = (permute_token_major(np.asarray(t[b, h], np.float64), F, P)
                              for t in (q, k, v))
                o[b, h] = permute_frame_major(block_sparse_attention(qt, kt, vt, ip, ix, T), F, P)
            else:
                o[b, h] = block_sparse_attention(q[b, h], k[b, h], v[b, h], ip, ix, T)
    return o, mode, mse
