"""Plain, slow, fp64 CPU oracle for block-sparse and piecewise (PISA) attention.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module. The product path (the CUDA
library and its Python binding) never calls it, and this module shares no code with
the CUDA path.

Every function works on ONE (batch, head) slice: q, k, v are [L, d] arrays. Inputs
are the bf16-rounded values the GPU sees, upcast to float64; everything below is
float64. Notation follows the pages: block size B, M = L/B blocks, scale s, query
block i, selected KV blocks S_i, unselected blocks U_i.

Sources (page title, section):
  [BSA]  "多模态 DiT 上的块稀疏 Attention" (block-sparse attention on multimodal DiT,
         dpshk.com engineering blog): §3.3 keep-or-drop formula, §4.1 block layout,
         §4.2 build_sparse_mask, §4.3 block_sparse_attention, §5.4 index lists.
  [PISA] "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
         Transformers" (gist.science summary of arXiv 2602.01077), technical summary
         §2: core algorithm (N_t, D_t, alpha), global first-order correction with
         H-bar, covariance-aware routing with M_j = ||H_j - H-bar||.

Readings taken where the pages are silent:
  * scores carry the 1/sqrt(d) scale s; the first-order term is s * (q_t H-bar) *
    sum alpha (Taylor expansion of exp(s q k) about the centroid);
  * every exponent is shifted by m_t = max over the exact scores and the U_i
    centroid scores (cancels in N_t / D_t);
  * D_t = exact sum + B * alpha_{t,j} per unselected block (the first-order term
    adds sum_n (k_n - kbar) = 0 to the denominator);
  * H_j[a, c] = sum_n (k_{j,n} - kbar_j)[a] * v_{j,n}[c]  (d_k x d_v);
    H-bar = mean over all M blocks of the head; ||.|| is the Frobenius norm;
  * routing score_ij = softmax_j(s qbar_i . kbar_j) + lambda * M_j / sum_j' M_j',
    qbar_i = mean of the block's queries; top-k by descending score, ties to the
    smaller j; lists emitted in ascending j;
  * a keep-or-drop row with an empty list outputs zeros (lse = -inf);
  * token-level padding ([BSA] §4.1 pads the text segment to a multiple of the block
    size; §7.3 gives a timestep token its own block): ``key_valid[j]`` is the number of
    leading real tokens of block j (the rest are padding). Padded keys get no weight;
    centroids, value sums, H_j and pooled queries are taken over the real tokens; an
    unselected block's Taylor-tail weight is its number of real tokens; a padded block
    is always in S_i (routing places it there first), since a partial block's centroid
    is a poor expansion point and the pages keep such blocks fully connected anyway.
    Padded query rows are computed like any other row.

Parity pins live in tests/test_oracle.py. The overall approximation error of PISA
against dense attention is parity unpinned by the pages (they print no error
values): it is reported, never asserted.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------------
# a1. Multimodal fixed mask  ([BSA] §4.2 build_sparse_mask, generalised to a 2-D grid)
# ----------------------------------------------------------------------------------
def mask_dense(n_text_blocks: int, grid_h: int, grid_w: int, radius: int,
               global_stride: int, global_rows_full: int = 0) -> np.ndarray:
    """Dense [M, M] keep mask of the multimodal pattern.

    Text blocks (the first n_text_blocks) attend to, and are attended by, every block.
    Image block a (image-local index, row-major on the grid_h x grid_w block grid)
    keeps image block b when their Chebyshev distance on the grid is <= radius, or
    when b is a global block (b % global_stride == 0). With global_rows_full, a global
    image block's row is also full.
    """
    nt = n_text_blocks
    ni = grid_h * grid_w
    m = nt + ni
    keep = np.zeros((m, m), dtype=bool)
    for i in range(m):
        for j in range(m):
            if i < nt or j < nt:
                keep[i, j] = True
                continue
            a, b = i - nt, j - nt
            dist = max(abs(a // grid_w - b // grid_w), abs(a % grid_w - b % grid_w))
            if dist <= radius:
                keep[i, j] = True
            elif global_stride > 0 and b % global_stride == 0:
                keep[i, j] = True
            elif global_rows_full and global_stride > 0 and a % global_stride == 0:
                keep[i, j] = True
    return keep


def dense_to_csr(keep: np.ndarray) -> tuple:
    """Per-row index lists of kept key blocks ([BSA] §5.4), ascending, as CSR."""
    row_ptr = [0]
    cols = []
    for i in range(keep.shape[0]):
        js = [j for j in range(keep.shape[1]) if keep[i, j]]
        cols.extend(js)
        row_ptr.append(len(cols))
    return np.asarray(row_ptr, dtype=np.int32), np.asarray(cols, dtype=np.int32)


def _row(row_ptr, col_idx, i):
    return [int(c) for c in col_idx[row_ptr[i]:row_ptr[i + 1]]]


def _valid(key_valid, M, block):
    """Real tokens per block (all of them when there is no padding)."""
    return [block] * M if key_valid is None else [int(x) for x in key_valid]


def _keys(blocks, block, valid):
    """Token positions of the real keys of the given blocks, in order."""
    if not blocks:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(j * block, j * block + valid[j]) for j in blocks])


# ----------------------------------------------------------------------------------
# Dense softmax attention (reference for the approximation error)
# ----------------------------------------------------------------------------------
def dense_head(q, k, v, scale):
    """o_t = softmax(s q_t K^T) V over all L keys ([BSA] §3.3, full attention)."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    a = scale * (q @ k.T)
    m = a.max(axis=1, keepdims=True)
    p = np.exp(a - m)
    return (p @ v) / p.sum(axis=1, keepdims=True)


# ----------------------------------------------------------------------------------
# Keep-or-drop block-sparse attention  ([BSA] §3.3, §4.3)
# ----------------------------------------------------------------------------------
def keep_or_drop_head(q, k, v, row_ptr, col_idx, block, scale, qblocks=None, key_valid=None):
    """O_i = softmax(s Q_i K_{S_i}^T) V_{S_i}, the softmax taken over S_i only (over the
    real keys of S_i when ``key_valid`` marks padding).

    Returns (out [n, d], lse [n]) for the rows of the requested query blocks (all by
    default), in block order.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    L, d = q.shape
    M = L // block
    valid = _valid(key_valid, M, block)
    blocks = range(M) if qblocks is None else qblocks
    outs, lses = [], []
    for i in blocks:
        qi = q[i * block:(i + 1) * block]
        sel = _row(row_ptr, col_idx, i)
        if not sel:
            outs.append(np.zeros((block, v.shape[1])))
            lses.append(np.full(block, -np.inf))
            continue
        idx = _keys(sel, block, valid)
        a = scale * (qi @ k[idx].T)                       # [B, real keys of S_i]
        m = a.max(axis=1, keepdims=True)
        p = np.exp(a - m)
        den = p.sum(axis=1)
        outs.append((p @ v[idx]) / den[:, None])
        lses.append(m[:, 0] + np.log(den))
    return np.concatenate(outs), np.concatenate(lses)


# ----------------------------------------------------------------------------------
# a2. Per-block statistics  ([PISA] §2: centroids, value sums, H_j, H-bar, M_j)
# ----------------------------------------------------------------------------------
def precompute_head(k, v, block, key_valid=None):
    """Return kbar [M,d], vsum [M,d], H [M,d,d], Hbar [d,d], Mnorm [M].

    kbar_j = (1/B_j) sum_n k_{j,n};  vsum_j = sum_n v_{j,n};
    H_j = sum_n (k_{j,n} - kbar_j)^T v_{j,n}  (centred form, d_k rows x d_v cols);
    Hbar = (1/M) sum_j H_j;  Mnorm_j = ||H_j - Hbar||_F.
    The sums run over the B_j real tokens of block j (B_j = B without padding).
    """
    k, v = (np.asarray(x, dtype=np.float64) for x in (k, v))
    L, d = k.shape
    M = L // block
    valid = _valid(key_valid, M, block)
    kb = k.reshape(M, block, d)
    vb = v.reshape(M, block, v.shape[1])
    kbar = np.stack([kb[j, :valid[j]].mean(axis=0) for j in range(M)])
    vsum = np.stack([vb[j, :valid[j]].sum(axis=0) for j in range(M)])
    H = np.empty((M, d, v.shape[1]))
    for j in range(M):
        centred = kb[j, :valid[j]] - kbar[j]
        H[j] = centred.T @ vb[j, :valid[j]]
    Hbar = H.mean(axis=0)
    Mnorm = np.sqrt(((H - Hbar) ** 2).sum(axis=(1, 2)))
    return kbar, vsum, H, Hbar, Mnorm


# ----------------------------------------------------------------------------------
# a3. Covariance-aware top-k routing  ([PISA] §2 covariance-aware routing)
# ----------------------------------------------------------------------------------
def route_head(q, kbar, Mnorm, block, k_top, lam, scale, key_valid=None):
    """Top-k KV blocks per query block; returns (row_ptr, col_idx, scores [M, M]).

    qbar_i = mean of the real queries of block i; p_ij = softmax_j(s qbar_i . kbar_j);
    score_ij = p_ij + lam * Mnorm_j / sum_j' Mnorm_j' (second term 0 if the sum is 0).
    S_i = the padded blocks (every row), then the largest scores up to k_top, ties
    broken towards the smaller j; the list is emitted in ascending j.
    """
    q = np.asarray(q, dtype=np.float64)
    kbar = np.asarray(kbar, dtype=np.float64)
    Mnorm = np.asarray(Mnorm, dtype=np.float64)
    L, d = q.shape
    M = L // block
    valid = _valid(key_valid, M, block)
    forced = [j for j in range(M) if valid[j] < block]
    if len(forced) > k_top:
        raise ValueError("k_top is smaller than the number of padded blocks")
    qb = q.reshape(M, block, d)
    qbar = np.stack([qb[i, :valid[i]].mean(axis=0) for i in range(M)])
    a = scale * (qbar @ kbar.T)                           # [M, M]
    p = np.exp(a - a.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    tot = Mnorm.sum()
    cov = Mnorm / tot if tot > 0 else np.zeros_like(Mnorm)
    scores = p + lam * cov[None, :]
    row_ptr = np.arange(M + 1, dtype=np.int32) * k_top
    col_idx = np.empty(M * k_top, dtype=np.int32)
    for i in range(M):
        order = sorted((j for j in range(M) if j not in forced), key=lambda j: (-scores[i, j], j))
        col_idx[i * k_top:(i + 1) * k_top] = sorted(forced + order[:k_top - len(forced)])
    return row_ptr, col_idx, scores


# ----------------------------------------------------------------------------------
# a4-a6. Piecewise sparse attention  ([PISA] §2: o_t = N_t / D_t)
# ----------------------------------------------------------------------------------
def pisa_head(q, k, v, row_ptr, col_idx, block, scale, kbar, vsum, Hbar,
              qblocks=None, Hblocks=None, key_valid=None):
    """Exact terms over S_i, zeroth-order centroid terms and the first-order
    correction over U_i, inside one normalisation.

    N_t = sum_{j in S_i} sum_n e^{s q_t.k_{j,n} - m_t} v_{j,n}
          + sum_{j in U_i} alpha_tj vsum_j
          + s (q_t Hbar) sum_{j in U_i} alpha_tj
    D_t = sum_{j in S_i} sum_n e^{s q_t.k_{j,n} - m_t} + sum_{j in U_i} B_j alpha_tj
    alpha_tj = e^{s q_t.kbar_j - m_t};  o_t = N_t / D_t.
    B_j is the block's number of real tokens (B without padding); the exact sums run
    over real keys only.

    With ``Hblocks`` ([M, d, d]) the first-order term uses each block's own H_j,
    s alpha_tj (q_t H_j), instead of the shared Hbar: the per-block variant that the
    PISA summary names as the bandwidth-bound alternative to Hbar.
    Returns (out [n, d], lse [n]) with lse = m_t + log D_t.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    kbar, vsum, Hbar = (np.asarray(x, dtype=np.float64) for x in (kbar, vsum, Hbar))
    L, d = q.shape
    M = L // block
    valid = _valid(key_valid, M, block)
    blocks = range(M) if qblocks is None else qblocks
    outs, lses = [], []
    for i in blocks:
        qi = q[i * block:(i + 1) * block]
        sel = _row(row_ptr, col_idx, i)
        uns = [j for j in range(M) if j not in set(sel)]
        if sel:
            idx = _keys(sel, block, valid)
            a_ex = scale * (qi @ k[idx].T)                # exact scores [B, real keys]
        else:
            idx = np.zeros(0, dtype=np.int64)
            a_ex = np.zeros((block, 0))
        a_un = scale * (qi @ kbar[uns].T)                 # centroid scores [B, |U_i|]
        m = np.full(block, -np.inf)
        if a_ex.shape[1]:
            m = np.maximum(m, a_ex.max(axis=1))
        if a_un.shape[1]:
            m = np.maximum(m, a_un.max(axis=1))
        p = np.exp(a_ex - m[:, None])
        alpha = np.exp(a_un - m[:, None])
        num = p @ v[idx] + alpha @ vsum[uns]
        if Hblocks is None:
            num += scale * (qi @ Hbar) * alpha.sum(axis=1)[:, None]
        else:
            for c, j in enumerate(uns):
                num += scale * alpha[:, c:c + 1] * (qi @ Hblocks[j])
        den = p.sum(axis=1) + alpha @ np.asarray([valid[j] for j in uns], dtype=np.float64)
        outs.append(num / den[:, None])
        lses.append(m + np.log(den))
    return np.concatenate(outs), np.concatenate(lses)


def zeroth_order_head(q, k, v, row_ptr, col_idx, block, scale, kbar, vsum, qblocks=None):
    """PISA without the first-order correction (Hbar = 0): used by the Taylor-order
    pins to show that the correction removes the first-order error term."""
    d = np.asarray(q).shape[1]
    return pisa_head(q, k, v, row_ptr, col_idx, block, scale, kbar, vsum,
                     np.zeros((d, np.asarray(v).shape[1])), qblocks=qblocks)


# ----------------------------------------------------------------------------------
# Batched wrappers over [batch, heads, L, d]
# ----------------------------------------------------------------------------------
def _bh(x):
    x = np.asarray(x, dtype=np.float64)
    return x.reshape(-1, x.shape[-2], x.shape[-1])


def precompute(k, v, block, key_valid=None):
    """Apply precompute_head to every (batch, head); arrays stacked on axis 0."""
    res = [precompute_head(kk, vv, block, key_valid) for kk, vv in zip(_bh(k), _bh(v))]
    return tuple(np.stack([r[n] for r in res]) for n in range(5))


def route(q, kbar, Mnorm, block, k_top, lam, scale, key_valid=None):
    """Per-head routing. row_ptr is [heads, M+1] (flattened) holding absolute offsets
    into the stacked col_idx; head h's lists start at h * M * k_top."""
    qs = _bh(q)
    M = qs.shape[1] // block
    rps, cis, scs = [], [], []
    for h, qq in enumerate(qs):
        rp, ci, sc = route_head(qq, kbar[h], Mnorm[h], block, k_top, lam, scale, key_valid)
        rps.append(rp + h * M * k_top)
        cis.append(ci)
        scs.append(sc)
    return (np.concatenate(rps).astype(np.int32), np.concatenate(cis).astype(np.int32),
            np.stack(scs))


def head_csr(row_ptr, col_idx, h, M, per_head):
    """The CSR of head h, with row offsets rebased to 0."""
    if not per_head:
        return np.asarray(row_ptr), np.asarray(col_idx)
    rp = np.asarray(row_ptr[h * (M + 1):(h + 1) * (M + 1)], dtype=np.int64)
    return (rp - rp[0]).astype(np.int32), np.asarray(col_idx[rp[0]:rp[-1]])
