"""Plain float64 CPU oracle of the hybrid Top-k+Top-p block-sparse attention path.

TEST INFRASTRUCTURE. This module is the parity authority for the CUDA library
in ``trainable_block_sparse_pooled_b200``. It is slow on purpose: every step is
written as the pages state it, with library primitives (matmul, sort, exp) as
steps and no blocking, fusion or reordering beyond what the method defines.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import it; the CUDA path never does, and the two share no
code.

Sources (web summaries of arXiv 2602.13515, "SpargeAttention2: Trainable Sparse
Attention via Hybrid Top-k+Top-p Masking and Distillation Fine-Tuning"):

* [rainbus]  paper.rainbus.top summary. Sections used: 前置知识 (prerequisites:
  "稀疏注意力" sparse attention, "Top-k 和 Top-p 掩码", "块稀疏注意力" block-sparse
  attention), 研究动机 (motivation, the two worked rows), 方法步骤详情 (method
  steps 1-4), 技术新颖性 (novelty: union formula and error decomposition).
* [gist]     gist.science summary, section 2 "Methodology", A "Hybrid Top-k +
  Top-p Masking" and C "Efficient Kernel Implementation".
* [gist-nl]  gist.science/nl summary, "Methodologie" 1 (the union formula).
* [chatpaper] chatpaper.ai abstract ("efficient trainable sparse attention
  implementation": forward and backward).

Readings taken where the pages are silent:

* pool = arithmetic mean over the rows of a block; the last block of a ragged
  sequence is averaged over its valid rows only.
* block counts T_m = ceil(N / b_q), T_n = ceil(N / b_kv).
* Top-k count K = clamp(floor(k * T_n + 1/2), 1, T_n), computed in double from
  the float32 k (pins "ten 0.1 blocks, Top-20% keeps 2").
* Top-p is inclusive ("reaches p"): walk the row in rank order and keep a block
  while the mass of the blocks before it is below p. Masses are quantised to
  q_j = floor(P_j * 2^32) and p to floor(p * 2^32) so that the running sum is
  exact integer arithmetic (pins "[0.6 sink, 0.2, 0.1, ...] under Top-p 60%
  keeps only the sink").
* rank order = (P value descending, block index ascending); the union of the
  Top-k and Top-p sets is then the longer of two prefixes of that order.
* selection runs on a float32 P-bar row (the oracle rounds its float64 P-bar to
  float32 first); attention and gradients hold the mask constant.
* attention is bidirectional (no causal mask); LSE is the natural log of the
  row sum of exp(scaled logits).
"""

from __future__ import annotations

import math

import numpy as np

TWO32 = 4294967296  # 2**32, the Top-p mass quantum


# --------------------------------------------------------------------------
# Step 1: block partition  ([rainbus] 方法步骤详情, step 1)
# --------------------------------------------------------------------------
def block_counts(N: int, bq: int, bkv: int) -> tuple[int, int]:
    """T_m query blocks of b_q rows and T_n key/value blocks of b_kv rows.

    The pages write T_m = N / b_q and T_n = N / b_kv; a ragged last block is
    counted (ceil).
    """
    return -(-N // bq), -(-N // bkv)


# --------------------------------------------------------------------------
# Step 2a: block pooling  ([rainbus] 方法步骤详情, step 2: pool(Q), pool(K))
# --------------------------------------------------------------------------
def pool_blocks(X: np.ndarray, b: int) -> np.ndarray:
    """Mean of each run of ``b`` rows of X[..., N, d] (last run may be short)."""
    X = np.asarray(X, dtype=np.float64)
    N = X.shape[-2]
    T = -(-N // b)
    out = np.empty(X.shape[:-2] + (T, X.shape[-1]), dtype=np.float64)
    for t in range(T):
        lo, hi = t * b, min(N, (t + 1) * b)
        out[..., t, :] = X[..., lo:hi, :].sum(axis=-2) / float(hi - lo)
    return out


# --------------------------------------------------------------------------
# Step 2b: pooled block attention  ([rainbus] 方法步骤详情, step 2)
#   P-bar = softmax(pool(Q) pool(K)^T / sqrt(d)), row by row
# --------------------------------------------------------------------------
def pooled_attention(Qbar: np.ndarray, Kbar: np.ndarray, d: int) -> np.ndarray:
    S = np.matmul(Qbar, np.swapaxes(Kbar, -1, -2)) / math.sqrt(d)
    S = S - S.max(axis=-1, keepdims=True)
    E = np.exp(S)
    return E / E.sum(axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# Step 3: hybrid Top-k + Top-p selection
#   [rainbus] 前置知识 "Top-k 和 Top-p 掩码"; 方法步骤详情 step 3;
#   技术新颖性 (M_ij = 1 iff j in Top-k(P_i,:, k%) U Top-p(P_i,:, p%));
#   [gist] 2A; [gist-nl] Methodologie 1 (same formula)
# --------------------------------------------------------------------------
def rank_order(row32: np.ndarray) -> np.ndarray:
    """Block ids sorted by (value descending, block id ascending)."""
    v = np.asarray(row32, dtype=np.float32).astype(np.float64)
    ids = np.arange(v.shape[0])
    return np.lexsort((ids, -v))


def topk_count(k_frac: float, Tn: int) -> int:
    """Number of blocks Top-k keeps: round-half-up of k * T_n, at least 1."""
    kd = float(np.float32(k_frac))
    K = int(math.floor(kd * Tn + 0.5))
    return max(1, min(Tn, K))


def topp_count(row32: np.ndarray, order: np.ndarray, p_frac: float) -> int:
    """Size of the smallest rank-order prefix whose mass reaches p.

    Rank r is kept while the (quantised) mass of ranks 0..r-1 is below p.
    """
    v = np.asarray(row32, dtype=np.float32).astype(np.float64)
    q = np.floor(v * TWO32).astype(np.uint64)            # exact for float32 v in [0, 1]
    thr = int(math.floor(float(np.float32(p_frac)) * TWO32))
    before = 0
    R = 0
    for j in order:
        if before < thr:
            R += 1
        else:
            break
        before += int(q[j])
    return R


def select_row(row32: np.ndarray, k_frac: float, p_frac: float) -> np.ndarray:
    """Kept block ids (ascending) of one float32 P-bar row."""
    row32 = np.asarray(row32, dtype=np.float32)
    order = rank_order(row32)
    K = topk_count(k_frac, row32.shape[0])
    R = topp_count(row32, order, p_frac)
    n = max(K, R)          # both sets are prefixes of `order`: the union is the longer
    return np.sort(order[:n])


def select_blocks(pbar32: np.ndarray, k_frac: float, p_frac: float) -> np.ndarray:
    """Boolean block mask [..., T_m, T_n] from float32 P-bar rows."""
    pbar32 = np.asarray(pbar32, dtype=np.float32)
    lead = pbar32.shape[:-1]
    flat = pbar32.reshape(-1, pbar32.shape[-1])
    mask = np.zeros(flat.shape, dtype=bool)
    for r in range(flat.shape[0]):
        mask[r, select_row(flat[r], k_frac, p_frac)] = True
    return mask.reshape(lead + (pbar32.shape[-1],))


def block_mask(Q, K, bq: int, bkv: int, k_frac: float, p_frac: float):
    """Steps 1-3. Returns (P-bar float64, P-bar float32, bool mask [B,H,T_m,T_n])."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    d = Q.shape[-1]
    pbar = pooled_attention(pool_blocks(Q, bq), pool_blocks(K, bkv), d)
    pbar32 = pbar.astype(np.float32)
    return pbar, pbar32, select_blocks(pbar32, k_frac, p_frac)


# --------------------------------------------------------------------------
# Step 4: block-sparse attention  ([rainbus] 前置知识 "稀疏注意力": P <- P (.) M,
#   masked Q_i K_j^T and P_ij V_j are skipped; "块稀疏注意力": each (i, j) block
#   pair is all-kept or all-masked; 方法步骤详情 step 4)
# --------------------------------------------------------------------------
def token_mask(mask_blocks: np.ndarray, N: int, bq: int, bkv: int) -> np.ndarray:
    """Expand a [T_m, T_n] block mask to the [N, N] token mask it stands for."""
    mask_blocks = np.asarray(mask_blocks, dtype=bool)
    r = np.arange(N) // bq
    c = np.arange(N) // bkv
    return mask_blocks[r][:, c]


def _kept_cols(mask_row: np.ndarray, N: int, bkv: int) -> np.ndarray:
    cols = [np.arange(j * bkv, min(N, (j + 1) * bkv)) for j in np.flatnonzero(mask_row)]
    return np.concatenate(cols) if cols else np.zeros(0, dtype=np.int64)


def _row_block_softmax(Qi, Kc, scale):
    s = (Qi @ Kc.T) * scale
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


def masked_attn_fwd_rows(Q, K, V, mask, bq, bkv, scale, b, h, qblocks):
    """Forward for selected query blocks of head (b, h): {i: (O_i, LSE_i)}."""
    N = Q.shape[-2]
    out = {}
    Kh = np.asarray(K[b, h], dtype=np.float64)
    Vh = np.asarray(V[b, h], dtype=np.float64)
    for i in qblocks:
        lo, hi = i * bq, min(N, (i + 1) * bq)
        Qi = np.asarray(Q[b, h, lo:hi], dtype=np.float64)
        cols = _kept_cols(mask[b, h, i], N, bkv)
        P, lse = _row_block_softmax(Qi, Kh[cols], scale)
        out[i] = (P @ Vh[cols], lse)
    return out


def masked_attn_fwd(Q, K, V, mask, bq: int, bkv: int, scale: float | None = None):
    """O [B,H,N,d] and LSE [B,H,N] under a block mask [B,H,T_m,T_n]."""
    B, H, N, d = Q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    Tm = -(-N // bq)
    O = np.zeros((B, H, N, V.shape[-1]), dtype=np.float64)
    LSE = np.zeros((B, H, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            rows = masked_attn_fwd_rows(Q, K, V, mask, bq, bkv, scale, b, h, range(Tm))
            for i, (Oi, li) in rows.items():
                O[b, h, i * bq:i * bq + Oi.shape[0]] = Oi
                LSE[b, h, i * bq:i * bq + Oi.shape[0]] = li
    return O, LSE


# --------------------------------------------------------------------------
# Backward through the same block mask ([rainbus] 核心方法: the kernel covers
#   forward and backward; [chatpaper] abstract (ii)). Standard softmax-attention
#   calculus with the mask held constant.
# --------------------------------------------------------------------------
def masked_attn_bwd(Q, K, V, mask, dO, bq: int, bkv: int, scale: float | None = None,
                    heads=None):
    """dQ, dK, dV [B,H,N,d]. ``heads`` restricts to a list of (b, h)."""
    B, H, N, d = Q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    Tm = -(-N // bq)
    dQ = np.zeros((B, H, N, d), dtype=np.float64)
    dK = np.zeros((B, H, N, d), dtype=np.float64)
    dV = np.zeros((B, H, N, V.shape[-1]), dtype=np.float64)
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in heads:
        Kh = np.asarray(K[b, h], dtype=np.float64)
        Vh = np.asarray(V[b, h], dtype=np.float64)
        for i in range(Tm):
            lo, hi = i * bq, min(N, (i + 1) * bq)
            Qi = np.asarray(Q[b, h, lo:hi], dtype=np.float64)
            dOi = np.asarray(dO[b, h, lo:hi], dtype=np.float64)
            cols = _kept_cols(mask[b, h, i], N, bkv)
            P, _ = _row_block_softmax(Qi, Kh[cols], scale)
            dV[b, h, cols] += P.T @ dOi
            dP = dOi @ Vh[cols].T
            D = (P * dP).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dQ[b, h, lo:hi] = (dS @ Kh[cols]) * scale
            dK[b, h, cols] += (dS.T @ Qi) * scale
    return dQ, dK, dV


def masked_attn_bwd_blocks(Q, K, V, mask, dO, bq: int, bkv: int, scale, b: int, h: int, qblocks, kvblocks):
    """Sampled backward of head (b, h): dQ of ``qblocks`` and dK, dV of ``kvblocks``.

    Same arithmetic as ``masked_attn_bwd``, restricted to the q-blocks that are
    sampled or keep a sampled kv-block. Returns ({i: dQ_i}, {j: (dK_j, dV_j)}).
    """
    N = Q.shape[-2]
    Tm = -(-N // bq)
    qset, kvset = set(qblocks), set(kvblocks)
    Kh = np.asarray(K[b, h], dtype=np.float64)
    Vh = np.asarray(V[b, h], dtype=np.float64)
    dQ = {}
    dKV = {j: (np.zeros((min(N, (j + 1) * bkv) - j * bkv, K.shape[-1])),
               np.zeros((min(N, (j + 1) * bkv) - j * bkv, V.shape[-1]))) for j in kvset}
    for i in range(Tm):
        kept = set(np.flatnonzero(mask[b, h, i]).tolist())
        if i not in qset and not (kept & kvset):
            continue
        lo, hi = i * bq, min(N, (i + 1) * bq)
        Qi = np.asarray(Q[b, h, lo:hi], dtype=np.float64)
        dOi = np.asarray(dO[b, h, lo:hi], dtype=np.float64)
        cols = _kept_cols(mask[b, h, i], N, bkv)
        P, _ = _row_block_softmax(Qi, Kh[cols], scale)
        dP = dOi @ Vh[cols].T
        D = (P * dP).sum(axis=1, keepdims=True)
        dS = P * (dP - D)
        if i in qset:
            dQ[i] = (dS @ Kh[cols]) * scale
        pos = 0
        for j in sorted(kept):
            w = min(N, (j + 1) * bkv) - j * bkv
            if j in kvset:
                dKV[j][0][:] += (dS[:, pos:pos + w].T @ Qi) * scale
                dKV[j][1][:] += P[:, pos:pos + w].T @ dOi
            pos += w
    return dQ, dKV


def masked_attn_bwd_rows(Q, K, V, mask, dO, bq: int, bkv: int, scale, b: int, h: int, qblocks):
    """Backward contributions of the q-blocks ``qblocks`` of head (b, h).

    Returns ({i: dQ_i}, dK_part, dV_part) where dK_part / dV_part [N, d] hold
    the sums over the listed q-blocks only (the full dK, dV sum every q-block).
    """
    N = Q.shape[-2]
    Kh = np.asarray(K[b, h], dtype=np.float64)
    Vh = np.asarray(V[b, h], dtype=np.float64)
    dQ = {}
    dKp = np.zeros((N, K.shape[-1]))
    dVp = np.zeros((N, V.shape[-1]))
    for i in qblocks:
        lo, hi = i * bq, min(N, (i + 1) * bq)
        Qi = np.asarray(Q[b, h, lo:hi], dtype=np.float64)
        dOi = np.asarray(dO[b, h, lo:hi], dtype=np.float64)
        cols = _kept_cols(mask[b, h, i], N, bkv)
        P, _ = _row_block_softmax(Qi, Kh[cols], scale)
        dVp[cols] += P.T @ dOi
        dP = dOi @ Vh[cols].T
        D = (P * dP).sum(axis=1, keepdims=True)
        dS = P * (dP - D)
        dQ[i] = (dS @ Kh[cols]) * scale
        dKp[cols] += (dS.T @ Qi) * scale
    return dQ, dKp, dVp


def attn_flops(mask, N: int, bq: int, bkv: int, d: int) -> float:
    """Forward flops 4*d*sum over kept (i, j) of valid q rows x valid kv cols."""
    mask = np.asarray(mask, dtype=bool)
    Tm, Tn = mask.shape[-2], mask.shape[-1]
    rows = np.array([min(N, (i + 1) * bq) - i * bq for i in range(Tm)], dtype=np.float64)
    cols = np.array([min(N, (j + 1) * bkv) - j * bkv for j in range(Tn)], dtype=np.float64)
    per = rows[:, None] * cols[None, :]
    return float(4.0 * d * (mask * per).sum())
