"""Float64 CPU oracle for block-hybrid attention (test infrastructure only).

What this module is
-------------------
A plain, slow, obviously-correct NumPy float64 statement of what the block-hybrid
attention layer computes, written from "Retrofitting Linear Attention into Diffusion
Language Models":

* §2.2 "Linear attention": causal softmax attention, eq. (1) (linear attention with a
  feature map phi) and the recurrent states S_i, Z_i.
* §3.1 "Block-hybrid attention": within-block softmax sums sm_num / sm_den, the Hedgehog
  feature map phi(x) = [softmax(xW), softmax(-xW)], the committed states S_n / Z_n and
  their block-commit update, the cross-block read lin_num / lin_den, and the gated
  shared-normaliser merge out = (w sm_num + lin_num) / (w sm_den + lin_den), w = sigmoid(alpha).

It is test infrastructure: only the test suite, the package smoke check and the bench's
CPU-baseline leg may import it.  It shares no code with the CUDA path and imports
nothing from the package.

Conventions (readings where the paper leaves a step open)
---------------------------------------------------------
* F is the TOTAL feature dimension: phi(x) has F entries, W is d x F/2 (the paper writes
  phi in R^{2F} with W in R^{d x F}; only the naming differs).
* W and the states S/Z belong to a KV head; the G = Hq/Hkv query heads of a group share
  them (the paper keeps them per query head; grouping is this library's layout choice,
  and Hkv = Hq reproduces the paper's per-query-head layout exactly).
* Query head h reads group g = floor(h / G) (contiguous GQA groups).
* The gate w = sigmoid(alpha_h) multiplies the softmax branch; alpha absent means w = 1.
* The 1/sqrt(d) temperature applies to the softmax branch only; phi has none.
* Keys of the active block enter the softmax branch only; the linear branch reads the
  states of committed blocks only (no double counting).
* A 0/0 shared denominator (possible only with w = 0 and an empty prefix) gives 0.
* Token-major ragged layout: request r owns rows cu_blk[r] .. cu_blk[r+1]-1.

Parity pins live in tests/test_oracle.py (closed forms, a hand-worked example,
brute-force prefix sums, commit associativity, invariants, and an independent library
routine for plain softmax attention).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "softmax_last",
    "phi",
    "featuremap",
    "state_from_tokens",
    "commit",
    "block_hybrid_head",
    "block_hybrid_head_bruteforce",
    "hybrid_attn",
    "commit_block",
    "softmax_attn_head",
    "full_prefix_attn",
    "gate",
]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def softmax_last(u):
    """softmax over the last axis: exp(u_f) / sum_f' exp(u_f').

    Evaluated as exp(u - max u) / sum exp(u - max u); subtracting a constant from every
    entry leaves a softmax unchanged, so this is the same function without overflow.
    """
    u = _f64(u)
    e = np.exp(u - u.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def phi(x, W):
    """Hedgehog feature map (§3.1): phi(x) = [softmax(xW), softmax(-xW)].

    x: [..., d] rows; W: [d, F/2].  Returns [..., F]: the first F/2 entries are the
    softmax of xW, the last F/2 the softmax of -xW, each normalised over its own half.
    """
    u = _f64(x) @ _f64(W)
    return np.concatenate([softmax_last(u), softmax_last(-u)], axis=-1)


def gate(alpha):
    """Per-query-head gate w = sigmoid(alpha) (§3.1, "Combining the two branches")."""
    return 1.0 / (1.0 + np.exp(-_f64(alpha)))


def state_from_tokens(K, V, W):
    """Recurrent states over a set of tokens (§2.2; §3.1 definition of S_n, Z_n).

    S = sum_t phi(k_t) v_t^T  (F x d),   Z = sum_t phi(k_t)  (F).
    K, V: [n, d].  n = 0 gives zero states.
    The sum of outer products over t is written as the matrix product phi(K)^T V.
    """
    d = np.asarray(W).shape[0]
    K = _f64(K).reshape(-1, d)
    V = _f64(V).reshape(K.shape[0], np.asarray(V).shape[-1])
    P = phi(K, W)  # [n, F]
    return P.T @ V, P.sum(axis=0)


def commit(S, Z, K_blk, V_blk, W):
    """Block commit (§3.1): S_n = S_{n-1} + sum_{t in B_n} phi(k_t) v_t^T, Z likewise."""
    dS, dZ = state_from_tokens(K_blk, V_blk, W)
    return _f64(S) + dS, _f64(Z) + dZ


def _merge(sm_num, sm_den, lin_num, lin_den, w):
    """Shared-normaliser merge (§3.1): (w sm_num + lin_num) / (w sm_den + lin_den)."""
    num = w * sm_num + lin_num
    den = w * sm_den + lin_den
    out = np.zeros_like(num)
    ok = den != 0.0
    out[ok] = num[ok] / den[ok][:, None]
    return out


def block_hybrid_head(q, k, v, S, Z, W, w=1.0):
    """One query head over one active block (§3.1).

    q, k, v: [b, d], the active block's rows for this head (k, v from its KV head).
    S: [F, d], Z: [F], the committed states S_{n-1}, Z_{n-1}.
      a_ij    = exp(q_i . k_j / sqrt(d)) for every j in the block (bidirectional, unmasked)
      sm_num  = sum_j a_ij v_j,           sm_den  = sum_j a_ij
      lin_num = phi(q_i)^T S,             lin_den = phi(q_i)^T Z
      out_i   = (w sm_num + lin_num) / (w sm_den + lin_den)
    The exponent is taken unshifted, as written; float64 keeps it exact for |q.k/sqrt d| < 700.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    d = q.shape[-1]
    a = np.exp((q @ k.T) / np.sqrt(d))
    sm_num = a @ v
    sm_den = a.sum(axis=1)
    fq = phi(q, W)
    lin_num = fq @ _f64(S)
    lin_den = fq @ _f64(Z)
    return _merge(sm_num, sm_den, lin_num, lin_den, w)


def block_hybrid_head_bruteforce(q, k, v, K_pre, V_pre, W, w=1.0):
    """Same output as block_hybrid_head, with the linear branch as an explicit prefix sum.

    Linear attention (§2.2, eq. (1)) replaces exp(q.k/sqrt d) by phi(q)^T phi(k_t), so
      lin_num = sum_t (phi(q)^T phi(k_t)) v_t,   lin_den = sum_t phi(q)^T phi(k_t)
    over the committed prefix tokens t.  No recurrent state is formed.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    d = q.shape[-1]
    a = np.exp((q @ k.T) / np.sqrt(d))
    sm_num = a @ v
    sm_den = a.sum(axis=1)
    fq = phi(q, W)
    b = q.shape[0]
    lin_num = np.zeros((b, d))
    lin_den = np.zeros(b)
    for t in range(np.asarray(K_pre).shape[0]):
        kern = fq @ phi(K_pre[t], W)  # [b]
        lin_num += np.outer(kern, _f64(V_pre[t]))
        lin_den += kern
    return _merge(sm_num, sm_den, lin_num, lin_den, w)


def featuremap(x, W):
    """phi applied to a token-major tensor x [T, H, d] with per-head weights W [Hw, d, F/2].

    Head h uses W[floor(h * Hw / H)].  Returns [T, H, F].
    """
    x = _f64(x)
    T, H, d = x.shape
    Hw = np.asarray(W).shape[0]
    F = 2 * np.asarray(W).shape[2]
    out = np.zeros((T, H, F))
    for h in range(H):
        out[:, h, :] = phi(x[:, h, :], W[(h * Hw) // H])
    return out


def hybrid_attn(cu_blk, Q, K, V, S, Z, W, alpha=None, state_slot=None):
    """Block-hybrid attention for a ragged batch of requests (one denoising step, one layer).

    cu_blk: [R+1] row offsets; Q: [T, Hq, d]; K, V: [T, Hkv, d];
    S: [slots, Hkv, F, d]; Z: [slots, Hkv, F]; W: [Hkv, d, F/2];
    alpha: [Hq] or None (w = 1); state_slot: [R] or None (request r uses slot r).
    Returns O [T, Hq, d].
    """
    Q = _f64(Q)
    T, Hq, d = Q.shape
    Hkv = np.asarray(K).shape[1]
    G = Hq // Hkv
    O = np.zeros((T, Hq, d))
    R = len(cu_blk) - 1
    for r in range(R):
        lo, hi = int(cu_blk[r]), int(cu_blk[r + 1])
        if hi == lo:
            continue
        slot = r if state_slot is None else int(state_slot[r])
        for h in range(Hq):
            g = h // G
            w = 1.0 if alpha is None else float(gate(alpha[h]))
            O[lo:hi, h] = block_hybrid_head(
                Q[lo:hi, h], K[lo:hi, g], V[lo:hi, g], S[slot, g], Z[slot, g], W[g], w
            )
    return O


def commit_block(cu_blk, K, V, W, S, Z, state_slot=None):
    """Fold each request's finished block into its states (§3.1 commit).  Returns new S, Z."""
    S = _f64(S).copy()
    Z = _f64(Z).copy()
    Hkv = np.asarray(K).shape[1]
    R = len(cu_blk) - 1
    for r in range(R):
        lo, hi = int(cu_blk[r]), int(cu_blk[r + 1])
        slot = r if state_slot is None else int(state_slot[r])
        for g in range(Hkv):
            S[slot, g], Z[slot, g] = commit(S[slot, g], Z[slot, g], K[lo:hi, g], V[lo:hi, g], W[g])
    return S, Z


def softmax_attn_head(q, k, v):
    """Exact softmax attention of each query over every given key (§2.2, without the
    causal restriction: every listed key is visible).  q: [b, d]; k, v: [n, d]."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    d = q.shape[-1]
    s = (q @ k.T) / np.sqrt(d)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p @ v) / p.sum(axis=1, keepdims=True)


def full_prefix_attn(cu_blk, kv_len, Q, Kc, Vc):
    """The softmax teacher: each active-block query attends to its request's whole cache
    (committed prefix followed by the active block), unmasked.

    Q: [T, Hq, d]; Kc, Vc: [R, Hkv, L, d] with request r's keys at [r, g, :kv_len[r]].
    Returns O [T, Hq, d].
    """
    Q = _f64(Q)
    T, Hq, d = Q.shape
    Hkv = np.asarray(Kc).shape[1]
    G = Hq // Hkv
    O = np.zeros((T, Hq, d))
    for r in range(len(cu_blk) - 1):
        lo, hi = int(cu_blk[r]), int(cu_blk[r + 1])
        n = int(kv_len[r])
        if hi == lo or n == 0:
            continue
        for h in range(Hq):
            g = h // G
            O[lo:hi, h] = softmax_attn_head(Q[lo:hi, h], Kc[r, g, :n], Vc[r, g, :n])
    return O
