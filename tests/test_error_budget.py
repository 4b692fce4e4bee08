"""Error budget of the tensor-core decode step's precision choices, computed on the CPU.

The tensor-core decode kernel reformulates the block-hybrid layer ("Retrofitting Linear
Attention into Diffusion Language Models", §3.1) for the hardware:
- u = qW and the block scores s = qK^T are computed in fp32 from bf16 operands;
- e+ = 2^{(u - max u) log2 e} and e- = 2^{(min u - u) log2 e} stay unnormalised in fp32 and are
  read by the tensor cores as tf32, against the fp32 states S, also read as tf32;
- the block softmax weights P = w 2^{s log2e/sqrt d - m} are scaled by kappa = sum e+ / 2^{-m}
  and rounded to bf16 for the P V product, which joins A+ = e+ S+ in the same accumulator;
- the epilogue applies f+/- = 2^{-m} / (sum e+/- . den) in fp32, and the output is bf16.

This test applies exactly those roundings, step by step in NumPy (bf16 round-to-nearest-even,
tf32 as fp32 with the low 13 mantissa bits dropped, fp32 after every step), at the serving
shape. The shape is d 128, F 256, 4 query heads per KV head, 32-token blocks, states of
1024-token prefixes and a random gate. It then compares the result with the float64
oracle. It shows how much of the parity tolerance (max-abs 2e-2, rel-L2 5e-3) the design's
roundings use by themselves, and which rounding dominates. What is left covers summation
order and the hardware exp2 approximation. A second model applies the commit kernel's
roundings in the same way: phi of the block's keys in fp32, rounded to bf16 for the phi^T V
product, fp32 accumulation and fp32 read-modify-write of S and Z. It shows what 32
sequential commits cost the states, and what that costs the decode step. The models share
no code with the CUDA path.
"""
import numpy as np

from linear_attention_diffusion_hedgehog_b200 import inputs
from oracle import bha_ref as ref

LOG2E = 1.0 / np.log(2.0)
TOL = dict(max_abs=2e-2, rel_l2=5e-3)


def f32(x):
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)


def tf32(x):
    b = np.ascontiguousarray(np.asarray(x, np.float32)).view(np.uint32) & np.uint32(0xFFFFE000)
    return b.view(np.float32).astype(np.float64)


def bf16(x):
    return inputs.bf16_round(np.asarray(x, np.float32)).astype(np.float64)


def exact(x):
    return np.asarray(x, np.float64)


def model_unit(q, k, v, S, Z, W, w, state_read=tf32):
    """One (request, KV head) tile: q [rows, d] (rows = 4 t + head), k, v [n, d], S [F, d],
    Z [F], W [d, F/2], w [rows] gate.  Returns the bf16 output rows as float64."""
    d, Fh = q.shape[1], W.shape[1]
    a = f32(f32(q @ W) * LOG2E)
    bp, bm = a.max(1, keepdims=True), a.min(1, keepdims=True)
    ep, en = f32(np.exp2(a - bp)), f32(np.exp2(bm - a))
    esp, esm = f32(ep.sum(1)), f32(en.sum(1))
    zsp, zsm = f32(ep @ Z[:Fh]), f32(en @ Z[Fh:])
    Ap = f32(tf32(ep) @ state_read(S[:Fh]))
    Am = f32(tf32(en) @ state_read(S[Fh:]))
    s = f32(q @ k.T)
    sl = LOG2E / np.sqrt(d)
    m2 = np.clip(s.max(1, keepdims=True) * sl, -6 * LOG2E, 90.0)
    em = np.exp2(-m2)[:, 0]
    kappa = f32(esp / em)
    P = bf16(w[:, None] * np.exp2(s * sl - m2) * kappa[:, None])
    Ap = f32(Ap + P @ v)
    den = f32(f32(P.sum(1)) / kappa + em * (zsp / esp + zsm / esm))
    return bf16(f32(em / esp / den)[:, None] * Ap + f32(em / esm / den)[:, None] * Am)


def model_decode(c, S, Z, state_read=tf32):
    w = 1.0 / (1.0 + np.exp(-c.alpha.astype(np.float64)))
    G = c.Hq // c.Hkv
    O = np.zeros((c.T, c.Hq, c.d))
    for r in range(c.R):
        lo, hi = c.cu_blk[r], c.cu_blk[r + 1]
        n = hi - lo
        for g in range(c.Hkv):
            q = c.Q[lo:hi, G * g:G * g + G].astype(np.float64).reshape(n * G, c.d)
            out = model_unit(q, c.K[lo:hi, g].astype(np.float64), c.V[lo:hi, g].astype(np.float64),
                             S[r, g], Z[r, g], c.W[g].astype(np.float64),
                             np.tile(w[G * g:G * g + G], n), state_read)
            O[lo:hi, G * g:G * g + G] = out.reshape(n, G, c.d)
    return O


def _serving_case(q_scale=1.0):
    c = inputs.decode_case(R=8, Hq=16, Hkv=4, d=128, F=256, block_lens=32, prefix_lens=1024,
                           seed=2, dtype="bf16", with_alpha=True)
    c.Q = (c.Q * np.float32(q_scale)).astype(np.float32)   # powers of two: exact in bf16
    S = np.zeros((c.R, c.Hkv, c.F, c.d))
    Z = np.zeros((c.R, c.Hkv, c.F))
    for r in range(c.R):
        lo, hi = c.cu_pre[r], c.cu_pre[r + 1]
        for g in range(c.Hkv):
            S[r, g], Z[r, g] = ref.state_from_tokens(c.K_pre[lo:hi, g], c.V_pre[lo:hi, g], c.W[g])
    return c, f32(S), f32(Z)


def _err(got, want):
    diff = got - want
    return np.abs(diff).max(), np.linalg.norm(diff) / np.linalg.norm(want)


def test_design_roundings_use_under_half_the_tolerance():
    c, S, Z = _serving_case()
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S, Z, c.W, c.alpha)
    max_abs, rel = _err(model_decode(c, S, Z), want)
    assert max_abs <= 0.5 * TOL["max_abs"] and rel <= 0.5 * TOL["rel_l2"], (max_abs, rel)
    # the final bf16 rounding of the output is most of it
    _, rel_out = _err(bf16(want), want)
    assert rel_out >= 0.6 * rel, (rel_out, rel)


def test_state_read_precision_is_not_what_limits_accuracy():
    """Reading the fp32 states as tf32 (what the tensor cores take without conversion) costs
    nothing measurable at this shape: the result matches an exact fp32 read to within a
    tenth of the modelled error."""
    c, S, Z = _serving_case()
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S, Z, c.W, c.alpha)
    _, rel_tf32 = _err(model_decode(c, S, Z, tf32), want)
    _, rel_fp32 = _err(model_decode(c, S, Z, exact), want)
    assert abs(rel_tf32 - rel_fp32) <= 0.1 * rel_fp32, (rel_tf32, rel_fp32)


def test_budget_holds_for_large_queries():
    """Queries scaled by 4 (wider feature spread, peakier block softmax): still within the
    tolerance by the model alone."""
    c, S, Z = _serving_case(q_scale=4.0)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S, Z, c.W, c.alpha)
    max_abs, rel = _err(model_decode(c, S, Z), want)
    assert max_abs <= TOL["max_abs"] and rel <= TOL["rel_l2"], (max_abs, rel)


def model_phi(x, W):
    """phi as the commit kernel forms it: u in fp32, each half's softmax in fp32."""
    u = f32(x @ W)

    def half(z):
        e = f32(np.exp(z - z.max(-1, keepdims=True)))
        return f32(e / f32(e.sum(-1, keepdims=True)))

    return np.concatenate([half(u), half(-u)], -1)


def model_commits(Kp, Vp, W, blk=32):
    """States built by sequential commits of `blk`-token blocks: S += bf16(phi)^T V and
    Z += sum of bf16(phi), accumulated in fp32 and stored in fp32."""
    S = np.zeros((2 * W.shape[1], W.shape[0]))
    Z = np.zeros(2 * W.shape[1])
    for s0 in range(0, Kp.shape[0], blk):
        P = bf16(model_phi(Kp[s0:s0 + blk].astype(np.float64), W))
        S = f32(S + f32(P.T @ Vp[s0:s0 + blk].astype(np.float64)))
        Z = f32(Z + f32(P.sum(0)))
    return S, Z


def test_commit_roundings_and_the_decode_on_committed_states():
    """32 commits of 32 tokens: the states stay within half the tolerance of the oracle's
    one-shot states, and the decode step on them within half the tolerance of the oracle."""
    c, S, Z = _serving_case()
    Sm, Zm = np.zeros_like(S), np.zeros_like(Z)
    for r in range(c.R):
        lo, hi = c.cu_pre[r], c.cu_pre[r + 1]
        for g in range(c.Hkv):
            Sm[r, g], Zm[r, g] = model_commits(c.K_pre[lo:hi, g], c.V_pre[lo:hi, g],
                                               c.W[g].astype(np.float64))
    for got, ref_state in ((Sm, S), (Zm, Z)):
        max_abs, rel = _err(got, ref_state)
        assert max_abs <= 0.5 * TOL["max_abs"] and rel <= 0.5 * TOL["rel_l2"], (max_abs, rel)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S, Z, c.W, c.alpha)
    max_abs, rel = _err(model_decode(c, Sm, Zm), want)
    assert max_abs <= 0.5 * TOL["max_abs"] and rel <= 0.5 * TOL["rel_l2"], (max_abs, rel)
