"""Pins for the float64 oracle: each test checks it against something other than itself.

Source of every fact used here: "Retrofitting Linear Attention into Diffusion Language
Models", §2.2 (softmax attention, eq. (1), recurrent states) and §3.1 (block-hybrid
attention).  The pins are chosen so that a plausible slip in the oracle (a wrong sign on
the -xW half, a transposed W, a dropped normaliser term, 1/d instead of 1/sqrt d, block keys
counted in the linear branch, a wrong GQA index) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

from oracle import bha_ref as ref
from linear_attention_diffusion_hedgehog_b200 import inputs

RNG = np.random.default_rng(1234)


def _sdpa64(q, k, v):
    """Plain softmax attention through torch's library routine, in float64 on the CPU."""
    tq = torch.from_numpy(np.asarray(q, np.float64))[None, None]
    tk = torch.from_numpy(np.asarray(k, np.float64))[None, None]
    tv = torch.from_numpy(np.asarray(v, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, 0].numpy()


# ---------------------------------------------------------------- feature map (§3.1)

def test_phi_hand_values(golden):
    g = golden("hand_phi.txt")
    W = g["W"][0].reshape(2, 2)
    for x, want in zip(g["x"], g["phi"]):
        np.testing.assert_allclose(ref.phi(x, W), want, rtol=0, atol=1e-15)


def test_phi_halves_are_simplices():
    d, Fh = 24, 40
    x = RNG.standard_normal((50, d)) * 3
    W = RNG.standard_normal((d, Fh))
    p = ref.phi(x, W)
    assert p.shape == (50, 2 * Fh)
    assert (p > 0).all()
    np.testing.assert_allclose(p[:, :Fh].sum(1), 1.0, atol=1e-13)
    np.testing.assert_allclose(p[:, Fh:].sum(1), 1.0, atol=1e-13)


def test_phi_zero_weight_is_uniform():
    x = RNG.standard_normal((7, 16))
    p = ref.phi(x, np.zeros((16, 8)))
    np.testing.assert_allclose(p, 1.0 / 8, atol=1e-15)


def test_phi_negative_half_mirrors_positive_half():
    # softmax(-u) is softmax(u) evaluated at -x, because xW is linear in x.
    x = RNG.standard_normal((9, 12))
    W = RNG.standard_normal((12, 6))
    np.testing.assert_allclose(ref.phi(x, W)[:, 6:], ref.phi(-x, W)[:, :6], atol=1e-15)


def test_featuremap_head_to_weight_map():
    T, H, Hw, d, Fh = 5, 8, 2, 6, 4
    x = RNG.standard_normal((T, H, d))
    W = RNG.standard_normal((Hw, d, Fh))
    out = ref.featuremap(x, W)
    for h in range(H):
        np.testing.assert_array_equal(out[:, h], ref.phi(x[:, h], W[h * Hw // H]))
    # heads 0..3 use W[0]; heads 4..7 use W[1]
    assert not np.allclose(out[:, 3], ref.phi(x[:, 3], W[1]))


# ---------------------------------------------------------------- merge (§3.1)

def test_merge_hand_example(golden):
    g = golden("hand_merge.txt")
    q, k, v = g["q"][0][None], g["k"][0][None], g["v"][0][None]
    W = np.eye(2)
    S, Z = ref.state_from_tokens(g["k_p"][0][None], g["v_p"][0][None], W)
    np.testing.assert_allclose(S.reshape(-1), g["S"][0], atol=1e-15)
    np.testing.assert_allclose(Z, g["Z"][0], atol=1e-15)
    np.testing.assert_allclose(ref.block_hybrid_head(q, k, v, S, Z, W, 1.0)[0],
                               g["out_w1"][0], rtol=1e-14)
    np.testing.assert_allclose(ref.block_hybrid_head(q, k, v, S, Z, W, float(ref.gate(0.0)))[0],
                               g["out_w_half"][0], rtol=1e-14)
    np.testing.assert_allclose(
        ref.block_hybrid_head(q, k, v, np.zeros_like(S), np.zeros_like(Z), W, 1.0)[0],
        g["out_empty_prefix"][0], atol=1e-15)


@pytest.mark.parametrize("w", [1.0, 0.3])
def test_recurrent_read_equals_bruteforce_prefix_sum(w):
    d, Fh, b, P = 8, 6, 5, 13
    W = RNG.standard_normal((d, Fh)) / math.sqrt(d)
    q, k, v = (RNG.standard_normal((b, d)) for _ in range(3))
    Kp, Vp = RNG.standard_normal((P, d)), RNG.standard_normal((P, d))
    S, Z = ref.state_from_tokens(Kp, Vp, W)
    a = ref.block_hybrid_head(q, k, v, S, Z, W, w)
    bf = ref.block_hybrid_head_bruteforce(q, k, v, Kp, Vp, W, w)
    np.testing.assert_allclose(a, bf, rtol=1e-12, atol=1e-13)


def test_empty_prefix_is_exact_block_softmax():
    d, Fh, b = 16, 8, 7
    W = RNG.standard_normal((d, Fh))
    q, k, v = (RNG.standard_normal((b, d)) for _ in range(3))
    S, Z = np.zeros((2 * Fh, d)), np.zeros(2 * Fh)
    want = _sdpa64(q, k, v)
    for w in (1.0, 0.25):  # with no prefix the gate cancels
        np.testing.assert_allclose(ref.block_hybrid_head(q, k, v, S, Z, W, w), want,
                                   rtol=1e-12, atol=1e-13)


def test_zero_weight_closed_form():
    # W = 0 makes phi uniform (1/Fh), so phi(q).phi(k) = 2/Fh for every pair and
    # out = (w A softmax_out + (2/Fh) sum_t v_t) / (w A + 2P/Fh), A = sum_j exp(q.k_j/sqrt d).
    d, Fh, b, P, w = 12, 5, 6, 9, 0.7
    W = np.zeros((d, Fh))
    q, k, v = (RNG.standard_normal((b, d)) for _ in range(3))
    Kp, Vp = RNG.standard_normal((P, d)), RNG.standard_normal((P, d))
    S, Z = ref.state_from_tokens(Kp, Vp, W)
    A = torch.logsumexp(torch.from_numpy(q @ k.T / math.sqrt(d)), dim=1).exp().numpy()
    want = (w * A[:, None] * _sdpa64(q, k, v) + (2.0 / Fh) * Vp.sum(0)) / (w * A + 2.0 * P / Fh)[:, None]
    np.testing.assert_allclose(ref.block_hybrid_head(q, k, v, S, Z, W, w), want, rtol=1e-12)


def test_zero_gate_is_plain_linear_attention():
    # w -> 0 leaves eq. (1): a kernel smoother with kernel phi(q).phi(k_t) over the prefix.
    d, Fh, b, P = 8, 4, 3, 11
    W = RNG.standard_normal((d, Fh))
    q, k, v = (RNG.standard_normal((b, d)) for _ in range(3))
    Kp, Vp = RNG.standard_normal((P, d)), RNG.standard_normal((P, d))
    S, Z = ref.state_from_tokens(Kp, Vp, W)
    kern = ref.phi(q, W) @ ref.phi(Kp, W).T
    want = (kern @ Vp) / kern.sum(1, keepdims=True)
    got = ref.block_hybrid_head(q, k, v, S, Z, W, float(ref.gate(-np.inf)))
    np.testing.assert_allclose(got, want, rtol=1e-12)


def test_zero_denominator_gives_zero():
    d, Fh = 4, 2
    q = RNG.standard_normal((2, d))
    out = ref.block_hybrid_head(q, q, q, np.zeros((4, d)), np.zeros(4), np.zeros((d, Fh)), 0.0)
    assert np.all(out == 0)


def test_block_is_bidirectional_permutation_equivariant():
    d, Fh, b, P = 8, 6, 9, 5
    W = RNG.standard_normal((d, Fh))
    q, k, v = (RNG.standard_normal((b, d)) for _ in range(3))
    S, Z = ref.state_from_tokens(RNG.standard_normal((P, d)), RNG.standard_normal((P, d)), W)
    perm = RNG.permutation(b)
    a = ref.block_hybrid_head(q, k, v, S, Z, W)
    bp = ref.block_hybrid_head(q[perm], k[perm], v[perm], S, Z, W)
    np.testing.assert_allclose(bp, a[perm], rtol=1e-13)
    # and the first query sees the last key (no causal mask inside the block)
    k2 = k.copy()
    k2[-1] += 1.0
    assert not np.allclose(ref.block_hybrid_head(q, k2, v, S, Z, W)[0], a[0])


def test_block_keys_do_not_enter_the_linear_branch():
    # Committing the active block first and then reading would count it twice; the read
    # must use the states of earlier blocks only.
    d, Fh, b = 6, 4, 4
    W = RNG.standard_normal((d, Fh))
    q, k, v = (RNG.standard_normal((b, d)) for _ in range(3))
    zeroS, zeroZ = np.zeros((2 * Fh, d)), np.zeros(2 * Fh)
    np.testing.assert_allclose(ref.block_hybrid_head(q, k, v, zeroS, zeroZ, W), _sdpa64(q, k, v),
                               rtol=1e-12)


# ---------------------------------------------------------------- commit (§3.1)

def test_incremental_commits_equal_one_shot():
    d, Fh = 10, 7
    W = RNG.standard_normal((d, Fh))
    lens = [4, 0, 7, 1, 5]
    Ks = [RNG.standard_normal((n, d)) for n in lens]
    Vs = [RNG.standard_normal((n, d)) for n in lens]
    S, Z = np.zeros((2 * Fh, d)), np.zeros(2 * Fh)
    for Kb, Vb in zip(Ks, Vs):
        S, Z = ref.commit(S, Z, Kb, Vb, W)
    S1, Z1 = ref.state_from_tokens(np.concatenate(Ks), np.concatenate(Vs), W)
    np.testing.assert_allclose(S, S1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(Z, Z1, rtol=1e-12)
    # Z counts tokens: each half of phi sums to 1, so sum(Z) = 2 * (number of tokens)
    np.testing.assert_allclose(Z.sum(), 2 * sum(lens), rtol=1e-13)


def test_commit_of_empty_block_is_identity():
    d, Fh = 4, 3
    S, Z = RNG.standard_normal((6, d)), RNG.random(6)
    S2, Z2 = ref.commit(S, Z, np.zeros((0, d)), np.zeros((0, d)), RNG.standard_normal((d, Fh)))
    np.testing.assert_array_equal(S2, S)
    np.testing.assert_array_equal(Z2, Z)


def test_state_outer_product_orientation():
    # one token: S = phi(k) v^T, so S[f, :] is v scaled by phi(k)[f]
    d, Fh = 3, 2
    W = RNG.standard_normal((d, Fh))
    k, v = RNG.standard_normal(d), np.array([1.0, -2.0, 5.0])
    S, Z = ref.state_from_tokens(k[None], v[None], W)
    p = ref.phi(k, W)
    for f in range(2 * Fh):
        np.testing.assert_allclose(S[f], p[f] * v, rtol=1e-15)
    np.testing.assert_allclose(Z, p, rtol=1e-15)


# ---------------------------------------------------------------- batched layout

def test_batched_hybrid_matches_per_head_with_gqa_slots_and_gate():
    c = inputs.decode_case(R=3, Hq=4, Hkv=2, d=8, F=12, block_lens=[3, 0, 5], prefix_lens=[2, 4, 0],
                           seed=7, dtype="f32", with_alpha=True)
    slots = np.array([2, 0, 1])
    S, Z = inputs.random_states(3, 2, 12, 8, 6, seed=3)
    O = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S, Z, c.W, c.alpha, slots)
    for r in range(3):
        lo, hi = c.cu_blk[r], c.cu_blk[r + 1]
        for h in range(4):
            g = h // 2
            want = ref.block_hybrid_head(c.Q[lo:hi, h], c.K[lo:hi, g], c.V[lo:hi, g],
                                         S[slots[r], g], Z[slots[r], g], c.W[g],
                                         1 / (1 + math.exp(-c.alpha[h])))
            np.testing.assert_array_equal(O[lo:hi, h], want)
    assert O.shape == (8, 4, 8)


def test_batched_commit_matches_one_shot_with_slots():
    c = inputs.decode_case(R=2, Hq=2, Hkv=2, d=6, F=8, block_lens=[4, 2], prefix_lens=0,
                           seed=9, dtype="f32")
    S0, Z0 = inputs.random_states(3, 2, 8, 6, 10, seed=4)
    slots = np.array([2, 0])
    S, Z = ref.commit_block(c.cu_blk, c.K, c.V, c.W, S0, Z0, slots)
    np.testing.assert_array_equal(S[1], S0[1])  # slot 1 untouched
    for r, s in enumerate(slots):
        lo, hi = c.cu_blk[r], c.cu_blk[r + 1]
        for g in range(2):
            dS, dZ = ref.state_from_tokens(c.K[lo:hi, g], c.V[lo:hi, g], c.W[g])
            np.testing.assert_allclose(S[s, g], S0[s, g] + dS, rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(Z[s, g], Z0[s, g] + dZ, rtol=1e-13)


def test_tiny_case_recurrent_equals_bruteforce():
    c = inputs.tiny_case(seed=0)
    S, Z = ref.state_from_tokens(c.K_pre[:, 0], c.V_pre[:, 0], c.W[0])
    got = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S[None, None], Z[None, None], c.W)
    bf = ref.block_hybrid_head_bruteforce(c.Q[:, 0], c.K[:, 0], c.V[:, 0], c.K_pre[:, 0],
                                          c.V_pre[:, 0], c.W[0])
    np.testing.assert_allclose(got[:, 0], bf, rtol=1e-12)


# ---------------------------------------------------------------- teacher

def test_full_prefix_attention_equals_sdpa():
    R, Hq, Hkv, d, L = 2, 4, 2, 16, 20
    kv_len = np.array([20, 9])
    cu = np.array([0, 3, 5])
    Q = RNG.standard_normal((5, Hq, d))
    Kc, Vc = RNG.standard_normal((R, Hkv, L, d)), RNG.standard_normal((R, Hkv, L, d))
    O = ref.full_prefix_attn(cu, kv_len, Q, Kc, Vc)
    for r in range(R):
        for h in range(Hq):
            g = h // 2
            want = _sdpa64(Q[cu[r]:cu[r + 1], h], Kc[r, g, :kv_len[r]], Vc[r, g, :kv_len[r]])
            np.testing.assert_allclose(O[cu[r]:cu[r + 1], h], want, rtol=1e-12, atol=1e-13)


def test_hybrid_with_linear_kernel_equal_to_exp_is_teacher():
    # If phi(q).phi(k) were exactly exp(q.k/sqrt d), the hybrid would be the teacher.  Pin the
    # merge algebra by substituting the exact kernel into the brute-force linear branch.
    d, b, P = 8, 4, 6
    q, k, v = (RNG.standard_normal((b, d)) for _ in range(3))
    Kp, Vp = RNG.standard_normal((P, d)), RNG.standard_normal((P, d))
    a_blk = np.exp(q @ k.T / math.sqrt(d))
    a_pre = np.exp(q @ Kp.T / math.sqrt(d))
    num = a_blk @ v + a_pre @ Vp
    den = a_blk.sum(1) + a_pre.sum(1)
    want = _sdpa64(q, np.concatenate([Kp, k]), np.concatenate([Vp, v]))
    np.testing.assert_allclose(num / den[:, None], want, rtol=1e-12)
    # and the oracle's teacher agrees with the same library routine
    O = ref.full_prefix_attn([0, b], [P + b], q[:, None], np.concatenate([Kp, k])[None, None],
                             np.concatenate([Vp, v])[None, None])
    np.testing.assert_allclose(O[:, 0], want, rtol=1e-12)


# ---------------------------------------------------------------- generator

def test_bf16_round_is_rne():
    x = np.array([1.0, 1.00390625, 1.005859375, 1.0078125, -3.14159265, 0.0], np.float32)
    y = inputs.bf16_round(x)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: ties go to the even mantissa (1.0)
    assert y[1] == 1.0
    assert y[2] == np.float32(1.0078125)
    assert y[3] == np.float32(1.0078125)
    assert y[5] == 0.0
    t = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(y, t)


def test_generator_is_seeded_and_stable():
    a = inputs.decode_case(2, 4, 2, 8, 8, 3, 5, seed=11)
    b = inputs.decode_case(2, 4, 2, 8, 8, 3, 5, seed=11)
    np.testing.assert_array_equal(a.Q, b.Q)
    np.testing.assert_array_equal(a.W, b.W)
    assert np.all(inputs.bf16_round(a.Q) == a.Q)
