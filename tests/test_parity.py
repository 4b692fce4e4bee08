"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on identical
seeded inputs.  Tolerances are stated in tests/gpu_util.py."""
import numpy as np
import pytest
import torch

from linear_attention_diffusion_hedgehog_b200 import bha, inputs
from oracle import bha_ref as ref
from tests.gpu_util import (TOL_BF16, TOL_F32, TOL_STATE_LONG, act_dtype, assert_close,
                            build_states_on_gpu, dev, host64)

pytestmark = pytest.mark.gpu


def oracle_states(case, reqs=None):
    reqs = range(case.R) if reqs is None else reqs
    S = np.zeros((case.R, case.Hkv, case.F, case.d))
    Z = np.zeros((case.R, case.Hkv, case.F))
    for r in reqs:
        lo, hi = case.cu_pre[r], case.cu_pre[r + 1]
        for g in range(case.Hkv):
            S[r, g], Z[r, g] = ref.state_from_tokens(case.K_pre[lo:hi, g], case.V_pre[lo:hi, g],
                                                     case.W[g])
    return S, Z


def run_hybrid(case, S, Z, alpha=None, state_slot=None, dtype=None):
    dtype = dtype or act_dtype(case)
    cu = torch.tensor(case.cu_blk, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O = bha.hybrid_attn(cu, dev(case.Q, dtype), dev(case.K, dtype), dev(case.V, dtype), S, Z,
                        dev(case.W, dtype), max_block=int(max(case.block_lens.max(), 1)),
                        alpha=None if alpha is None else dev(alpha, torch.float32),
                        state_slot=state_slot, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return O


def rows_of(case, reqs):
    return np.concatenate([np.arange(case.cu_blk[r], case.cu_blk[r + 1]) for r in reqs])


# ------------------------------------------------------------------- tiny fp32 case

@pytest.mark.parametrize("with_alpha", [False, True])
def test_tiny_fp32_decode_step_and_commit(with_alpha):
    c = inputs.tiny_case(seed=0, with_alpha=with_alpha)
    S, Z = build_states_on_gpu(c, block=8)
    So, Zo = oracle_states(c)
    assert_close(host64(S), So, TOL_F32, "S after 3 commits")
    assert_close(host64(Z), Zo, TOL_F32, "Z after 3 commits")
    O = run_hybrid(c, S, Z, alpha=c.alpha)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, So, Zo, c.W, c.alpha)
    assert_close(host64(O), want, TOL_F32, "O")


# ------------------------------------------------------------------- feature map

@pytest.mark.parametrize("dt,out_dt", [("bf16", torch.float32), ("bf16", torch.bfloat16),
                                       ("f32", torch.float32)])
def test_featuremap(dt, out_dt):
    c = inputs.decode_case(R=3, Hq=8, Hkv=2, d=128, F=256, block_lens=[32, 7, 1], prefix_lens=0,
                           seed=21, dtype=dt)
    x = dev(c.Q, act_dtype(c))
    phi = bha.featuremap(x, dev(c.W, act_dtype(c)), out_dtype=out_dt)
    torch.cuda.synchronize()
    want = ref.featuremap(c.Q, c.W)
    got = host64(phi)
    if out_dt == torch.float32 and dt == "f32":
        assert_close(got, want, TOL_F32, "phi")
    elif out_dt == torch.float32:
        assert_close(got, want, dict(rel_l2=1e-5, max_abs=1e-6), "phi")
    else:  # bf16 output: one rounding of values in (0, 1)
        assert_close(got, want, dict(rel_l2=5e-3, max_abs=4e-3), "phi")
    # each half of phi sums to 1
    np.testing.assert_allclose(got[..., :128].sum(-1), 1.0, atol=2e-2 if out_dt == torch.bfloat16 else 1e-5)
    # the checked entry point: the same output, and a clean error word
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    phi2 = bha.featuremap(x, dev(c.W, act_dtype(c)), out_dtype=out_dt, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(phi2, phi)


def test_featuremap_odd_dims_and_head_map():
    c = inputs.decode_case(R=2, Hq=6, Hkv=3, d=40, F=70, block_lens=[5, 9], prefix_lens=0, seed=5,
                           dtype="f32")
    phi = bha.featuremap(dev(c.Q, torch.float32), dev(c.W, torch.float32))
    torch.cuda.synchronize()
    assert_close(host64(phi), ref.featuremap(c.Q, c.W), TOL_F32, "phi")


def _check_phi(got, want, out_dt):
    if out_dt == torch.float32:
        assert_close(got, want, dict(rel_l2=1e-5, max_abs=1e-6), "phi")
    else:  # bf16 output: one rounding of values in (0, 1)
        assert_close(got, want, dict(rel_l2=5e-3, max_abs=4e-3), "phi")


@pytest.mark.parametrize("H,Hkv,T", [(4, 4, 300), (16, 1, 77), (128, 1, 5), (64, 2, 33)])
def test_featuremap_tensor_core_head_groupings(H, Hkv, T):
    """G = H / Hkv heads per weight matrix from 1 to 128, so a warp's 32 output rows are 32
    tokens of one head, several heads of several tokens, or a slice of one token's heads;
    token counts that leave a ragged last tile (128 / G tokens per tile)."""
    rng = np.random.default_rng(1000 * H + T)
    x = inputs.bf16_round(rng.standard_normal((T, H, 128)).astype(np.float32))
    W = inputs.bf16_round((rng.standard_normal((Hkv, 128, 128)) / np.sqrt(128)).astype(np.float32))
    dims = bha.make_dims(0, H, Hkv, 128, 256, 1, T, 0, torch.bfloat16)
    assert bha.kernel_variant(dims, 0) == 1
    want = ref.featuremap(x, W)
    for out_dt in (torch.float32, torch.bfloat16):
        phi = bha.featuremap(dev(x, torch.bfloat16), dev(W, torch.bfloat16), out_dtype=out_dt)
        torch.cuda.synchronize()
        _check_phi(host64(phi), want, out_dt)


def test_featuremap_output_16_byte_aligned_matches_32_byte_aligned():
    """phi rows are stored as whole 32-byte sectors when the output is 32-byte aligned, and
    through staged bulk tensor stores when it is only 16-byte aligned (the alignment the API
    asks for); both give the same bits, fp32 and bf16 output, with a ragged last tile."""
    rng = np.random.default_rng(77)
    T, H, Hkv = 301, 16, 4
    x = dev(inputs.bf16_round(rng.standard_normal((T, H, 128)).astype(np.float32)), torch.bfloat16)
    W = dev(inputs.bf16_round((rng.standard_normal((Hkv, 128, 128)) / np.sqrt(128)).astype(np.float32)),
            torch.bfloat16)
    for out_dt, shift in ((torch.float32, 4), (torch.bfloat16, 8)):  # 16 bytes of the element type
        outs = []
        for sh in (0, shift):
            buf = torch.full((T * H * 256 + shift,), float("nan"), dtype=out_dt, device="cuda")
            phi = buf[sh:sh + T * H * 256].view(T, H, 256)
            assert (phi.data_ptr() % 32 == 0) == (sh == 0)
            bha.featuremap(x, W, out_dtype=out_dt, out=phi)
            torch.cuda.synchronize()
            outs.append(phi.clone())
        assert torch.equal(outs[0], outs[1]), f"{out_dt}: output depends on its alignment"


def test_featuremap_group_size_not_a_power_of_two_takes_the_generic_kernel():
    rng = np.random.default_rng(3)
    x = inputs.bf16_round(rng.standard_normal((20, 12, 128)).astype(np.float32))
    W = inputs.bf16_round((rng.standard_normal((4, 128, 128)) / np.sqrt(128)).astype(np.float32))
    assert bha.kernel_variant(bha.make_dims(0, 12, 4, 128, 256, 1, 20, 0, torch.bfloat16), 0) == 0
    phi = bha.featuremap(dev(x, torch.bfloat16), dev(W, torch.bfloat16))
    torch.cuda.synchronize()
    _check_phi(host64(phi), ref.featuremap(x, W), torch.float32)


def test_featuremap_serving_size_sampled_rows():
    """The bench's workload: x [4096, 16, 128] bf16, 4 weight matrices, fp32 phi; 64 sampled
    (token, head) rows against the oracle, and every row's halves sum to 1."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    x = torch.randn((4096, 16, 128), generator=gen, device="cuda").to(torch.bfloat16)
    W = (torch.randn((4, 128, 128), generator=gen, device="cuda") / 128 ** 0.5).to(torch.bfloat16)
    phi = bha.featuremap(x, W)
    torch.cuda.synchronize()
    rng = np.random.default_rng(12)
    toks = rng.integers(0, 4096, 64)
    heads = rng.integers(0, 16, 64)
    xs = host64(x[toks, heads])
    Wh = host64(W)
    got = host64(phi[toks, heads])
    want = np.stack([ref.phi(xs[i:i + 1], Wh[heads[i] // 4])[0] for i in range(64)])
    _check_phi(got, want, torch.float32)
    sums = phi.double().view(4096, 16, 2, 128).sum(-1)
    assert torch.allclose(sums, torch.ones_like(sums), atol=1e-5)


# ------------------------------------------------------------------- decode step, bf16

def test_decode_step_one_layer_128_requests():
    """128 requests, 16 query / 4 KV heads, d 128, F 256, 32-token blocks, 1024-token prefixes
    folded into S/Z by 32 commits; the states and every output row of every request checked,
    each request on its own as well as in aggregate."""
    c = inputs.decode_case(R=128, Hq=16, Hkv=4, d=128, F=256, block_lens=32, prefix_lens=1024,
                           seed=2, dtype="bf16")
    S, Z = build_states_on_gpu(c, block=32)
    O = run_hybrid(c, S, Z)
    So, Zo = oracle_states(c)
    Sh, Zh, Oh = host64(S), host64(Z), host64(O)
    assert_close(Sh, So, TOL_BF16, "S")
    assert_close(Zh, Zo, TOL_BF16, "Z")
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, So, Zo, c.W)
    assert_close(Oh, want, TOL_BF16, "O")
    for r in range(c.R):
        rows = rows_of(c, [r])
        assert_close(Oh[rows], want[rows], TOL_BF16, f"O[{r}]")


def test_decode_step_and_commit_1024_requests_many_units_per_cta():
    """1024 requests (4096 (request, KV head) units: about 28 per CTA for the decode step, and
    1024 four-request units for the commits that build the 64-token prefixes), so each CTA
    walks many units with its buffers and W_g reused; 8 sampled requests checked in full."""
    c = inputs.decode_case(R=1024, Hq=16, Hkv=4, d=128, F=256, block_lens=32, prefix_lens=64,
                           seed=31, dtype="bf16")
    S, Z = build_states_on_gpu(c, block=32)
    O = run_hybrid(c, S, Z)
    reqs = np.random.default_rng(5).choice(1024, 8, replace=False)
    So, Zo = oracle_states(c, reqs)
    Oh = host64(O)
    for r in reqs:
        assert_close(host64(S[r]), So[r], TOL_BF16, f"S[{r}]")
        assert_close(host64(Z[r]), Zo[r], TOL_BF16, f"Z[{r}]")
        lo, hi = c.cu_blk[r], c.cu_blk[r + 1]
        want = ref.hybrid_attn([0, hi - lo], c.Q[lo:hi], c.K[lo:hi], c.V[lo:hi], So[r:r + 1],
                               Zo[r:r + 1], c.W)
        assert_close(Oh[lo:hi], want, TOL_BF16, f"O[{r}]")


def test_decode_step_three_kv_heads_grid_stays_on_one_weight():
    """Hkv = 3 (12 query heads), 50 requests: 150 units on a grid sized to a multiple of 3, so
    every CTA keeps one W_g; ragged blocks and prefixes; every row checked."""
    lens = np.random.default_rng(2).integers(1, 33, 50)
    c = inputs.decode_case(R=50, Hq=12, Hkv=3, d=128, F=256, block_lens=lens, prefix_lens=64,
                           seed=32, dtype="bf16")
    d = bha.make_dims(50, 12, 3, 128, 256, 32, int(c.cu_blk[-1]), 50, torch.bfloat16)
    assert bha.kernel_variant(d, 1) == 1
    S, Z = build_states_on_gpu(c, block=32)
    O = run_hybrid(c, S, Z)
    So, Zo = oracle_states(c)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, So, Zo, c.W)
    assert_close(host64(O), want, TOL_BF16, "O")


def test_decode_step_ragged_slots_gate_isolated_states():
    """Ragged blocks (0, 1, 31, 32 tokens), a permuted slot map, the sigmoid gate, and
    directly drawn states, so the cross-block read is checked on its own."""
    lens = [32, 0, 1, 31, 17, 32, 8, 2]
    c = inputs.decode_case(R=8, Hq=16, Hkv=4, d=128, F=256, block_lens=lens, prefix_lens=0,
                           seed=33, dtype="bf16", with_alpha=True)
    S_np, Z_np = inputs.random_states(10, 4, 256, 128, prefix_len=700, seed=8)
    slots = np.array([3, 9, 0, 5, 1, 2, 8, 6], dtype=np.int32)
    S, Z = dev(S_np, torch.float32), dev(Z_np, torch.float32)
    O = run_hybrid(c, S, Z, alpha=c.alpha, state_slot=torch.tensor(slots, device="cuda"))
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S_np, Z_np, c.W, c.alpha, slots)
    assert_close(host64(O), want, TOL_BF16, "O")


def test_decode_step_large_queries_mixed_shift_paths():
    """Queries of some 8-token groups scaled by 4, and of one request by 8 (exact in bf16), so
    that in those rows max u - min u may reach ~50-100 log2 units: the feature-map warps that
    hold them take the full max/min pass, the other warps of the same units keep the shift
    from their first 32 features; ragged blocks, the gate and drawn states; every row checked."""
    c = inputs.decode_case(R=6, Hq=16, Hkv=4, d=128, F=256, block_lens=[32, 32, 20, 9, 32, 32],
                           prefix_lens=0, seed=41, dtype="bf16", with_alpha=True)
    Q = c.Q.copy()
    lo = c.cu_blk
    Q[lo[0] + 8:lo[0] + 16] *= 4
    Q[lo[2]:lo[3]] *= 8
    Q[lo[4]:lo[4] + 8] *= 4
    Q[lo[5] + 24:lo[5] + 32] *= 4
    c.Q = Q
    S_np, Z_np = inputs.random_states(6, 4, 256, 128, prefix_len=500, seed=9)
    S, Z = dev(S_np, torch.float32), dev(Z_np, torch.float32)
    O = run_hybrid(c, S, Z, alpha=c.alpha)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S_np, Z_np, c.W, c.alpha)
    assert np.isfinite(host64(O)).all()
    assert_close(host64(O), want, TOL_BF16, "O")


def test_empty_prefix_is_block_softmax():
    c = inputs.decode_case(R=4, Hq=16, Hkv=4, d=128, F=256, block_lens=[32, 5, 32, 1],
                           prefix_lens=0, seed=4, dtype="bf16", with_alpha=True)
    S = torch.zeros((4, 4, 256, 128), device="cuda")
    Z = torch.zeros((4, 4, 256), device="cuda")
    O = run_hybrid(c, S, Z, alpha=c.alpha)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, np.zeros((4, 4, 256, 128)),
                           np.zeros((4, 4, 256)), c.W, c.alpha)
    assert_close(host64(O), want, TOL_BF16, "O")


def test_permuting_block_tokens_permutes_outputs():
    c = inputs.decode_case(R=2, Hq=16, Hkv=4, d=128, F=256, block_lens=32, prefix_lens=0,
                           seed=12, dtype="bf16")
    S_np, Z_np = inputs.random_states(2, 4, 256, 128, prefix_len=300, seed=1)
    S, Z = dev(S_np, torch.float32), dev(Z_np, torch.float32)
    O = host64(run_hybrid(c, S, Z))
    perm = np.concatenate([np.random.default_rng(3).permutation(32), 32 + np.arange(32)])
    c.Q, c.K, c.V = c.Q[perm], c.K[perm], c.V[perm]
    Op = host64(run_hybrid(c, S, Z))
    assert_close(Op, O[perm], dict(max_abs=2e-2, rel_l2=1e-3), "permuted")


# ------------------------------------------------------------------- commit, bf16

def test_commit_one_block_onto_31_and_32_sequential():
    """Fold a 32-token block into states holding 31 earlier blocks (128 requests x 4 KV
    heads) and compare with a one-shot build over all 32 blocks; every request checked."""
    c = inputs.decode_case(R=128, Hq=4, Hkv=4, d=128, F=256, block_lens=32, prefix_lens=32 * 32,
                           seed=3, dtype="bf16")
    S, Z = build_states_on_gpu(c, block=32)   # 32 sequential commits from zero
    reqs = range(c.R)
    So, Zo = oracle_states(c, reqs)
    for r in reqs:
        assert_close(host64(S[r]), So[r], TOL_BF16, f"S[{r}] after 32 commits")
        assert_close(host64(Z[r]), Zo[r], TOL_BF16, f"Z[{r}] after 32 commits")
    # 31 blocks then the last one as a separate commit of the active block rows
    c31 = inputs.decode_case(R=128, Hq=4, Hkv=4, d=128, F=256, block_lens=32, prefix_lens=31 * 32,
                             seed=3, dtype="bf16")
    S31, Z31 = build_states_on_gpu(c31, block=32)
    cu = torch.tensor(c31.cu_blk, dtype=torch.int32, device="cuda")
    bha.commit_block(cu, dev(c31.K, torch.bfloat16), dev(c31.V, torch.bfloat16),
                     dev(c31.W, torch.bfloat16), S31, Z31, max_block=32)
    torch.cuda.synchronize()
    for r in reqs:
        lo, hi = c31.cu_pre[r], c31.cu_pre[r + 1]
        for g in range(4):
            Kall = np.concatenate([c31.K_pre[lo:hi, g], c31.K[32 * r:32 * r + 32, g]])
            Vall = np.concatenate([c31.V_pre[lo:hi, g], c31.V[32 * r:32 * r + 32, g]])
            So1, Zo1 = ref.state_from_tokens(Kall, Vall, c31.W[g])
            assert_close(host64(S31[r, g]), So1, TOL_BF16, f"S[{r},{g}] 31+1")
            assert_close(host64(Z31[r, g]), Zo1, TOL_BF16, f"Z[{r},{g}] 31+1")


def test_commit_ragged_with_slots_and_empty_blocks():
    lens = [0, 5, 32, 1, 17]
    c = inputs.decode_case(R=5, Hq=4, Hkv=4, d=128, F=256, block_lens=lens, prefix_lens=0, seed=6,
                           dtype="bf16")
    S_np, Z_np = inputs.random_states(7, 4, 256, 128, prefix_len=64, seed=2)
    slots = np.array([6, 0, 3, 2, 5], dtype=np.int32)
    S, Z = dev(S_np, torch.float32), dev(Z_np, torch.float32)
    cu = torch.tensor(c.cu_blk, dtype=torch.int32, device="cuda")
    bha.commit_block(cu, dev(c.K, torch.bfloat16), dev(c.V, torch.bfloat16),
                     dev(c.W, torch.bfloat16), S, Z, max_block=32,
                     state_slot=torch.tensor(slots, device="cuda"))
    torch.cuda.synchronize()
    So, Zo = ref.commit_block(c.cu_blk, c.K, c.V, c.W, S_np, Z_np, slots)
    assert_close(host64(S), So, TOL_BF16, "S")
    assert_close(host64(Z), Zo, TOL_BF16, "Z")
    np.testing.assert_array_equal(host64(S[6]), S_np[6])   # b = 0: untouched
    np.testing.assert_array_equal(host64(S[1]), S_np[1])   # no request: untouched


@pytest.mark.parametrize("bmax,lens", [
    (64, [64, 0, 1, 63, 40, 64, 17]),          # two requests per tile
    (48, [48, 3, 0, 47, 48]),                  # rounded up to 64-row request slots
    (128, [128, 0, 1, 127, 100, 128, 65]),     # one request per tile
    (128, [100]),                              # one request, fewer tokens than the tile
])
def test_commit_large_blocks_tensor_core(bmax, lens):
    """Blocks of up to 64 or 128 tokens on the tensor-core commit (64- or 128-row request
    slots, so 2 or 1 requests per 128-row tile): ragged lengths including empty blocks, a
    permuted slot map and random initial states, against the oracle's commit."""
    R = len(lens)
    c = inputs.decode_case(R=R, Hq=4, Hkv=4, d=128, F=256, block_lens=lens, prefix_lens=0,
                           seed=60 + bmax + R, dtype="bf16")
    dims = bha.make_dims(R, 4, 4, 128, 256, bmax, int(c.cu_blk[-1]), R + 2, torch.bfloat16)
    assert bha.kernel_variant(dims, 2) == 1
    S_np, Z_np = inputs.random_states(R + 2, 4, 256, 128, prefix_len=256, seed=bmax)
    slots = np.random.default_rng(bmax + R).permutation(R + 2)[:R].astype(np.int32)
    S, Z = dev(S_np, torch.float32), dev(Z_np, torch.float32)
    cu = torch.tensor(c.cu_blk, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bha.commit_block(cu, dev(c.K, torch.bfloat16), dev(c.V, torch.bfloat16),
                     dev(c.W, torch.bfloat16), S, Z, max_block=bmax,
                     state_slot=torch.tensor(slots, device="cuda"), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    So, Zo = ref.commit_block(c.cu_blk, c.K, c.V, c.W, S_np, Z_np, slots)
    assert_close(host64(S), So, TOL_BF16, "S")
    assert_close(host64(Z), Zo, TOL_BF16, "Z")
    for sl in set(range(R + 2)) - {int(slots[r]) for r in range(R) if lens[r] > 0}:
        np.testing.assert_array_equal(host64(S[sl]), S_np[sl])   # no token committed there


def test_commit_128_token_blocks_128_requests_one_shot():
    """128 requests x 4 KV heads folding 1024-token prefixes into zero states in 8 commits of
    128-token blocks (the large-block commit at full width); every request against the
    oracle's one-shot build."""
    c = inputs.decode_case(R=128, Hq=4, Hkv=4, d=128, F=256, block_lens=32, prefix_lens=1024,
                           seed=61, dtype="bf16")
    dims = bha.make_dims(128, 4, 4, 128, 256, 128, 128 * 128, 128, torch.bfloat16)
    assert bha.kernel_variant(dims, 2) == 1
    S, Z = build_states_on_gpu(c, block=128)
    So, Zo = oracle_states(c)
    assert_close(host64(S), So, TOL_BF16, "S after 8 commits of 128 tokens")
    assert_close(host64(Z), Zo, TOL_BF16, "Z after 8 commits of 128 tokens")


# ------------------------------------------------------------------- generic dims

def test_generic_max_dims_fp32():
    """Largest dims the library accepts: d 256, F 512, a 128-token block (fp32)."""
    c = inputs.decode_case(R=2, Hq=2, Hkv=1, d=256, F=512, block_lens=[128, 3], prefix_lens=[128, 0],
                           seed=13, dtype="f32", with_alpha=True)
    S, Z = build_states_on_gpu(c, block=128)
    So, Zo = oracle_states(c)
    assert_close(host64(S), So, TOL_F32, "S")
    O = run_hybrid(c, S, Z, alpha=c.alpha)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, So, Zo, c.W, c.alpha)
    assert_close(host64(O), want, TOL_F32, "O")


def test_small_odd_dims_bf16():
    c = inputs.decode_case(R=3, Hq=6, Hkv=2, d=24, F=20, block_lens=[7, 1, 13], prefix_lens=[9, 0, 30],
                           seed=17, dtype="bf16")
    S, Z = build_states_on_gpu(c, block=16)
    So, Zo = oracle_states(c)
    O = run_hybrid(c, S, Z)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, So, Zo, c.W)
    assert_close(host64(O), want, TOL_BF16, "O")


# ------------------------------------------------------------------- device-side validation

def test_bad_cu_blk_sets_dev_err_and_skips():
    c = inputs.decode_case(R=2, Hq=4, Hkv=4, d=128, F=256, block_lens=[16, 16], prefix_lens=0,
                           seed=1, dtype="bf16")
    S = torch.zeros((2, 4, 256, 128), device="cuda")
    Z = torch.zeros((2, 4, 256), device="cuda")
    cu = torch.tensor([0, 20, 32], dtype=torch.int32, device="cuda")   # block 0 longer than 16
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O = torch.full((32, 4, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    bha.hybrid_attn(cu, dev(c.Q, torch.bfloat16), dev(c.K, torch.bfloat16),
                    dev(c.V, torch.bfloat16), S, Z, dev(c.W, torch.bfloat16), max_block=16,
                    out=O, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == bha.BHA_ERR_INVALID
    assert torch.all(O[:20] == 7.0)           # request 0 skipped
    assert not torch.all(O[20:] == 7.0)       # request 1 computed
    bad_slot = torch.tensor([0, 5], dtype=torch.int32, device="cuda")
    err.zero_()
    bha.commit_block(torch.tensor([0, 16, 32], dtype=torch.int32, device="cuda"),
                     dev(c.K, torch.bfloat16), dev(c.V, torch.bfloat16), dev(c.W, torch.bfloat16),
                     S, Z, max_block=16, state_slot=bad_slot, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == bha.BHA_ERR_INVALID


# ------------------------------------------------------------------- softmax teacher

@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_full_prefix_teacher(dt):
    R, Hq, Hkv, d, cap = 3, 8, 2, 128, 300
    kv_len = np.array([300, 33, 0], dtype=np.int32)
    lens = np.array([32, 1, 4])
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rng = np.random.default_rng(5)
    cast = inputs.bf16_round if dt == "bf16" else (lambda x: x.astype(np.float32))
    Q = cast(rng.standard_normal((cu[-1], Hq, d)).astype(np.float32))
    Kc = cast(rng.standard_normal((R, Hkv, cap, d)).astype(np.float32))
    Vc = cast(rng.standard_normal((R, Hkv, cap, d)).astype(np.float32))
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    O = bha.full_prefix_attn(torch.tensor(cu, device="cuda"), torch.tensor(kv_len, device="cuda"),
                             dev(Q, tdt), dev(Kc, tdt), dev(Vc, tdt), max_block=32)
    torch.cuda.synchronize()
    want = ref.full_prefix_attn(cu, kv_len, Q, Kc, Vc)
    assert_close(host64(O), want, TOL_BF16 if dt == "bf16" else TOL_F32, "O")


def test_tensor_core_path_is_taken_for_the_serving_shape():
    d = bha.make_dims(128, 16, 4, 128, 256, 32, 4096, 128, torch.bfloat16)
    assert bha.kernel_variant(d, 1) == 1
    d32 = bha.make_dims(128, 16, 4, 128, 256, 32, 4096, 128, torch.float32)
    assert bha.kernel_variant(d32, 1) == 0   # fp32 activations take the fp32 CUDA-core path
    assert bha.kernel_variant(d, 2) == 1     # block commit on tensor cores
    assert bha.kernel_variant(d32, 2) == 0
    assert bha.kernel_variant(d, 3) == 1     # softmax teacher on tensor cores
    assert bha.kernel_variant(d, 0) == 1     # feature map of the queries on tensor cores
    assert bha.kernel_variant(d32, 0) == 0


def test_linear_branch_dominant_states():
    """Large S and small Z make phi(q)^T S carry most of the output, so the feature map and
    the state contraction are checked directly (not hidden behind the softmax branch)."""
    c = inputs.decode_case(R=16, Hq=16, Hkv=4, d=128, F=256, block_lens=32, prefix_lens=0, seed=44,
                           dtype="bf16")
    rng = np.random.default_rng(9)
    S_np = (5.0 * rng.standard_normal((16, 4, 256, 128))).astype(np.float32)
    Z_np = rng.uniform(0.0, 0.5, size=(16, 4, 256)).astype(np.float32)
    O = run_hybrid(c, dev(S_np, torch.float32), dev(Z_np, torch.float32))
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S_np, Z_np, c.W)
    assert_close(host64(O), want, TOL_BF16, "O")


def test_zero_weight_closed_form_full_size():
    """W = 0 makes phi uniform (1/128), so with states built from P prefix tokens
    out_i = (sum_j a_ij v_j + (2/128) sum_t v_t) / (sum_j a_ij + 2P/128); checked at the serving
    size (128 requests, 1024-token prefixes) without the oracle."""
    c = inputs.decode_case(R=128, Hq=16, Hkv=4, d=128, F=256, block_lens=32, prefix_lens=1024,
                           seed=5, dtype="bf16")
    c.W = np.zeros_like(c.W)
    S, Z = build_states_on_gpu(c, block=32)
    O = host64(run_hybrid(c, S, Z))
    P, Fh, G = 1024, 128, 4
    Vsum = c.V_pre.astype(np.float64).reshape(128, P, 4, 128).sum(axis=1)          # [R, Hkv, d]
    q = c.Q.astype(np.float64).reshape(128, 32, 16, 128)
    k = c.K.astype(np.float64).reshape(128, 32, 4, 128)
    v = c.V.astype(np.float64).reshape(128, 32, 4, 128)
    kh = np.repeat(k, G, axis=2)
    vh = np.repeat(v, G, axis=2)
    s = np.einsum("rihd,rjhd->rhij", q, kh) / np.sqrt(128.0)
    a = np.exp(s)
    num = np.einsum("rhij,rjhd->rihd", a, vh) + (2.0 / Fh) * np.repeat(Vsum, G, axis=1)[:, None]
    den = a.sum(-1).transpose(0, 2, 1)[..., None] + 2.0 * P / Fh
    want = (num / den).reshape(4096, 16, 128)
    assert_close(O, want, TOL_BF16, "O (closed form)")


@pytest.mark.parametrize("poison", [False, True])
def test_full_prefix_teacher_split_kv(poison):
    """Long caches take the split-KV path (partials in the workspace, then a combine).  Cache
    rows past kv_len may hold anything: with poison=True they are NaN and must not matter."""
    R, Hq, Hkv, d, cap = 3, 8, 2, 128, 2000
    kv_len = np.array([2000, 130, 0], dtype=np.int32)
    lens = np.array([32, 17, 5])
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rng = np.random.default_rng(21)
    Q = inputs.bf16_round(rng.standard_normal((cu[-1], Hq, d)).astype(np.float32))
    Kc = inputs.bf16_round(rng.standard_normal((R, Hkv, cap, d)).astype(np.float32))
    Vc = inputs.bf16_round(rng.standard_normal((R, Hkv, cap, d)).astype(np.float32))
    tK, tV = dev(Kc, torch.bfloat16), dev(Vc, torch.bfloat16)
    if poison:
        for r in range(R):
            tK[r, :, kv_len[r]:] = float("nan")
            tV[r, :, kv_len[r]:] = float("nan")
    assert bha.full_prefix_workspace_bytes(R, Hq, Hkv, d, 32, int(cu[-1]), cap) > 0
    O = bha.full_prefix_attn(torch.tensor(cu, device="cuda"), torch.tensor(kv_len, device="cuda"),
                             dev(Q, torch.bfloat16), tK, tV, max_block=32)
    torch.cuda.synchronize()
    want = ref.full_prefix_attn(cu, kv_len, Q, Kc, Vc)
    assert_close(host64(O), want, TOL_BF16, "O")


def test_full_prefix_teacher_serving_size_sampled():
    """64 requests, 16 query / 4 KV heads, 2048-token prefixes plus the 32-token block; every
    output row of 6 sampled requests checked against the oracle."""
    R, Hq, Hkv, d, P = 64, 16, 4, 128, 2048
    L = P + 32
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    Kc = torch.randn((R, Hkv, L, d), generator=g, device="cuda").to(torch.bfloat16)
    Vc = torch.randn((R, Hkv, L, d), generator=g, device="cuda").to(torch.bfloat16)
    Q = torch.randn((R * 32, Hq, d), generator=g, device="cuda").to(torch.bfloat16)
    cu = torch.arange(0, (R + 1) * 32, 32, dtype=torch.int32, device="cuda")
    kv_len = torch.full((R,), L, dtype=torch.int32, device="cuda")
    O = host64(bha.full_prefix_attn(cu, kv_len, Q, Kc, Vc, max_block=32))
    reqs = np.random.default_rng(2).choice(R, 6, replace=False)
    Qh, Kh, Vh = host64(Q), host64(Kc), host64(Vc)
    for r in reqs:
        sl = slice(32 * r, 32 * r + 32)
        want = ref.full_prefix_attn([0, 32], [L], Qh[sl], Kh[r:r + 1], Vh[r:r + 1])
        assert_close(O[sl], want, TOL_BF16, f"O[{r}]")


# ------------------------------------------------------------------- watchdog

def test_bounded_wait_gives_up_and_reports_timeout():
    """The bounded wait every tensor-core kernel uses, on an mbarrier nothing arrives at:
    after its limit it reports BHA_ERR_TIMEOUT through dev_err and the context stays usable
    (a feature map right after runs and matches the oracle)."""
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bha.selftest_bounded_wait(2_000_000, err)  # about a millisecond of SM cycles
    torch.cuda.synchronize()
    assert int(err.item()) == -4, bha.status_string(int(err.item()))
    rng = np.random.default_rng(8)
    x = inputs.bf16_round(rng.standard_normal((40, 8, 128)).astype(np.float32))
    W = inputs.bf16_round((rng.standard_normal((2, 128, 128)) / np.sqrt(128)).astype(np.float32))
    phi = bha.featuremap(dev(x, torch.bfloat16), dev(W, torch.bfloat16))
    torch.cuda.synchronize()
    _check_phi(host64(phi), ref.featuremap(x, W), torch.float32)


# ------------------------------------------------------------------- extreme block logits

def _extreme_logit_case(sign, aligned_all, prefix, seed, dtype="bf16", d=128, F=256, Hq=16, Hkv=4,
                        level=100.0):
    """Block scores near sign * level (natural units).  aligned_all: every key of a request is
    close to one direction v0 and every query is sign * v0, so all of a row's scores are about
    sign * level; otherwise each query copies one key of its block (scaled by sign), so one
    score per row is about sign * level and the rest are O(level / 4).  prefix: states drawn
    from 700-token prefixes, or all zero."""
    lens = [32, 17, 1, 32]
    c = inputs.decode_case(R=4, Hq=Hq, Hkv=Hkv, d=d, F=F, block_lens=lens, prefix_lens=0,
                           seed=seed, dtype=dtype)
    rng = np.random.default_rng(seed + 100)
    rnd = inputs.bf16_round if dtype == "bf16" else (lambda a: a.astype(np.float32))
    G = Hq // Hkv
    K = np.empty_like(c.K)
    Q = np.empty_like(c.Q)
    amp = np.sqrt(level * np.sqrt(d) / d)  # |q| |k| / sqrt d ~ level for unit-variance directions
    for r in range(4):
        lo, hi = c.cu_blk[r], c.cu_blk[r + 1]
        for g in range(Hkv):
            if aligned_all:
                v0 = rng.standard_normal(d)
                K[lo:hi, g] = amp * (v0 + 0.05 * rng.standard_normal((hi - lo, d)))
                for h in range(G):
                    Q[lo:hi, g * G + h] = sign * amp * v0
            else:
                K[lo:hi, g] = amp * rng.standard_normal((hi - lo, d))
                for h in range(G):
                    Q[lo:hi, g * G + h] = sign * K[lo + rng.permutation(hi - lo), g]
    c.K, c.Q = rnd(K), rnd(Q)
    if prefix:
        S_np, Z_np = inputs.random_states(4, Hkv, F, d, prefix_len=700, seed=seed)
    else:
        S_np, Z_np = np.zeros((4, Hkv, F, d), np.float32), np.zeros((4, Hkv, F), np.float32)
    return c, S_np, Z_np


@pytest.mark.parametrize("sign,aligned_all,prefix,level", [
    (+1, False, False, 100), (+1, False, True, 100), (+1, True, False, 100), (+1, True, True, 100),
    (-1, True, False, 100), (-1, True, True, 100), (+1, True, True, 180), (+1, False, True, 180)])
def test_decode_step_extreme_block_logits(sign, aligned_all, prefix, level):
    """Scores of about +100 overflow exp in fp32 unless shifted, and a row whose scores are
    all about -100 underflows it: with an empty prefix the output must still be the block
    softmax, with a prefix the linear branch must dominate (softmax weight ~e^-100).  At +180
    the shift that keeps P finite flushes every linear-branch exponential to 0 and the output
    is the block softmax.  Checked against the float64 oracle on the tensor-core path."""
    c, S_np, Z_np = _extreme_logit_case(sign, aligned_all, prefix, seed=50 + 7 * aligned_all + 3 * prefix,
                                        level=float(level))
    d = bha.make_dims(4, 16, 4, 128, 256, 32, int(c.cu_blk[-1]), 4, torch.bfloat16)
    assert bha.kernel_variant(d, 1) == 1
    s = np.einsum("thd,tgd->th", c.Q.reshape(-1, 4, 4, 128).astype(np.float64)[:, :, 0, :],
                  c.K.astype(np.float64)) / np.sqrt(128.0)
    assert np.abs(s).max() > 0.8 * level  # the case really reaches the edge
    O = run_hybrid(c, dev(S_np, torch.float32), dev(Z_np, torch.float32))
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S_np.astype(np.float64), Z_np.astype(np.float64), c.W)
    assert_close(host64(O), want, TOL_BF16, "O")


@pytest.mark.parametrize("aligned_all,level", [(True, 180), (False, 100)])
def test_fused_step_and_commit_extreme_block_logits(aligned_all, level):
    """The fused step and commit at the same edges (states from 700-token prefixes, scores of
    about +level): the output against the oracle's step, the states (entries of up to ~40, the
    size of long-prefix states) against its commit."""
    c, S_np, Z_np = _extreme_logit_case(+1, aligned_all, True, seed=57 + 7 * aligned_all, level=float(level))
    d = bha.make_dims(4, 16, 4, 128, 256, 32, int(c.cu_blk[-1]), 4, torch.bfloat16)
    assert bha.kernel_variant(d, 4) == 1
    S, Z = dev(S_np, torch.float32), dev(Z_np, torch.float32)
    O = _run_fused(c, S, Z)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S_np.astype(np.float64), Z_np.astype(np.float64), c.W)
    assert_close(host64(O), want, TOL_BF16, "O")
    So, Zo = ref.commit_block(c.cu_blk, c.K, c.V, c.W, S_np.astype(np.float64), Z_np.astype(np.float64))
    assert_close(host64(S), So, TOL_STATE_LONG, "S")
    assert_close(host64(Z), Zo, TOL_STATE_LONG, "Z")


@pytest.mark.parametrize("sign,prefix", [(+1, False), (+1, True), (-1, False), (-1, True)])
def test_generic_kernel_extreme_block_logits(sign, prefix):
    """The same edges on the CUDA-core kernel (fp32 activations, all of a row's scores about
    sign * 100)."""
    c, S_np, Z_np = _extreme_logit_case(sign, True, prefix, seed=70 + 3 * prefix, dtype="f32",
                                        d=64, F=64, Hq=4, Hkv=2)
    O = run_hybrid(c, dev(S_np, torch.float32), dev(Z_np, torch.float32))
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S_np.astype(np.float64), Z_np.astype(np.float64), c.W)
    assert_close(host64(O), want, dict(rel_l2=1e-4, rel_max=1e-4), "O")


def test_decode_step_output_16_byte_aligned_matches_32_byte_aligned():
    """O rows are written as whole 32-byte sectors when O is 32-byte aligned, and as 16-byte
    pieces when it is only 16-byte aligned (the alignment the API asks for); the same step
    into both gives the same bits, for the decode step and for the fused step."""
    c = inputs.decode_case(R=6, Hq=16, Hkv=4, d=128, F=256, block_lens=[32, 5, 32, 1, 17, 32],
                           prefix_lens=64, seed=97, dtype="bf16", with_alpha=True)
    S, Z = build_states_on_gpu(c, block=32)
    T = int(c.cu_blk[-1])
    cu = torch.tensor(c.cu_blk, dtype=torch.int32, device="cuda")
    args = (cu, dev(c.Q, torch.bfloat16), dev(c.K, torch.bfloat16), dev(c.V, torch.bfloat16))
    W = dev(c.W, torch.bfloat16)
    alpha = dev(c.alpha, torch.float32)
    outs = []
    for shift in (0, 8):  # 8 bf16 = 16 bytes past a 256-byte-aligned allocation
        buf = torch.full((T * 16 * 128 + 16,), float("nan"), dtype=torch.bfloat16, device="cuda")
        O = buf[shift:shift + T * 16 * 128].view(T, 16, 128)
        assert (O.data_ptr() % 32 == 0) == (shift == 0)
        bha.hybrid_attn(*args, S, Z, W, max_block=32, alpha=alpha, out=O)
        S2, Z2 = S.clone(), Z.clone()
        buf2 = torch.full_like(buf, float("nan"))
        O2 = buf2[shift:shift + T * 16 * 128].view(T, 16, 128)
        bha.hybrid_attn_commit(*args, S2, Z2, W, max_block=32, alpha=alpha, out=O2)
        torch.cuda.synchronize()
        outs.append((O.clone(), O2.clone()))
    assert torch.equal(outs[0][0], outs[1][0]), "decode step: output depends on O's alignment"
    assert torch.equal(outs[0][1], outs[1][1]), "fused step: output depends on O's alignment"
    assert torch.equal(outs[0][0], outs[0][1])
    So, Zo = oracle_states(c)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, So, Zo, c.W, c.alpha)
    assert_close(host64(outs[1][0]), want, TOL_BF16, "O (16-byte aligned)")


@pytest.mark.parametrize("big_group", [1, 3])
def test_decode_step_shift_moves_when_a_later_feature_group_dominates(big_group):
    """The tensor-core step may shift e+ / e- by the max / min of each row's first 32 features
    and move the shift when a later group passes it.  Here the W columns of one later group
    are ten times larger, so u there spans about +-30 against +-3 in the first group, and every
    row's largest and smallest features sit in that group.  States from 64-token prefixes,
    ragged blocks; every row checked against the oracle."""
    lens = [32, 7, 32, 1]
    c = inputs.decode_case(R=4, Hq=16, Hkv=4, d=128, F=256, block_lens=lens, prefix_lens=64,
                           seed=95 + big_group, dtype="bf16")
    W = c.W.astype(np.float64).copy()
    W[:, :, 32 * big_group:32 * big_group + 32] *= 10.0
    c.W = inputs.bf16_round(W)
    S, Z = build_states_on_gpu(c, block=32)
    So, Zo = oracle_states(c)
    O = run_hybrid(c, S, Z)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, So, Zo, c.W)
    assert_close(host64(O), want, TOL_BF16, "O")


# ------------------------------------------------------------------- query heads per KV head

@pytest.mark.parametrize("Hq,Hkv", [(16, 16), (8, 4)])
def test_decode_step_one_and_two_query_heads_per_state(Hq, Hkv):
    """G = Hq / Hkv = 1 is the per-query-head layout (a W and a state per query head), G = 2 a
    smaller group; both take the tensor-core kernel, whose 128-row tile then holds 32 G live
    rows.  Ragged blocks, states committed from 64-token prefixes, the gate; every row checked."""
    lens = [32, 9, 1, 32, 20, 32]
    c = inputs.decode_case(R=6, Hq=Hq, Hkv=Hkv, d=128, F=256, block_lens=lens, prefix_lens=64,
                           seed=80 + Hq, dtype="bf16", with_alpha=True)
    d = bha.make_dims(6, Hq, Hkv, 128, 256, 32, int(c.cu_blk[-1]), 6, torch.bfloat16)
    assert bha.kernel_variant(d, 1) == 1
    S, Z = build_states_on_gpu(c, block=32)
    So, Zo = oracle_states(c)
    O = run_hybrid(c, S, Z, alpha=c.alpha)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, So, Zo, c.W, c.alpha)
    assert_close(host64(O), want, TOL_BF16, "O")


def test_decode_step_per_query_head_serving_size_sampled():
    """128 requests with a W and a state per query head (16 / 16 heads), 32-token blocks,
    states from 256-token prefixes committed through the library; 4 sampled requests."""
    c = inputs.decode_case(R=128, Hq=16, Hkv=16, d=128, F=256, block_lens=32, prefix_lens=256,
                           seed=91, dtype="bf16")
    S, Z = build_states_on_gpu(c, block=32)
    O = host64(run_hybrid(c, S, Z))
    reqs = np.random.default_rng(4).choice(128, 4, replace=False)
    So, Zo = oracle_states(c, reqs)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, So, Zo, c.W)
    rows = rows_of(c, reqs)
    assert_close(O[rows], want[rows], TOL_BF16, "O")


# ------------------------------------------------------------------- decode step fused with the commit

def _run_fused(c, S, Z, alpha=None, state_slot=None, dtype=None):
    dtype = dtype or act_dtype(c)
    cu = torch.tensor(c.cu_blk, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O = bha.hybrid_attn_commit(cu, dev(c.Q, dtype), dev(c.K, dtype), dev(c.V, dtype), S, Z,
                               dev(c.W, dtype), max_block=int(max(c.block_lens.max(), 1)),
                               alpha=None if alpha is None else dev(alpha, torch.float32),
                               state_slot=state_slot, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, bha.status_string(int(err.item()))
    return O


@pytest.mark.parametrize("Hq,Hkv", [(16, 4), (16, 8), (16, 16)])
def test_fused_step_and_commit_ragged_slots_gate(Hq, Hkv):
    """The last step of a block with its commit in one call: ragged blocks (0, 1, 31, 32
    tokens), a permuted slot map, the gate and drawn states.  The output reads the states as
    passed in; afterwards S and Z hold them plus each request's block, as the oracle's commit
    gives (slots no request names stay as they were)."""
    lens = [32, 0, 1, 31, 17, 32, 8, 2]
    c = inputs.decode_case(R=8, Hq=Hq, Hkv=Hkv, d=128, F=256, block_lens=lens, prefix_lens=0,
                           seed=61 + Hkv, dtype="bf16", with_alpha=True)
    d = bha.make_dims(8, Hq, Hkv, 128, 256, 32, int(c.cu_blk[-1]), 10, torch.bfloat16)
    assert bha.kernel_variant(d, 4) == 1
    S_np, Z_np = inputs.random_states(10, Hkv, 256, 128, prefix_len=700, seed=12)
    slots = np.array([3, 9, 0, 5, 1, 2, 8, 6], dtype=np.int32)
    S, Z = dev(S_np, torch.float32), dev(Z_np, torch.float32)
    O = _run_fused(c, S, Z, alpha=c.alpha, state_slot=torch.tensor(slots, device="cuda"))
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, S_np, Z_np, c.W, c.alpha, slots)
    assert_close(host64(O), want, TOL_BF16, "O")
    So, Zo = ref.commit_block(c.cu_blk, c.K, c.V, c.W, S_np, Z_np, slots)
    assert_close(host64(S), So, TOL_BF16, "S")
    assert_close(host64(Z), Zo, TOL_BF16, "Z")
    for untouched in (4, 7, 9):  # slot 9 holds an empty block, slots 4 and 7 no request
        np.testing.assert_array_equal(host64(S[untouched]), S_np[untouched])


def test_fused_step_and_commit_many_units_per_cta_matches_separate_calls():
    """600 requests (about 17 units per CTA), states committed from 64-token prefixes: the
    fused call's output equals the decode-only call's bit for bit (same kernel arithmetic),
    and its states match a separate commit's and, for 6 sampled requests, the oracle's."""
    c = inputs.decode_case(R=600, Hq=16, Hkv=4, d=128, F=256, block_lens=32, prefix_lens=64,
                           seed=63, dtype="bf16")
    S, Z = build_states_on_gpu(c, block=32)
    S2, Z2 = S.clone(), Z.clone()
    O_sep = run_hybrid(c, S2, Z2)
    cu = torch.tensor(c.cu_blk, dtype=torch.int32, device="cuda")
    bha.commit_block(cu, dev(c.K, torch.bfloat16), dev(c.V, torch.bfloat16),
                     dev(c.W, torch.bfloat16), S2, Z2, max_block=32)
    O = _run_fused(c, S, Z)
    assert torch.equal(O, O_sep)
    assert_close(host64(S), host64(S2), TOL_BF16, "S vs separate commit")
    assert_close(host64(Z), host64(Z2), TOL_BF16, "Z vs separate commit")
    reqs = np.random.default_rng(7).choice(600, 6, replace=False)
    for r in reqs:
        lo, hi = c.cu_pre[r], c.cu_pre[r + 1]
        b0, b1 = c.cu_blk[r], c.cu_blk[r + 1]
        for g in range(4):
            Kall = np.concatenate([c.K_pre[lo:hi, g], c.K[b0:b1, g]])
            Vall = np.concatenate([c.V_pre[lo:hi, g], c.V[b0:b1, g]])
            So, Zo = ref.state_from_tokens(Kall, Vall, c.W[g])
            assert_close(host64(S[r, g]), So, TOL_BF16, f"S[{r},{g}]")
            assert_close(host64(Z[r, g]), Zo, TOL_BF16, f"Z[{r},{g}]")


def test_fused_step_and_commit_generic_dims():
    """Dims outside the tensor-core kernel (fp32, small odd sizes) take the generic decode step
    and commit as two launches; same results against the oracle."""
    c = inputs.decode_case(R=3, Hq=6, Hkv=2, d=24, F=20, block_lens=[7, 1, 13], prefix_lens=[9, 0, 30],
                           seed=65, dtype="f32", with_alpha=True)
    assert bha.kernel_variant(bha.make_dims(3, 6, 2, 24, 20, 13, 21, 3, torch.float32), 4) == 0
    S, Z = build_states_on_gpu(c, block=16)
    So, Zo = oracle_states(c)
    O = _run_fused(c, S, Z, alpha=c.alpha)
    want = ref.hybrid_attn(c.cu_blk, c.Q, c.K, c.V, So, Zo, c.W, c.alpha)
    assert_close(host64(O), want, TOL_F32, "O")
    S1, Z1 = ref.commit_block(c.cu_blk, c.K, c.V, c.W, So, Zo)
    assert_close(host64(S), S1, TOL_F32, "S")
    assert_close(host64(Z), Z1, TOL_F32, "Z")
