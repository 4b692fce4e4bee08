"""GPU parity at the serving sizes of the prefix sweep and of the ragged serving mix.

The prefix sweep (64 requests, 16 query / 4 KV heads, d 128, F 256, 32-token blocks) reads
states committed from prefixes of up to 32768 tokens, and its comparison point, the softmax
teacher, reads caches of the same length through its split-KV path.  The serving mix runs
128 requests with prefixes uniform on {0, 32, ..., 8192}, 6 layers with independent W, 8
denoising steps, a commit and the next step.  Inputs are drawn on the GPU from seeded
generators; the oracle recomputes the sampled requests from the same bytes copied to the
host.  Tolerances are those of tests/gpu_util.py.
"""
import numpy as np
import pytest
import torch

from linear_attention_diffusion_hedgehog_b200 import bha, inputs
from oracle import bha_ref as ref
from tests.gpu_util import TOL_BF16, TOL_STATE_LONG, assert_close, host64

pytestmark = pytest.mark.gpu

HQ, HKV, D, F, B = 16, 4, 128, 256, 32
BF = torch.bfloat16


def _weights(gen, layers=1):
    return [(torch.randn((HKV, D, F // 2), generator=gen, device="cuda") / D ** 0.5).to(BF)
            for _ in range(layers)]


def _commit_prefix(Kp, Vp, W, S, Z, block, lens=None):
    """Fold prefixes into S/Z with the library's commit, `block` tokens per call.  Kp, Vp:
    [R, P, Hkv, d]; lens[r] (default P) tokens of request r are committed."""
    R, P = Kp.shape[:2]
    lens = np.full(R, P) if lens is None else np.asarray(lens)
    for j in range(0, int(lens.max()), block):
        n = np.clip(lens - j, 0, block)
        if n.sum() == 0:
            break
        cu = torch.tensor(np.concatenate([[0], np.cumsum(n)]), dtype=torch.int32, device="cuda")
        rows = [Kp[r, j:j + n[r]] for r in range(R) if n[r] > 0]
        vals = [Vp[r, j:j + n[r]] for r in range(R) if n[r] > 0]
        bha.commit_block(cu, torch.cat(rows).contiguous(), torch.cat(vals).contiguous(), W, S, Z,
                         max_block=block)


@pytest.mark.parametrize("block", [32, 128])
@pytest.mark.parametrize("P", [2048, 8192, 32768])
def test_prefix_sweep_states_from_long_prefixes(P, block):
    """64 requests whose states are committed from P-token prefixes, 32 tokens per call (four
    requests per 128-row tile of the tensor-core commit) or 128 (one request per tile); the
    states and the decode step of 8 sampled requests against the oracle, which builds the
    states in one shot."""
    R = 64
    gen = torch.Generator(device="cuda")
    gen.manual_seed(P + block)
    (W,) = _weights(gen)
    Kp = torch.randn((R, P, HKV, D), generator=gen, device="cuda").to(BF)
    Vp = torch.randn((R, P, HKV, D), generator=gen, device="cuda").to(BF)
    S = torch.zeros((R, HKV, F, D), device="cuda")
    Z = torch.zeros((R, HKV, F), device="cuda")
    _commit_prefix(Kp, Vp, W, S, Z, block)
    Q = torch.randn((R * B, HQ, D), generator=gen, device="cuda").to(BF)
    K = torch.randn((R * B, HKV, D), generator=gen, device="cuda").to(BF)
    V = torch.randn((R * B, HKV, D), generator=gen, device="cuda").to(BF)
    cu = torch.arange(0, (R + 1) * B, B, dtype=torch.int32, device="cuda")
    O = bha.hybrid_attn(cu, Q, K, V, S, Z, W, max_block=B)
    torch.cuda.synchronize()
    Wh = host64(W)
    for r in np.random.default_rng(P).choice(R, 8, replace=False):
        So = np.zeros((1, HKV, F, D))
        Zo = np.zeros((1, HKV, F))
        Kr, Vr = host64(Kp[r]), host64(Vp[r])
        for g in range(HKV):
            So[0, g], Zo[0, g] = ref.state_from_tokens(Kr[:, g], Vr[:, g], Wh[g])
        # the states themselves grow with the prefix (|S| reaches ~10 at 32K tokens), so they
        # are held to the relative bounds; the outputs below keep the absolute one
        assert_close(host64(S[r]), So[0], TOL_STATE_LONG, f"S[{r}] after {P // block} commits")
        assert_close(host64(Z[r]), Zo[0], TOL_STATE_LONG, f"Z[{r}]")
        sl = slice(B * r, B * r + B)
        want = ref.hybrid_attn([0, B], host64(Q[sl]), host64(K[sl]), host64(V[sl]), So, Zo, Wh)
        assert_close(host64(O[sl]), want, TOL_BF16, f"O[{r}] at prefix {P}")


@pytest.mark.parametrize("P", [8192, 32768])
def test_prefix_sweep_teacher_long_caches(P):
    """The softmax teacher at 64 requests over caches of P + 32 tokens (at 32K split into key
    ranges and combined); every row of 8 sampled requests against the oracle."""
    R, L = 64, P + B
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7 * P)
    Kc = torch.randn((R, HKV, L, D), generator=gen, device="cuda").to(BF)
    Vc = torch.randn((R, HKV, L, D), generator=gen, device="cuda").to(BF)
    Q = torch.randn((R * B, HQ, D), generator=gen, device="cuda").to(BF)
    cu = torch.arange(0, (R + 1) * B, B, dtype=torch.int32, device="cuda")
    kv_len = torch.full((R,), L, dtype=torch.int32, device="cuda")
    # 64 requests x 4 KV heads fill the GPU up to 8K-token caches (one key range each); the
    # 32K cache is split into key ranges whose partials are combined
    assert (bha.full_prefix_workspace_bytes(R, HQ, HKV, D, B, R * B, L) > 0) == (P == 32768)
    O = host64(bha.full_prefix_attn(cu, kv_len, Q, Kc, Vc, max_block=B))
    for r in np.random.default_rng(P + 1).choice(R, 8, replace=False):
        sl = slice(B * r, B * r + B)
        want = ref.full_prefix_attn([0, B], [L], host64(Q[sl]), host64(Kc[r:r + 1]), host64(Vc[r:r + 1]))
        assert_close(O[sl], want, TOL_BF16, f"teacher O[{r}] at prefix {P}")


def test_serving_cycle_ragged_mix_six_layers():
    """128 requests with prefixes uniform on {0, 32, ..., 8192} (committed 128 tokens per call,
    as the serving bench does), 6 layers with independent W, 8 denoising steps of fresh
    activations, a commit of the last step's K/V in every layer, then one more step.  The
    request with the empty prefix, the one with the longest and six others are checked in
    every layer at the first and last step and at the step after the commit."""
    R, layers, steps = 128, 6, 8
    plen = inputs.ragged_prefix_lengths(R, seed=5)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    Ws = _weights(gen, layers)
    Pmax = int(plen.max())
    pre = []
    Ss = [torch.zeros((R, HKV, F, D), device="cuda") for _ in range(layers)]
    Zs = [torch.zeros((R, HKV, F), device="cuda") for _ in range(layers)]
    for l in range(layers):
        Kp = torch.randn((R, Pmax, HKV, D), generator=gen, device="cuda").to(BF)
        Vp = torch.randn((R, Pmax, HKV, D), generator=gen, device="cuda").to(BF)
        _commit_prefix(Kp, Vp, Ws[l], Ss[l], Zs[l], 128, lens=plen)
        pre.append((Kp, Vp))
    cu = torch.arange(0, (R + 1) * B, B, dtype=torch.int32, device="cuda")

    def acts():
        return [dict(Q=torch.randn((R * B, HQ, D), generator=gen, device="cuda").to(BF),
                     K=torch.randn((R * B, HKV, D), generator=gen, device="cuda").to(BF),
                     V=torch.randn((R * B, HKV, D), generator=gen, device="cuda").to(BF))
                for _ in range(layers)]

    checked = {}
    for st in range(steps + 1):
        a = acts()
        if st == steps:  # the block of the previous step is committed before this step
            for l in range(layers):
                bha.commit_block(cu, last[l]["K"], last[l]["V"], Ws[l], Ss[l], Zs[l], max_block=B)
        for l in range(layers):
            O = bha.hybrid_attn(cu, a[l]["Q"], a[l]["K"], a[l]["V"], Ss[l], Zs[l], Ws[l], max_block=B)
            if st in (0, steps - 1, steps):
                checked[(st, l)] = (a[l], O)
        last = a
    torch.cuda.synchronize()

    order = np.argsort(plen)
    rng = np.random.default_rng(2)
    reqs = [int(order[0]), int(order[-1])] + [int(r) for r in rng.choice(order[1:-1], 6, replace=False)]
    assert plen[reqs[0]] == 0 and plen[reqs[1]] == Pmax
    for l in range(layers):
        Wh = host64(Ws[l])
        for r in reqs:
            n = int(plen[r])
            So = np.zeros((1, HKV, F, D))
            Zo = np.zeros((1, HKV, F))
            if n:
                Kr, Vr = host64(pre[l][0][r, :n]), host64(pre[l][1][r, :n])
                for g in range(HKV):
                    So[0, g], Zo[0, g] = ref.state_from_tokens(Kr[:, g], Vr[:, g], Wh[g])
            sl = slice(B * r, B * r + B)
            for st in (0, steps - 1, steps):
                if st == steps:
                    blk = checked[(steps - 1, l)][0]
                    So, Zo = ref.commit_block([0, B], host64(blk["K"][sl]), host64(blk["V"][sl]), Wh, So, Zo)
                a, O = checked[(st, l)]
                want = ref.hybrid_attn([0, B], host64(a["Q"][sl]), host64(a["K"][sl]), host64(a["V"][sl]), So, Zo, Wh)
                assert_close(host64(O[sl]), want, TOL_BF16, f"layer {l} step {st} request {r} (prefix {n})")
