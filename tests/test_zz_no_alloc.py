"""The allocation-free softmax-teacher entry point (bha_full_prefix_attn_noalloc).

It serves callers that cannot allocate device memory on the call path (an engine that
reserves its whole memory budget up front, a plugin whose host owns all allocation): the
split partials live in a fixed device array inside the library instead of a caller
workspace.  The GPU test calls it through the C ABI twice in a row, on different inputs that
both need the scratch, and checks that each result equals the allocating entry point's.  The file
is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_attention_diffusion_hedgehog_b200 import bha, inputs


def _case(seed, kv_len, R=3, Hq=8, Hkv=2, d=128, cap=2000):
    rng = np.random.default_rng(seed)
    lens = np.array([32, 17, 5])[:R]
    kv_len = np.asarray(kv_len, dtype=np.int32)[:R]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Q = inputs.bf16_round(rng.standard_normal((cu[-1], Hq, d)).astype(np.float32))
    Kc = inputs.bf16_round(rng.standard_normal((R, Hkv, cap, d)).astype(np.float32))
    Vc = inputs.bf16_round(rng.standard_normal((R, Hkv, cap, d)).astype(np.float32))
    t = lambda x: torch.from_numpy(x).cuda().to(torch.bfloat16)
    return (torch.tensor(cu, device="cuda"), torch.tensor(kv_len, device="cuda"), t(Q), t(Kc), t(Vc))


def test_rejects_calls_needing_more_than_the_fixed_scratch():
    # 128 requests x 16 query heads over 32K-token caches need far more than 16 MiB of partials;
    # the call is refused on the host before anything is launched (no GPU needed).
    dims = bha.make_dims(128, 16, 4, 128, 2, 32, 4096, 0, torch.bfloat16)
    assert bha.lib().bha_full_prefix_workspace_bytes(ctypes.byref(dims), 32800) > bha.NOALLOC_SCRATCH_BYTES
    P = ctypes.c_void_p
    st = bha.lib().bha_full_prefix_attn_noalloc(ctypes.byref(dims), P(0x1000), P(0x2000), P(0x10000),
                                                P(0x20000), P(0x30000), 32800, P(0x40000), None, None)
    assert st == bha.BHA_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_noalloc_matches_allocating_entry_point_twice():
    """Two calls in a row through the shared array.  The first has long caches for every
    request, so every split of every row leaves partials behind; the second has a short and an
    empty cache, whose later splits hold nothing of their own and must not pick up the first
    call's leftovers.  The kernels and the split plan are those of the allocating entry point,
    so each result must equal its result bit for bit."""
    for seed, kv_len in ((1, [2000, 2000, 2000]), (2, [2000, 131, 0])):
        cu, kv, Q, Kc, Vc = _case(seed, kv_len)
        need = bha.full_prefix_workspace_bytes(3, 8, 2, 128, 32, int(Q.shape[0]), Kc.shape[2])
        assert 0 < need <= bha.NOALLOC_SCRATCH_BYTES      # the scratch is really used
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = bha.full_prefix_attn_noalloc(cu, kv, Q, Kc, Vc, max_block=32, dev_err=err)
        want = bha.full_prefix_attn(cu, kv, Q, Kc, Vc, max_block=32)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.equal(got, want), f"call {seed}: differs from the allocating entry point"
