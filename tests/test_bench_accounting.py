"""The roofline numerators bench.py reports: algorithmic bytes and FLOPs per launch, checked on
the CPU against the figures stated for each workload, and against the byte sizes of the
tensors each call reads and writes once (numel x element size)."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_accounting", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_decode_step_bytes_and_flops():
    b = _bench()
    R, Hq, Hkv, d, F, B = 128, 16, 4, 128, 256, 32
    T = R * B
    tensors = {  # numel x bytes, each read or written once per step
        "S": R * Hkv * F * d * 4, "Z": R * Hkv * F * 4, "Q": T * Hq * d * 2, "K": T * Hkv * d * 2,
        "V": T * Hkv * d * 2, "O": T * Hq * d * 2, "W": Hkv * d * (F // 2) * 2,
    }
    assert tensors == {"S": 67_108_864, "Z": 524_288, "Q": 16_777_216, "K": 4_194_304,
                       "V": 4_194_304, "O": 16_777_216, "W": 131_072}
    assert b.step_bytes() == sum(tensors.values()) == 109_707_264
    # per (request, query head): q.W 1,048,576 + q.k 262,144 + P.V 262,144 + phi.S 2,097,152
    # + phi.Z 16,384 FLOPs over the block's 32 queries
    assert b.step_flops() == R * Hq * 3_686_400 == 7_549_747_200


def test_commit_bytes():
    b = _bench()
    R, Hkv, d, F, B = 128, 4, 128, 256, 32
    rmw = 2 * (R * Hkv * F * d * 4 + R * Hkv * F * 4)
    kv = 2 * R * B * Hkv * d * 2
    assert b.commit_bytes() == rmw + kv + Hkv * d * (F // 2) * 2 == 143_785_984


def test_large_block_commit_bytes_and_flops():
    """128-token blocks: four times the K/V bytes of the serving commit, the same state
    traffic; per token k.W (d x F/2), phi(k) v^T (F x d) and the phi sum (F)."""
    b = _bench()
    R, Hkv, d, F, B = 128, 4, 128, 256, 128
    rmw = 2 * (R * Hkv * F * d * 4 + R * Hkv * F * 4)
    kv = 2 * R * B * Hkv * d * 2
    assert b.commit_bytes(B=B) == rmw + kv + Hkv * d * (F // 2) * 2 == 168_951_808
    assert b.commit_flops(B=B) == 2 * R * Hkv * B * (d * F // 2 + F * d + F) == 6_476_005_376
    assert b.commit_flops() * 4 == b.commit_flops(B=B)


def test_teacher_bytes_over_the_prefix_sweep():
    b = _bench()
    for P, want in ((512, 88_080_384), (2048, 289_406_976), (8192, 1_094_713_344),
                    (32768, 4_315_938_816)):
        assert b.teacher_bytes(64, 16, 4, 128, 32, P) == 16_777_216 + 131_072 * (P + 32) == want


def test_fused_step_and_commit_bytes():
    """The fused call moves the decode step's bytes plus one write of S and Z; the separate
    calls move the decode step's bytes plus the commit's (S and Z read and written, K, V, W)."""
    b = _bench()
    R, Hkv, d, F = 128, 4, 128, 256
    assert b.fused_bytes() == b.step_bytes() + R * Hkv * (F * d * 4 + F * 4) == 177_340_416
    assert b.step_bytes() + b.commit_bytes() - b.fused_bytes() == 76_152_832  # S read + Z + K, V, W


def test_every_profiled_kernel_has_a_capture_of_its_current_source():
    """The DRAM traffic each roofline object reports comes from an ncu capture in profiles/
    whose recorded source hash matches the kernel as it is now; a kernel edited after its
    capture would report no traffic, so the captures are kept current."""
    b = _bench()
    lookups = {"hybrid_decode": "hybrid_tc.cu", "hybrid_per_qhead": "hybrid_tc.cu",
               "fused": "hybrid_commit_tc.cu", "commit": "commit_tc.cu",
               "commit_b128": "commit_tc.cu", "featuremap": "featuremap_tc.cu",
               "teacher_8k": "full_prefix_tc.cu"}
    for key, src in lookups.items():
        got = b.profiled_traffic(key, b.source_hash(src))
        assert got is not None and got > 0, f"{key}: no capture of the current {src}"
