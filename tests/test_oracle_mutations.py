"""The oracle's pins catch plausible slips: each case below plants one mistake in a copy of
the float64 oracle and runs the unchanged pin suite (tests/test_oracle.py) against that
copy in a subprocess; at least one pin must fail.  An unmutated copy in the same harness
must pass, so a kill is the planted slip's doing and not the harness's.

The slips are the ones the method invites ("Retrofitting Linear Attention into Diffusion
Language Models", §2.2 and §3.1): the sign of the -xW half of phi, one softmax over both
halves, W transposed, the 1/sqrt(d) temperature dropped or squared, the gate inverted or
moved to the other branch, a normaliser term dropped, keys and values swapped in the state,
a commit that overwrites instead of adding, Z as a mean, the active block also read through
the states, a causal mask inside the block, contiguous vs interleaved query-head groups (in
the decode and in the teacher), the feature-map head-to-weight map, the slot map and the
gate of the batched calls, the brute-force prefix sum's kernel, and the teacher's
temperature and key window.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_SRC = os.path.join(ROOT, "oracle", "bha_ref.py")

# (name, text in the oracle, replacement); each text must occur exactly once
MUTANTS = [
    ("phi: -xW half uses +xW",
     "return np.concatenate([softmax_last(u), softmax_last(-u)], axis=-1)",
     "return np.concatenate([softmax_last(u), softmax_last(u)], axis=-1)"),
    ("phi: one softmax over both halves",
     "return np.concatenate([softmax_last(u), softmax_last(-u)], axis=-1)",
     "return softmax_last(np.concatenate([u, -u], axis=-1))"),
    ("phi: W transposed",
     "u = _f64(x) @ _f64(W)\n",
     "u = _f64(x) @ _f64(W).T\n"),
    ("softmax normalised over rows instead of features",
     "return e / e.sum(axis=-1, keepdims=True)",
     "return e / e.sum(axis=0, keepdims=True)"),
    ("block softmax without 1/sqrt(d)",
     "a = np.exp((q @ k.T) / np.sqrt(d))\n    sm_num = a @ v\n    sm_den = a.sum(axis=1)\n"
     "    fq = phi(q, W)\n    lin_num = fq @ _f64(S)",
     "a = np.exp(q @ k.T)\n    sm_num = a @ v\n    sm_den = a.sum(axis=1)\n"
     "    fq = phi(q, W)\n    lin_num = fq @ _f64(S)"),
    ("block softmax with 1/d",
     "a = np.exp((q @ k.T) / np.sqrt(d))\n    sm_num = a @ v\n    sm_den = a.sum(axis=1)\n"
     "    fq = phi(q, W)\n    lin_num = fq @ _f64(S)",
     "a = np.exp((q @ k.T) / d)\n    sm_num = a @ v\n    sm_den = a.sum(axis=1)\n"
     "    fq = phi(q, W)\n    lin_num = fq @ _f64(S)"),
    ("causal mask inside the active block",
     "a = np.exp((q @ k.T) / np.sqrt(d))\n    sm_num = a @ v\n    sm_den = a.sum(axis=1)\n"
     "    fq = phi(q, W)\n    lin_num = fq @ _f64(S)",
     "a = np.tril(np.exp((q @ k.T) / np.sqrt(d)))\n    sm_num = a @ v\n    sm_den = a.sum(axis=1)\n"
     "    fq = phi(q, W)\n    lin_num = fq @ _f64(S)"),
    ("active block also read through the states",
     "lin_num = fq @ _f64(S)\n    lin_den = fq @ _f64(Z)",
     "S2, Z2 = commit(S, Z, k, v, W)\n    lin_num = fq @ S2\n    lin_den = fq @ Z2"),
    ("gate inverted: sigmoid(-alpha)",
     "return 1.0 / (1.0 + np.exp(-_f64(alpha)))",
     "return 1.0 / (1.0 + np.exp(_f64(alpha)))"),
    ("gate on the linear branch",
     "num = w * sm_num + lin_num\n    den = w * sm_den + lin_den",
     "num = sm_num + w * lin_num\n    den = sm_den + w * lin_den"),
    ("linear term dropped from the shared denominator",
     "den = w * sm_den + lin_den",
     "den = w * sm_den"),
    ("softmax term dropped from the shared denominator",
     "den = w * sm_den + lin_den",
     "den = lin_den"),
    ("state built from phi(v) instead of phi(k)",
     "P = phi(K, W)  # [n, F]",
     "P = phi(V, W)  # [n, F]"),
    ("commit overwrites the previous state",
     "return _f64(S) + dS, _f64(Z) + dZ",
     "return dS, dZ"),
    ("interleaved instead of contiguous query-head groups",
     "g = h // G\n            w = 1.0 if alpha",
     "g = h % Hkv\n            w = 1.0 if alpha"),
    ("feature-map head-to-weight map interleaved",
     "phi(x[:, h, :], W[(h * Hw) // H])",
     "phi(x[:, h, :], W[h % Hw])"),
    ("teacher without 1/sqrt(d)",
     "s = (q @ k.T) / np.sqrt(d)",
     "s = q @ k.T"),
    ("batched decode ignores the slot map",
     "if hi == lo:\n            continue\n        slot = r if state_slot is None else int(state_slot[r])",
     "if hi == lo:\n            continue\n        slot = r"),
    ("batched commit ignores the slot map",
     "lo, hi = int(cu_blk[r]), int(cu_blk[r + 1])\n        slot = r if state_slot is None else int(state_slot[r])",
     "lo, hi = int(cu_blk[r]), int(cu_blk[r + 1])\n        slot = r"),
    ("batched decode drops the gate",
     "w = 1.0 if alpha is None else float(gate(alpha[h]))",
     "w = 1.0"),
    ("Z as the mean of phi(k) instead of the sum",
     "return P.T @ V, P.sum(axis=0)",
     "return P.T @ V, P.mean(axis=0)"),
    ("brute-force linear kernel halved",
     "kern = fq @ phi(K_pre[t], W)  # [b]",
     "kern = 0.5 * (fq @ phi(K_pre[t], W))  # [b]"),
    ("teacher with interleaved query-head groups",
     "g = h // G\n            O[lo:hi, h] = softmax_attn_head",
     "g = h % Hkv\n            O[lo:hi, h] = softmax_attn_head"),
    ("teacher drops the last cached key",
     "softmax_attn_head(Q[lo:hi, h], Kc[r, g, :n], Vc[r, g, :n])",
     "softmax_attn_head(Q[lo:hi, h], Kc[r, g, :n - 1], Vc[r, g, :n - 1])"),
]


def _tree(base, oracle_text):
    """A throwaway tree with the (possibly mutated) oracle, the pin suite, its fixtures and
    the seeded input generators, so that `import oracle` resolves to the copy."""
    os.makedirs(os.path.join(base, "oracle"))
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), os.path.join(base, "oracle"))
    with open(os.path.join(base, "oracle", "bha_ref.py"), "w") as f:
        f.write(oracle_text)
    os.makedirs(os.path.join(base, "tests"))
    for name in ("conftest.py", "test_oracle.py"):
        shutil.copy(os.path.join(ROOT, "tests", name), os.path.join(base, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(base, "tests", "golden"))
    pkg = os.path.join(base, "linear_attention_diffusion_hedgehog_b200")
    os.makedirs(pkg)
    for name in ("__init__.py", "inputs.py"):
        shutil.copy(os.path.join(ROOT, "linear_attention_diffusion_hedgehog_b200", name), pkg)


def _run_pins(base):
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
    env.pop("PYTHONPATH", None)
    p = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle.py"], cwd=base, env=env, capture_output=True,
                       text=True, timeout=600)
    return p.returncode, p.stdout[-2000:] + p.stderr[-2000:]


def _mutate(src, a, b):
    assert src.count(a) == 1, f"mutation site not unique in the oracle: {a[:60]!r}"
    return src.replace(a, b)


def test_unmutated_copy_passes_in_the_harness(tmp_path):
    with open(ORACLE_SRC) as f:
        src = f.read()
    _tree(str(tmp_path / "clean"), src)
    rc, out = _run_pins(str(tmp_path / "clean"))
    assert rc == 0, out


def test_every_planted_slip_fails_a_pin(tmp_path):
    with open(ORACLE_SRC) as f:
        src = f.read()
    bases = []
    for i, (name, a, b) in enumerate(MUTANTS):
        base = str(tmp_path / f"m{i}")
        _tree(base, _mutate(src, a, b))
        bases.append((name, base))
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda nb: (nb[0],) + _run_pins(nb[1]), bases))
    survivors = [name for name, rc, _ in results if rc == 0]
    assert not survivors, f"slips no pin catches: {survivors}"
    # rc 1 means tests ran and failed; anything else (collection error, usage error) would
    # say nothing about the pins
    odd = [(name, rc, out[-400:]) for name, rc, out in results if rc != 1]
    assert not odd, odd
