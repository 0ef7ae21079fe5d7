"""Planted-mistake check of the oracle's pins. Run by hand (about two minutes):

    python tests/oracle_mutations.py

Each entry below is a plausible mistake in the oracle (its methods, number formats and
per-row step compositions): a dropped term, a wrong rounding, a transposed operand, a tie
broken the wrong way. For each one, a child process alters the
oracle module's source in memory (nothing is written to disk), installs the altered module
in place of the real one, and runs the oracle pin tests (`-m "not gpu"`). A mistake that no
pin catches is reported as MISSED. Two entries are rewrites that compute the same thing for
every input (marked "equivalent"); they are listed to show that the harness itself runs.
"""
from __future__ import annotations

import glob
import importlib.util
import os
import subprocess
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (module, name, original snippet, mistaken snippet)
MUTATIONS = [
    # projected-key writer, scorer, selector, attention
    ("method", "writer: product not rounded",
     "        prod = k32[:, i:i + 1] * P32[i:i + 1, :]       # float32 x float32 -> rounded float32\n"
     "        acc = acc + prod                                # rounded float32",
     "        prod = k32[:, i:i + 1].astype(np.float64) * P32[i:i + 1, :]\n"
     "        acc = (acc + prod).astype(np.float32)"),
    ("method", "writer: BF16 by truncation", "return F.f32_to_bf16_rne(acc)",
     "return (acc.view(np.uint32) >> 16).astype(np.uint16)"),
    ("method", "query: head sum, not mean",
     "qbar = F.bf16_to_f64(q_bits).mean(axis=0)\n    return qbar @ np.asarray(P, dtype=np.float64)",
     "qbar = F.bf16_to_f64(q_bits).sum(axis=0)\n    return qbar @ np.asarray(P, dtype=np.float64)"),
    ("method", "block score: mean, not max",
     "return s.reshape(s.shape[:-1] + (nb, S)).max(axis=-1)",
     "return np.nanmean(np.where(np.isinf(s), np.nan, s).reshape(s.shape[:-1] + (nb, S)), axis=-1)"),
    ("method", "select: ties to the higher index",
     "order = np.lexsort((rest, -beta[rest]))             # primary: -beta, secondary: index",
     "order = np.lexsort((-rest, -beta[rest]))"),
    ("method", "select: forced blocks not counted",
     "take = rest[order[: budget - len(forced)]]", "take = rest[order[: budget]]"),
    ("method", "attention: scale dropped",
     "logits = scale * (q @ Kt.T)                               # [G][T]", "logits = (q @ Kt.T)"),
    ("method", "combine: partials not rescaled", "w = np.exp(ms - M[None, :])", "w = np.ones_like(ms)"),
    ("method", "dense attention: last token dropped",
     "logits = scale * (q @ K[:L].T)\n    w = np.exp(logits - logits.max(axis=1, keepdims=True))\n"
     "    return (w @ V[:L])",
     "logits = scale * (q @ K[:L - 1].T)\n    w = np.exp(logits - logits.max(axis=1, keepdims=True))\n"
     "    return (w @ V[:L - 1])"),
    ("method", "gather: cut tokens kept", "            if t < L:\n                src[i * S + u] = t",
     "            src[i * S + u] = t"),
    # centroid scoring and calibration
    ("method", "centroid: divided by S, not the valid count",
     "cnt = np.minimum(S, L - np.arange(nb) * S).astype(np.float64)", "cnt = np.full(nb, float(S))"),
    ("method", "centroid: no restart (equivalent: the sums start at zero)",
     "out[j] = k32[t] if t % S == 0 else (out[j] + k32[t])   # one float32 rounding per add",
     "out[j] = out[j] + k32[t]"),
    ("method", "calibration: no unit-trace normalisation",
     "return cq / np.trace(cq) + ck / np.trace(ck)", "return cq + ck"),
    ("method", "basis: smallest eigenvalues", 'order = np.argsort(-w, kind="stable")[:r]',
     'order = np.argsort(w, kind="stable")[:r]'),
    ("method", "basis: sign convention flipped", "if P[i, c] < 0:", "if P[i, c] > 0:"),
    # NVFP4
    ("method", "NVFP4: scale from 4, not 6", "den = np.float32(np.float32(E2M1_MAX) * g)",
     "den = np.float32(np.float32(4.0) * g)"),
    ("method", "NVFP4: keys not centred",
     "return (F.bf16_to_f64(k_bits).astype(np.float32) - np.asarray(mu, dtype=np.float32)\n"
     "            ).astype(np.float32)",
     "return (F.bf16_to_f64(k_bits).astype(np.float32)).astype(np.float32)"),
    ("method", "NVFP4: heads averaged, not maxed", "return block_max(head_scores.max(axis=0), S)",
     "return block_max(head_scores.mean(axis=0), S)"),
    ("method", "NVFP4: kept blocks with the smallest error",
     "order = np.lexsort((valid, -err[valid]))", "order = np.lexsort((valid, err[valid]))"),
    ("method", "NVFP4 attended keys: centre not added before rounding",
     "    v = (v + np.asarray(mu, dtype=np.float32)[None, :]).astype(np.float32)\n    out = F.f32_to_bf16_rne(v)",
     "    out = F.f32_to_bf16_rne(v)"),
    ("method", "NVFP4 attended keys: BF16 by truncation",
     "    out = F.f32_to_bf16_rne(v)\n    bits = np.asarray(k_bits[:L], dtype=np.uint16)",
     "    out = (v.view(np.uint32) >> 16).astype(np.uint16)\n    bits = np.asarray(k_bits[:L], dtype=np.uint16)"),
    ("method", "NVFP4 attended keys: kept blocks not restored",
     "        out[t0:t1] = bits[t0:t1]\n    return out", "        pass\n    return out"),
    # binary proxy and top-p
    ("method", "binary: bit set at y = 0", "bits = (y > 0).astype(np.uint8)",
     "bits = (y >= 0).astype(np.uint8)"),
    ("method", "binary: |o| instead of |o|^2",
     "g = np.where(l1 > 0, (n2 / safe).astype(np.float32), np.float32(0.0)).astype(np.float32)",
     "g = np.where(l1 > 0, (np.sqrt(n2) / safe).astype(np.float32), np.float32(0.0)).astype(np.float32)"),
    ("method", "binary: rotation products fused",
     "        acc = acc + x32[:, j:j + 1] * R32[j:j + 1, :]",
     "        acc = (acc.astype(np.float64) + x32[:, j:j + 1].astype(np.float64) * R32[j:j + 1, :]"
     ").astype(np.float32)"),
    ("method", "binary: rotation transposed", "acc = acc + x32[:, j:j + 1] * R32[j:j + 1, :]",
     "acc = acc + x32[:, j:j + 1] * R32.T[j:j + 1, :]"),
    ("method", "binary: query rounded to nearest, not at random",
     "n = np.floor((t + np.asarray(u, dtype=np.float32)).astype(np.float32)).astype(np.int64)",
     "n = np.floor((t + np.float32(0.5)).astype(np.float32)).astype(np.int64)"),
    ("method", "binary: query code not clamped", "return np.minimum(n, RQ_QUERY_LEVELS), delta, vl, qbar",
     "return n, delta, vl, qbar"),
    ("method", "binary: 16 levels",
     "delta = np.float32(np.float32(vr - vl) / np.float32(RQ_QUERY_LEVELS))",
     "delta = np.float32(np.float32(vr - vl) / np.float32(16))"),
    ("method", "binary: centre term dropped",
     "return np.asarray(g, dtype=np.float64) * (sgn @ qhat) + shift",
     "return np.asarray(g, dtype=np.float64) * (sgn @ qhat)"),
    ("method", "block mass: max, not sum",
     "return np.concatenate([w, pad]).reshape(nb, S).sum(axis=1)",
     "return np.concatenate([w, pad]).reshape(nb, S).max(axis=1)"),
    ("method", "top-p: goal needs >, not >=", "if len(taken) >= budget or acc >= goal:",
     "if len(taken) >= budget or acc > goal:"),
    ("method", "top-p: forced mass not counted", "    for j in taken:\n        acc += float(mass[j])\n", ""),
    ("method", "top-p: ties to the higher index", "for j in rest[np.lexsort((rest, -mass[rest]))]:",
     "for j in rest[np.lexsort((-rest, -mass[rest]))]:"),
    # semantic blocks
    ("method", "k-means: farthest centroid", "assign = np.argmin(d2, axis=1)",
     "assign = np.argmax(d2, axis=1)"),
    ("method", "k-means: seeds at the first C keys",
     "cent = x[(np.arange(C) * L0) // C].copy()\n    assign = np.zeros(L0, dtype=np.int64)\n"
     "    for _ in range(max(iters, 1)):\n        d2",
     "cent = x[np.arange(C)].copy()\n    assign = np.zeros(L0, dtype=np.int64)\n"
     "    for _ in range(max(iters, 1)):\n        d2"),
    ("method", "k-means float32: seeds at the first C keys",
     "cent = x[(np.arange(C) * L0) // C].copy()\n    assign = np.zeros(L0, dtype=np.int64)\n"
     "    for _ in range(max(iters, 1)):\n        acc",
     "cent = x[np.arange(C)].copy()\n    assign = np.zeros(L0, dtype=np.int64)\n"
     "    for _ in range(max(iters, 1)):\n        acc"),
    ("method", "semantic: head sum, not mean", "return cent @ F.bf16_to_f64(q_bits).mean(axis=0)",
     "return cent @ F.bf16_to_f64(q_bits).sum(axis=0)"),
    ("method", "semantic: tokens after the prompt dropped",
     "return np.concatenate([members, np.arange(L0, L)]).astype(np.int64)",
     "return members.astype(np.int64)"),
    ("method", "k-means float32: distances in float64",
     "        acc = np.zeros((L0, C), dtype=np.float32)\n        for i in range(d):\n"
     "            diff = (x[:, i:i + 1] - cent[None, :, i]).astype(np.float32)\n"
     "            acc = (acc + (diff * diff).astype(np.float32)).astype(np.float32)",
     "        acc = ((x[:, None, :].astype(np.float64) - cent[None, :, :]) ** 2).sum(axis=2)"),
    ("method", "k-means float32: dimensions summed in reverse",
     "        for i in range(d):\n            diff = (x[:, i:i + 1] - cent[None, :, i]).astype(np.float32)",
     "        for i in reversed(range(d)):\n            diff = (x[:, i:i + 1] - cent[None, :, i]).astype(np.float32)"),
    ("method", "k-means float32: members summed pairwise",
     "            s = np.zeros(d, dtype=np.float32)\n            for t in members:                                                # token order\n"
     "                s = (s + x[t]).astype(np.float32)",
     "            s = x[members].sum(axis=0, dtype=np.float64).astype(np.float32)"),
    # the per-row step compositions
    ("step", "step: V decoded as BF16 when stored FP16",
     "return F.f16_to_f64(v_bits) if v_dtype == \"f16\" else F.bf16_to_f64(v_bits)",
     "return F.bf16_to_f64(v_bits)"),
    ("step", "step: attention over the oracle's selection, ignoring an accepted one",
     "    use = sel if sel_override is None else np.asarray(sel_override, dtype=np.int64)\n"
     "    tokens = M.block_tokens(use, p.S, L)\n    q = F.bf16_to_f64(q_bits)",
     "    use = sel\n    tokens = M.block_tokens(use, p.S, L)\n    q = F.bf16_to_f64(q_bits)"),
    ("step", "top-p step: weights without the softmax scale",
     "    w = M.estimated_weights(s, p.scale)", "    w = M.estimated_weights(s, 1.0)"),
    ("step", "top-p step: forced blocks dropped",
     "    forced = M.forced_blocks(mass.shape[0], p.force_sink, p.force_last)",
     "    forced = np.zeros(0, dtype=np.int64)"),
    ("step", "semantic step: tokens after the prompt dropped",
     "    tokens = M.semantic_tokens(assign, use, L0, L)",
     "    tokens = M.semantic_tokens(assign, use, L0, L0)"),
    ("step", "NVFP4 step: query packed with the key scale",
     "        q_codes, q_scales = M.nvfp4_pack(qx, g_q)",
     "        q_codes, q_scales = M.nvfp4_pack(qx, g_k)"),
    ("step", "step: kept blocks not forced",
     "    return M.forced_blocks(nb, p.force_sink, p.force_last, keep), keep",
     "    return M.forced_blocks(nb, p.force_sink, p.force_last), keep"),
    ("step", "step: projected query over the whole group, not its mean",
     "    qt = M.proxy_query(q_bits, P)\n    s = M.token_scores",
     "    qt = M.proxy_query(q_bits, P) * q_bits.shape[0]\n    s = M.token_scores"),
    ("step", "centroid step: sums of the blocks past the row read",
     "        return M.centroid_block_scores(q_bits, cache[:-(-L // p.S)], p.S, L)",
     "        return M.centroid_block_scores(q_bits, cache[:-(-L // p.S) - 1], p.S, L)"),
    # number formats
    ("formats", "BF16: ties away from zero", "y = np.round(x64 / step) * step            # np.round is half-to-even",
     "y = np.floor(x64 / step + 0.5) * step"),
    ("formats", "BF16: 7 significant bits", "step = np.ldexp(1.0, e - 8)", "step = np.ldexp(1.0, e - 7)"),
    ("formats", "table rounding: ties to odd", "return np.where(at_mid & odd, idx + 1, idx)",
     "return np.where(at_mid & ~odd, idx + 1, idx)"),
    ("formats", "table rounding: ties down", "return np.where(at_mid & odd, idx + 1, idx)", "return idx"),
    ("formats", "UE4M3: saturation line removed (equivalent: the table already saturates)",
     "return np.where(s64 >= 448.0, 126, code).astype(np.uint8)",
     "return np.minimum(code, 127).astype(np.uint8)"),
    ("formats", "E2M1: sign of -0 lost", "return (code | np.where(np.signbit(t64), 8, 0)).astype(np.uint8)",
     "return (code | np.where(t64 < 0, 8, 0)).astype(np.uint8)"),
    ("formats", "E4M3: sign of -0 lost", "return (mag | np.where(np.signbit(x64), 0x80, 0)).astype(np.uint8)",
     "return (mag | np.where(x64 < 0, 0x80, 0)).astype(np.uint8)"),
    ("formats", "UE4M3: subnormal step 2^-10",
     "v = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))",
     "v = np.where(e == 0, m * 2.0 ** -10, (1.0 + m / 8.0) * np.exp2(e - 7.0))"),
]


def _load(name: str, source: str, package):
    mod = types.ModuleType(f"oracle.{name}")
    mod.__package__ = "oracle"
    mod.__file__ = os.path.join(ROOT, "oracle", f"{name}.py")
    sys.modules[mod.__name__] = mod
    exec(compile(source, mod.__file__, "exec"), mod.__dict__)
    setattr(package, name, mod)
    return mod


def run_one(index: int) -> int:
    """In this process: install the mutated oracle, run the pins; pytest's exit status."""
    import pytest
    sys.path.insert(0, ROOT)
    target, _, old, new = MUTATIONS[index]
    spec = importlib.util.spec_from_file_location(
        "oracle", os.path.join(ROOT, "oracle", "__init__.py"),
        submodule_search_locations=[os.path.join(ROOT, "oracle")])
    package = importlib.util.module_from_spec(spec)
    sys.modules["oracle"] = package
    for name in ("formats", "method", "step"):            # in dependency order
        src = open(os.path.join(ROOT, "oracle", f"{name}.py")).read()
        if name == target:
            assert src.count(old) == 1, "snippet not found"
            src = src.replace(old, new)
        _load(name, src, package)
    tests = sorted(glob.glob(os.path.join(ROOT, "tests", "test_oracle_*.py")))
    return int(pytest.main(["-q", "-x", "-p", "no:cacheprovider", "-m", "not gpu",
                            "--rootdir", ROOT, *tests]))


def main() -> int:
    missed = 0
    for i, (_, name, _, _) in enumerate(MUTATIONS):
        r = subprocess.run([sys.executable, os.path.abspath(__file__), "--one", str(i)],
                           cwd=ROOT, capture_output=True, text=True)
        caught = r.returncode not in (0, 5)                   # 5: no tests collected
        if r.returncode == 5 or "snippet not found" in r.stderr:
            print(f"{name}: NOT RUN ({r.stderr.strip().splitlines()[-1:]})")
            missed += 1
            continue
        equivalent = "equivalent" in name
        verdict = "caught" if caught else ("not caught (equivalent rewrite)" if equivalent else "MISSED")
        missed += (not caught) and not equivalent
        print(f"{name}: {verdict}")
    print(f"{len(MUTATIONS)} planted mistakes, {missed} missed")
    return 1 if missed else 0


if __name__ == "__main__":
    if len(sys.argv) == 3 and sys.argv[1] == "--one":
        sys.exit(run_one(int(sys.argv[2])))
    sys.exit(main())
