"""Planted mistakes in the oracle must fail its pins.

Each mutant below is one plausible slip in the CPU oracle: a dropped term, a
wrong sign or comparison, an off-by-one bound, a transposed operand, the
wrong tie rule.  For each one the test writes a copy of the oracle package
with that single change into a temporary directory, runs
tests/test_oracle_pins.py against the copy in a child process, and requires
the pins to fail.  A mutant that survives is a gap in the pins.

Every mutant keeps every array access in bounds, so a child fails by an
assertion, never by a crash.  Nothing here touches the CUDA library.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

CPP, PY = "oracle.cpp", "__init__.py"

# (name, file, [(text, replacement), ...]); each text occurs exactly once.
MUTANTS = [
    # --- low-rank projection and block centroids ---
    ("projector transposed", CPP, [("static_cast<double>(P[d * r + c])", "static_cast<double>(P[c * D + d])")]),
    ("bf16 widened with the wrong shift", CPP, [("static_cast<uint32_t>(h) << 16", "static_cast<uint32_t>(h) << 15")]),
    ("centroid is a sum, not a mean", CPP, [("out[b * r + c] = acc[c] / B;", "out[b * r + c] = acc[c];")]),
    ("centroid drops the block's first key", CPP,
     [("for (long j = b * B; j < (b + 1) * B; ++j) {\n      project_row(k",
       "for (long j = b * B + 1; j < (b + 1) * B; ++j) {\n      project_row(k")]),
    # --- query summary and scores ---
    ("query summary not averaged over the block", CPP, [("acc[c] += mean[c] / B;", "acc[c] += mean[c];")]),
    ("query summary from one head", CPP,
     [("for (int h = 0; h < G; ++h) {\n      std::vector<double> mean(r, 0.0);",
       "for (int h = 0; h < 1; ++h) {\n      std::vector<double> mean(r, 0.0);")]),
    ("score with the centroids transposed", CPP, [("s += qbar[c] * C[j * r + c];", "s += qbar[c] * C[c * nb + j];")]),
    # --- fixed top-k selection ---
    ("sink block is a candidate", CPP, [("for (long j = 1; j <= last_cand; ++j)", "for (long j = 0; j <= last_cand; ++j)")]),
    ("candidate range one block short", CPP, [("long last_cand = t - n_local;", "long last_cand = t - n_local - 1;")]),
    ("lowest scores kept", CPP,
     [("return s[a] > s[b];\n        return a < b;\n      });\n      cand.resize(topk);",
       "return s[a] < s[b];\n        return a < b;\n      });\n      cand.resize(topk);")]),
    ("ties kept by higher index", CPP,
     [("return a < b;\n      });\n      cand.resize(topk);", "return a > b;\n      });\n      cand.resize(topk);")]),
    ("sink block dropped", CPP,
     [("std::vector<long> all(cand.begin(), cand.end());\n    all.push_back(0);",
       "std::vector<long> all(cand.begin(), cand.end());")]),
    ("one local block short", CPP,
     [("all(cand.begin(), cand.end());\n    all.push_back(0);\n    for (long j = std::max<long>(0, t - n_local + 1);",
       "all(cand.begin(), cand.end());\n    all.push_back(0);\n    for (long j = std::max<long>(0, t - n_local + 2);")]),
    ("k-th score taken from the best candidate", CPP, [("kth = s[cand.back()];", "kth = s[cand.front()];")]),
    # --- row-max scores ---
    ("row-max skips the block's first row", CPP,
     [("for (int i = 0; i < B; ++i) {\n      double s = 0.0;", "for (int i = 1; i < B; ++i) {\n      double s = 0.0;")]),
    ("row-max keeps the minimum", CPP, [("best = std::max(best, s);", "best = std::min(best, s);")]),
    ("row-max query from one head", CPP,
     [("u[static_cast<size_t>(i) * r + c] += qt[c];", "u[static_cast<size_t>(i) * r + c] = qt[c];")]),
    # --- dynamic budget ---
    ("dynamic cut is strict", CPP, [("if (prefix[e] >= mass * Z) {", "if (prefix[e] > mass * Z) {")]),
    ("dynamic cut one candidate late", CPP, [("nstar = e + 1;", "nstar = e + 2;")]),
    ("dynamic weights without beta", CPP,
     [("Z += std::exp(beta * (s[j] - smax));", "Z += std::exp(s[j] - smax);"),
      ("acc += std::exp(beta * (s[cand[e]] - smax));", "acc += std::exp(s[cand[e]] - smax);")]),
    ("dynamic minimum ignored", CPP, [("      nstar = std::max(nstar, std::min<long>(min_k, m));\n", "")]),
    ("dynamic cap ignored", CPP, [("      nstar = std::min(nstar, std::min<long>(cap, m));\n", "")]),
    # --- k-means ---
    ("k-means seeds at the first rows", CPP,
     [("const long j = (static_cast<long>(2 * c + 1) * n) / (2L * nc);", "const long j = static_cast<long>(c);")]),
    ("k-means ties to the higher index", CPP, [("if (dist < best) {", "if (dist <= best) {")]),
    ("k-means empty cluster zeroed", CPP,
     [("if (count[c] > 0)\n        for (int d = 0; d < r; ++d) mu[c * r + d] = sum[c * r + d] / count[c];",
       "for (int d = 0; d < r; ++d) mu[c * r + d] = count[c] > 0 ? sum[c * r + d] / count[c] : 0.0;")]),
    ("k-means one round fewer", CPP, [("for (int it = 0; it < iters; ++it) {", "for (int it = 1; it < iters; ++it) {")]),
    ("k-means mean over one more point", CPP,
     [("mu[c * r + d] = sum[c * r + d] / count[c];", "mu[c * r + d] = sum[c * r + d] / (count[c] + 1);")]),
    # --- attention over a key list ---
    ("key-list attention without the scale", CPP, [("s[e] = acc * scale;", "s[e] = acc;")]),
    ("key-list attention takes values from K", CPP,
     [("const double p = std::exp(s[e] - m);\n      l += p;\n      for (int d = 0; d < D; ++d) o[d] += p * widen_bf16(vc[",
       "const double p = std::exp(s[e] - m);\n      l += p;\n      for (int d = 0; d < D; ++d) o[d] += p * widen_bf16(kc[")]),
    # --- visible keys and row attention ---
    ("window one key wider", CPP,
     [("for (long j = std::max<long>(0, i - W + 1); j <= i && j < N; ++j)",
       "for (long j = std::max<long>(0, i - W); j <= i && j < N; ++j)")]),
    ("full head excludes the diagonal", CPP, [("for (long j = 0; j <= i && j < N; ++j)", "for (long j = 0; j < i && j < N; ++j)")]),
    ("selected blocks not causally masked", CPP,
     [("        if (j <= i) keys.push_back(j);\n    }\n  }\n  return", "        keys.push_back(j);\n    }\n  }\n  return")]),
    ("row attention without the scale", CPP,
     [("acc += qd[d] * widen_bf16(kj[d]);\n      s[e] = scale * acc;", "acc += qd[d] * widen_bf16(kj[d]);\n      s[e] = acc;")]),
    ("row attention takes values from K", CPP, [("const uint16_t* vj = v + keys[e] * D;", "const uint16_t* vj = k + keys[e] * D;")]),
    ("row attention not normalised", CPP,
     [("out[r * D + d] = keys.empty() ? 0.0 : o[d] / l;", "out[r * D + d] = keys.empty() ? 0.0 : o[d];")]),
    ("probabilities not normalised", CPP,
     [("probs[keys[e]] = std::exp(s[e] - m) / l;", "probs[keys[e]] = std::exp(s[e] - m);")]),
    # --- decode ---
    ("decode summary from one head", CPP, [("for (int c = 0; c < r; ++c) qbar[c] += qt[c];", "for (int c = 0; c < r; ++c) qbar[c] = qt[c];")]),
    ("decode selects for the previous token's block", CPP,
     [("int32_t t = static_cast<int32_t>(i / B);", "int32_t t = static_cast<int32_t>((i - 1) / B);")]),
    ("decode window one key wider", CPP,
     [("for (long j = std::max<long>(0, i - window + 1); j <= i; ++j) keys.push_back(j);",
       "for (long j = std::max<long>(0, i - window); j <= i; ++j) keys.push_back(j);")]),
    ("decode full head misses the new token", CPP,
     [("for (long j = 0; j <= i; ++j) keys.push_back(j);", "for (long j = 0; j < i; ++j) keys.push_back(j);")]),
    ("query summary rows read head-interleaved", CPP,
     [("project_row(q + (static_cast<long>(h) * N + i) * D, D, P, r, qt.data());\n        for (int c = 0; c < r; ++c) mean[c]",
       "project_row(q + (i * G + h) * D, D, P, r, qt.data());\n        for (int c = 0; c < r; ++c) mean[c]")]),
    ("query summary drops the block's first row", CPP,
     [("for (long i = t * B; i < (t + 1) * B; ++i) {", "for (long i = t * B + 1; i < (t + 1) * B; ++i) {")]),
    ("row-max scores with the centroids transposed", CPP,
     [("s += u[static_cast<size_t>(i) * r + c] * C[j * r + c];", "s += u[static_cast<size_t>(i) * r + c] * C[c * nb + j];")]),
    ("dynamic covered fraction before the cut off by one", CPP,
     [("cum_lo[q] = nstar >= 2 ? prefix[nstar - 2] / Z", "cum_lo[q] = nstar >= 2 ? prefix[nstar - 1] / Z")]),
    ("k-means with an absolute-value distance", CPP, [("dist += e * e;", "dist += std::fabs(e);")]),
    ("key-list attention ignores the list", CPP,
     [("widen_bf16(kc[keys[e] * D + d]);\n      s[e] = acc * scale;", "widen_bf16(kc[e * D + d]);\n      s[e] = acc * scale;")]),
    ("sparse rows read the first query block's selection", CPP,
     [("long b = sel[t * static_cast<long>(kmax) + e];", "long b = sel[e];")]),
    ("decode overrides a given selection", CPP, [("if (mode == 2 && !use_given_sel) {", "if (mode == 2) {")]),
    ("k-means seeds one row late", CPP,
     [("const long j = (static_cast<long>(2 * c + 1) * n) / (2L * nc);",
       "const long j = std::min(n - 1, (static_cast<long>(2 * c + 1) * n) / (2L * nc) + 1);")]),
    ("probabilities without the scale", CPP,
     [("acc += widen_bf16(q_row[d]) * widen_bf16(k[keys[e] * D + d]);\n    s[e] = scale * acc;",
       "acc += widen_bf16(q_row[d]) * widen_bf16(k[keys[e] * D + d]);\n    s[e] = acc;")]),
    ("decode drops the new token's own key from its block", CPP,
     [("        for (long j = b * B; j < (b + 1) * B; ++j)\n          if (j <= i) keys.push_back(j);",
       "        for (long j = b * B; j < (b + 1) * B; ++j)\n          if (j < i) keys.push_back(j);")]),
    ("projection drops the last dimension", CPP,
     [("for (int d = 0; d < D; ++d) s += static_cast<double>(P[d * r + c])",
       "for (int d = 0; d < D - 1; ++d) s += static_cast<double>(P[d * r + c])")]),
    ("k-means mean sums the first dimension only", CPP,
     [("sum[assign[j] * r + d] += X[j * r + d];", "sum[assign[j] * r + d] += X[j * r];")]),
    ("row attention reads the first query row for every row", CPP,
     [("qd[d] = widen_bf16(q_rows[r * D + d]);", "qd[d] = widen_bf16(q_rows[d]);")]),
    ("decode summary takes head 0 for every head", CPP,
     [("project_row(q + h * D, D, P, r, qt.data());\n      for (int c = 0; c < r; ++c) qbar[c] += qt[c];",
       "project_row(q, D, P, r, qt.data());\n      for (int c = 0; c < r; ++c) qbar[c] += qt[c];")]),
    # --- Python statements ---
    ("chunk ties kept by higher index", PY,
     [("order = np.lexsort((np.arange(s.size), -s))", "order = np.lexsort((-np.arange(s.size), -s))")]),
    ("lowest-scoring chunks kept", PY,
     [("order = np.lexsort((np.arange(s.size), -s))", "order = np.lexsort((np.arange(s.size), s))")]),
    ("clustered tail starts one key late", PY,
     [("keys.extend(range(clu_end, cache_len))", "keys.extend(range(clu_end + 1, cache_len))")]),
    ("clustered sink misses key 0", PY,
     [("keys = list(range(0, min(block, cache_len)))", "keys = list(range(1, min(block, cache_len)))")]),
    ("chosen chunk loses its last key", PY, [("members[s0:s0 + n]", "members[s0:s0 + n - 1]")]),
    ("cluster members in descending order", PY,
     [("order = np.lexsort((np.arange(a.size), a))", "order = np.lexsort((-np.arange(a.size), a))")]),
    ("chunks one key shorter", PY,
     [("chunks.append((c, s0, min(chunk, int(offsets[c + 1]) - s0)))",
       "chunks.append((c, s0, min(chunk - 1, int(offsets[c + 1]) - s0)))")]),
    ("bf16 rounding half away from zero", PY,
     [("r = ((u + np.uint64((1 << 44) - 1) + lsb) >> keep) << keep", "r = ((u + np.uint64(1 << 44)) >> keep) << keep")]),
    ("bf16 rounding truncates", PY,
     [("r = ((u + np.uint64((1 << 44) - 1) + lsb) >> keep) << keep", "r = (u >> keep) << keep")]),
    ("chunk top-k keeps one fewer", PY, [("return np.sort(order[:topk])", "return np.sort(order[:topk - 1])")]),
    ("cache centroids written for every head", PY,
     [("if int(kinds[h]) == SPARSE and n > 0:", "if n > 0:")]),
    ("append completes a block one row early", PY, [("if (pos + 1) % block == 0:", "if (pos + 2) % block == 0:")]),
    ("append writes the next block's centroid", PY,
     [("blk = (pos + 1) // block - 1", "blk = min((pos + 1) // block, Cn.shape[2] - 1)")]),
    ("bf16 subnormals on the wrong spacing", PY,
     [("out[tiny] = np.round(a[tiny] * 2.0 ** 133) * 2.0 ** -133", "out[tiny] = np.round(a[tiny] * 2.0 ** 132) * 2.0 ** -132")]),
    ("bf16 overflow kept finite", PY,
     [("out[over] = np.copysign(np.inf, a[over])", "out[over] = np.copysign(_BF16_MAX, a[over])")]),
    ("matrix attention window starts one key late", PY,
     [("keys = torch.arange(max(0, int(pp[idx].min()) - window + 1), hi + 1)",
       "keys = torch.arange(max(0, int(pp[idx].min()) - window + 2), hi + 1)")]),
    ("cluster sizes miss trailing empty clusters", PY,
     [("counts = np.bincount(a, minlength=n_clusters)", "counts = np.bincount(a)")]),
    ("matrix attention drops each selected block's last key", PY,
     [("torch.arange(b * block, (b + 1) * block) for b in blocks", "torch.arange(b * block, (b + 1) * block - 1) for b in blocks")]),
    ("bf16 rounding loses NaN", PY, [("    out[np.isnan(a)] = np.nan\n", "")]),
    ("chunk top-k left in score order", PY, [("return np.sort(order[:topk])", "return order[:topk]")]),
    ("clustered decode takes the previous chunk", PY,
     [("_, s0, n = chunks[int(x)]", "_, s0, n = chunks[int(x) - 1]")]),
    ("matrix attention uses the next row's query block", PY,
     [("tq = pp // block", "tq = np.minimum((pp + 1) // block, pp.max() // block)")]),
    ("matrix attention window one key wider", PY,
     [("visible &= keys[None, :] > i[:, None] - window", "visible &= keys[None, :] >= i[:, None] - window")]),
    ("matrix attention without the scale", PY,
     [("s = (qd @ kb[keys].double().T) * sc", "s = (qd @ kb[keys].double().T)")]),
    ("matrix attention not normalised", PY,
     [("o = (p @ vb[keys].double()) / p.sum(dim=1, keepdim=True)", "o = (p @ vb[keys].double())")]),
    ("matrix attention excludes the diagonal", PY,
     [("visible = keys[None, :] <= i[:, None]", "visible = keys[None, :] < i[:, None]")]),
]

# The child loads the mutated package under the name `oracle` before pytest
# imports the pins, so every `import oracle` there resolves to the copy.
_CHILD = r"""
import importlib.util, sys
pkg = sys.argv[1]
spec = importlib.util.spec_from_file_location("oracle", pkg + "/__init__.py", submodule_search_locations=[pkg])
mod = importlib.util.module_from_spec(spec)
sys.modules["oracle"] = mod
spec.loader.exec_module(mod)
mod.build()  # compiles the copy's oracle.cpp unless its library was copied in
import pytest
sys.exit(pytest.main(["-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu", sys.argv[2]]))
"""


def _write_mutant(base: str, index: int, file: str, edits) -> str:
    pkg = os.path.join(base, f"m{index:02d}", "oracle")
    os.makedirs(pkg)
    for name in (CPP, PY):
        shutil.copyfile(os.path.join(ORACLE_DIR, name), os.path.join(pkg, name))
    path = os.path.join(pkg, file)
    with open(path) as f:
        text = f.read()
    for old, new in edits:
        assert text.count(old) == 1, f"mutation text not found exactly once: {old!r}"
        text = text.replace(old, new)
    with open(path, "w") as f:
        f.write(text)
    if file == PY:  # the C++ is unchanged: reuse the built library (copied last, so it is not older)
        shutil.copyfile(oracle_lib(), os.path.join(pkg, os.path.basename(oracle_lib())))
    return pkg


def oracle_lib() -> str:
    import oracle

    return oracle.build()


def _run(pkg: str) -> tuple[int, str]:
    threads = {k: "1" for k in ("ORACLE_THREADS", "OMP_NUM_THREADS", "MKL_NUM_THREADS", "OPENBLAS_NUM_THREADS")}
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", **threads)
    p = subprocess.run([sys.executable, "-c", _CHILD, pkg, PINS], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return p.returncode, (p.stdout + p.stderr)[-1500:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    base = str(tmp_path_factory.mktemp("oracle_mutants"))
    pkgs = [_write_mutant(base, i, f, e) for i, (_, f, e) in enumerate(MUTANTS)]
    workers = max(1, min(16, os.cpu_count() or 1))
    with ThreadPoolExecutor(workers) as pool:
        return list(pool.map(_run, pkgs))


def test_unmutated_copy_passes(tmp_path):
    """The copying and loading machinery itself leaves the pins green."""
    pkg = _write_mutant(str(tmp_path), 0, PY, [])
    rc, out = _run(pkg)
    assert rc == 0, out


@pytest.mark.parametrize("index", range(len(MUTANTS)), ids=[m[0].replace(" ", "-") for m in MUTANTS])
def test_mutant_fails_the_pins(outcomes, index):
    rc, out = outcomes[index]
    assert rc != 0, f"mutant survived the pins: {MUTANTS[index][0]}"
    assert rc == 1, f"mutant child did not end in a test failure (rc {rc}):\n{out}"
