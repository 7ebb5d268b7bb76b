"""Mutation sweep of the library's host-side checks.

Each entry below is one plausible mistake in `csrc/qlora_nf4.cu` (a dropped shape, alignment
or argument check, a short workspace, a wrong scratch limit, a changed codebook derivation).
The sweep copies the repository into a temporary directory, applies one mistake, rebuilds the
library there with nvcc (no GPU needed) and runs the CPU ABI tests (`tests/test_abi.py`);
a mistake that no test catches "survives". Run from the repository root:

    python tests/host_check_mutation_sweep.py             # every mistake
    python tests/host_check_mutation_sweep.py H3_r_mod16  # some of them

Expected: every mistake is caught except H13 (the INT4 zero code), which the ABI does not
expose; the GPU codec tests catch it (an all-zero block under the INT4 codebook).
"""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
F = os.path.join("bit_quantized_lora_03_b200", "csrc", "qlora_nf4.cu")
MUTS = {
 "H1_h_mod64": [("q->in_features < 64 || q->in_features % 64 != 0", "q->in_features < 64")],
 "H2_s2_align": [("!aligned16(q->absmax_q8) || !aligned16(q->absmax_s2))", "!aligned16(q->absmax_q8))")],
 "H3_r_mod16": [("r > 256 || r % 16 != 0", "r > 256")],
 "H4_o_mod64": [("o < 64 || o % 64 != 0", "o < 64")],
 "H5_fwd_ws": [("ws_bytes < qlora_fwd_workspace_bytes(t, W->in_features, W->out_features, r))\n    return QLORA_ERR_WORKSPACE;\n  return fwd_core(",
                "ws_bytes < 1)\n    return QLORA_ERR_WORKSPACE;\n  return fwd_core(")],
 "H6_bwd_ws_half": [("  return 2 * lora_region_bytes(t, r);\n}", "  return lora_region_bytes(t, r);\n}")],
 "H7_noalloc_limit": [("if (need > QLORA_STATIC_SCRATCH_BYTES) return QLORA_ERR_SCRATCH_LIMIT;",
                       "if (need > 4 * static_cast<size_t>(QLORA_STATIC_SCRATCH_BYTES)) return QLORA_ERR_SCRATCH_LIMIT;")],
 "H8_adamw_eps": [("  if (!param || !grad || !m || !v || n <= 0 || n % 4 != 0 || step < 1) return QLORA_ERR_INVALID_ARG;\n  if (!std::isfinite(lr) || !std::isfinite(eps) || !std::isfinite(weight_decay) || eps <= 0.f ||",
                   "  if (!param || !grad || !m || !v || n <= 0 || n % 4 != 0 || step < 1) return QLORA_ERR_INVALID_ARG;\n  if (!std::isfinite(lr) || !std::isfinite(eps) || !std::isfinite(weight_decay) ||")],
 "H9_multi_mod4": [("counts[k] <= 0 || counts[k] % 4 != 0)", "counts[k] <= 0)")],
 "H10_drop_p1": [("p >= 0.0f && p < 1.0f", "p >= 0.0f && p <= 1.0f")],
 "H11_fwd_nan_s": [("if (!X || !L1 || !L2 || !Y) return QLORA_ERR_INVALID_ARG;\n  if (!std::isfinite(s)) return QLORA_ERR_INVALID_ARG;",
                    "if (!X || !L1 || !L2 || !Y) return QLORA_ERR_INVALID_ARG;")],
 "H12_newton_iters": [("for (int it = 0; it < 500; ++it) {", "for (int it = 0; it < 3; ++it) {")],
 "H13_int4_zero": [("        return finish(w, 8);", "        return finish(w, 7);")],
 "H14_delta": [("const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));", "const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 33.0));")],
}


def _copy_tree(d):
    skip = shutil.ignore_patterns("__pycache__", "*.so")
    for sub in ("oracle", "tests", "include", "bit_quantized_lora_03_b200"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(d, sub), ignore=skip)
    for f in ("pytest.ini", "bench.py"):
        shutil.copy2(os.path.join(ROOT, f), os.path.join(d, f))


def run(name, tmp):
    d = os.path.join(tmp, name)
    _copy_tree(d)
    path = os.path.join(d, F)
    text = open(path).read()
    for old, new in MUTS.get(name, []):
        if text.count(old) != 1:
            return name, f"PATTERN NOT FOUND ({old[:50]!r})"
        text = text.replace(old, new)
    with open(path, "w") as f:
        f.write(text)
    b = subprocess.run([sys.executable, "-c",
                        "from bit_quantized_lora_03_b200 import build; build.build(force=True)"],
                       cwd=d, capture_output=True, text=True)
    if b.returncode:
        return name, "BUILD FAILED " + b.stderr[-300:]
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_abi.py", "-q", "-x",
                        "-p", "no:cacheprovider"], cwd=d, capture_output=True, text=True,
                       timeout=900)
    failed = [line for line in r.stdout.splitlines() if line.startswith("FAILED")]
    outcome = "caught" if r.returncode else "SURVIVED"
    return name, outcome + (" by " + failed[0].split()[1] if failed else "")


def main():
    names = sys.argv[1:] or (["baseline"] + list(MUTS))
    with tempfile.TemporaryDirectory() as tmp, ThreadPoolExecutor(4) as ex:
        results = list(ex.map(lambda n: run(n, tmp), names))
    for name, res in results:
        print(f"{name}: {res}", flush=True)
    caught = sum(1 for n, r in results if n != "baseline" and r.startswith("caught"))
    print(f"{caught} of {sum(1 for n, _ in results if n != 'baseline')} caught")


if __name__ == "__main__":
    main()
