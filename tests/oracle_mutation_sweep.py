"""Mutation sweep of the oracle's CPU pins.

Each entry below is one plausible mistake in `oracle/nf4_oracle.py` (a tie rule, a rounding
mode, a multiply order, a constant, a sign, a layout). The sweep copies the repository's
oracle, tests, package and library into a temporary directory, applies one mistake, and runs
the CPU oracle tests there; a mistake that no test catches "survives". Run from the
repository root, with the library built (the ABI tests load it):

    python tests/oracle_mutation_sweep.py            # every mistake
    python tests/oracle_mutation_sweep.py M1_tie_ge  # some of them

Expected: every mistake is caught except three that change no tested result. Thresholds summed
in fp32 give the same values as in double for all three codebooks. A tighter merge error bound
still holds on the tested inputs. A signed absmax code clamped at -qmax - 1 instead of -qmax
never reaches the clamp, since |x| / scale <= qmax.
"""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join("oracle", "nf4_oracle.py")
TESTS = ["tests/test_oracle_adamw.py", "tests/test_oracle_codebook.py",
         "tests/test_oracle_codebooks.py", "tests/test_oracle_dropout.py",
         "tests/test_oracle_merge.py", "tests/test_oracle_products.py",
         "tests/test_oracle_quantize.py", "tests/test_oracle_scale_formats.py",
         "tests/test_abi.py", "tests/test_dp_gloo.py"]

MUTS = {
 "M1_tie_ge": [("codes += (xhat > mid[i]).astype(np.uint8)", "codes += (xhat >= mid[i]).astype(np.uint8)")],
 "M2_q8_half_away": [("np.clip(np.rint(ratio), 0, Q8_MAX)", "np.clip(np.floor(ratio + 0.5), 0, Q8_MAX)")],
 "M3_s2_div256": [("scale = np.float32(c2 / np.float32(Q8_MAX))", "scale = np.float32(c2 / np.float32(Q8_MAX + 1))")],
 "M4_nibble_swap_both": [("return ((c[:, 0] << 4) | c[:, 1]).astype(np.uint8)", "return ((c[:, 1] << 4) | c[:, 0]).astype(np.uint8)"),
                         ("out[0::2] = p >> 4\n    out[1::2] = p & 0xF", "out[1::2] = p >> 4\n    out[0::2] = p & 0xF")],
 "M5_deq_order": [("k = block_scales(packed.absmax_q8, packed.absmax_s2)\n    w = (q[codes] * k[:, None]).astype(np.float32)",
                   "g = np.arange(codes.shape[0]) // GROUP\n    w = ((q[codes] * packed.absmax_q8.astype(np.float32)[:, None]).astype(np.float32) * np.asarray(packed.absmax_s2, np.float32)[g][:, None]).astype(np.float32)")],
 "M6_bf16_trunc": [("rounded = ((u + 0x7FFF + lsb) >> 16)", "rounded = ((u + 0 * lsb) >> 16)")],
 "M7_bf16_ties_away": [("rounded = ((u + 0x7FFF + lsb) >> 16)", "rounded = ((u + 0x8000 + 0 * lsb) >> 16)")],
 "M8_group128": [("GROUP = 256 ", "GROUP = 128 ")],
 "M9_delta31": [("(1.0 - 1.0 / 30.0)", "(1.0 - 1.0 / 31.0)")],
 "M10_neg_steps8": [("neg = [delta + i * (0.5 - delta) / 7.0 for i in range(7)]", "neg = [delta + i * (0.5 - delta) / 8.0 for i in range(7)]")],
 "M11_mid_fp32": [("return ((q64[:-1] + q64[1:]) / 2.0).astype(np.float32)", "return ((q[:-1] + q[1:]) * np.float32(0.5)).astype(np.float32)")],
 "M12_fwd_no_s": [("Y = X @ Wt.T + s * (T @ L2)", "Y = X @ Wt.T + (T @ L2)")],
 "M13_dx_sign": [("dX = dY @ Wt + s * (U @ L1.T)", "dX = dY @ Wt - s * (U @ L1.T)")],
 "M14_dl2_no_s": [("dL2 = s * ((X @ L1).T @ dY)", "dL2 = ((X @ L1).T @ dY)")],
 "M15_adam_no_bc1": [("mhat = m / (1.0 - beta1 ** step)", "mhat = m")],
 "M16_adam_decay": [("p = p * (1.0 - lr * weight_decay)", "p = p * (1.0 - weight_decay)")],
 "M17_philox_w1": [("PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE85", "PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE86")],
 "M18_drop_gt": [("return (draw.astype(np.int64) >= thr).reshape(t, h)", "return (draw.astype(np.int64) > thr).reshape(t, h)")],
 "M19_drop_ctr_hi": [("ctr[:, 1] = groups >> np.uint64(32)", "ctr[:, 1] = groups & _MASK32")],
 "M20_merge_no_s": [("return Wt + s * (L2.T @ L1.T)", "return Wt + (L2.T @ L1.T)")],
 "M21_zero_code8": [("ZERO_CODE = 7 ", "ZERO_CODE = 8 ")],
 "M22_absmax_signed": [("    return np.max(np.abs(w), axis=1)\n", "    return np.max(w, axis=1)\n")],
 "M23_q8_clip254": [("np.clip(np.rint(ratio), 0, Q8_MAX)", "np.clip(np.rint(ratio), 0, Q8_MAX - 1)")],
 "M24_drop_scale": [("return 1.0 / (1.0 - float(np.float32(p)))", "return 1.0 / (1.0 - 0.5 * float(np.float32(p)))")],
 "M25_fp4_mag": [("mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]", "mags = [0.0, 0.5, 1.0, 1.5, 2.0, 2.5, 4.0, 6.0]")],
 "M26_philox_9rounds": [("for rnd in range(10):", "for rnd in range(9):")],
 "M27_dl1_transpose": [("dL1 = s * (X.T @ U)", "dL1 = s * (X.T @ (dY @ L2.T[:, ::-1]))")],
 "M28_adam_eps_inside": [("return p - lr * mhat / (np.sqrt(vhat) + eps), m, v", "return p - lr * mhat / np.sqrt(vhat + eps), m, v")],
}

MUTS.update({
 "N1_e4m3_sub": [("mag = np.where(e == 0, m * 2.0 ** -9,", "mag = np.where(e == 0, m * 2.0 ** -10,")],
 "N2_e4m3_bias": [("(1.0 + m / 8.0) * np.exp2(e - 7.0)", "(1.0 + m / 8.0) * np.exp2(e - 8.0)")],
 "N3_e4m3_tie_odd": [("np.where(lo % 2 == 0, lo, hi)", "np.where(lo % 2 == 1, lo, hi)")],
 "N4_e4m3_max": [("E4M3_MAX = 448.0", "E4M3_MAX = 480.0")],
 "N5_s8_qmax": [("absmax_int_quantize(seg, 127, signed=True)", "absmax_int_quantize(seg, 126, signed=True)")],
 "N7_fmt_order": [("k = (scale_code_values(packed.absmax_q8, fmt) *\n         np.asarray(packed.absmax_s2, dtype=np.float32)[g]).astype(np.float32)\n    w = (q[codes] * k[:, None]).astype(np.float32)",
                   "w = ((q[codes] * scale_code_values(packed.absmax_q8, fmt)[:, None]).astype(np.float32) * np.asarray(packed.absmax_s2, dtype=np.float32)[g][:, None]).astype(np.float32)")],
 "N8_philox_key_swap": [("words = philox4x32_10(ctr, (seed & 0xFFFFFFFF, seed >> 32))", "words = philox4x32_10(ctr, (seed >> 32, seed & 0xFFFFFFFF))")],
 "N9_mask_word_rev": [("(e & np.uint64(3)).astype(np.int64)]", "(np.uint64(3) - (e & np.uint64(3))).astype(np.int64)]")],
 "N10_fwd_sT_no_s": [("    return Y, s * T\n", "    return Y, T\n")],
 "N11_bwd_sU_no_s": [("return dX, dL1, dL2, s * U", "return dX, dL1, dL2, U")],
 "N12_fwd_rows_2s": [("Y, _ = qlora_linear_fwd(_f64(X)[rows], Wdq, L1, L2, s)", "Y, _ = qlora_linear_fwd(_f64(X)[rows], Wdq, L1, L2, 2 * s)")],
 "N13_dx_rows_no_s": [("return dY @ Wt + s * ((dY @ L2.T) @ L1.T)", "return dY @ Wt + ((dY @ L2.T) @ L1.T)")],
 "N14_merge_bound_tight": [("return 2.0 * (r + 2) * 2.0 ** -24 * mag", "return 0.25 * (r + 2) * 2.0 ** -24 * mag")],
 "N15_adam_v_lin": [("v = beta2 * v + (1.0 - beta2) * g * g", "v = beta2 * v + (1.0 - beta2) * np.abs(g)")],
 "N16_block_scale_group": [("    g = np.arange(q8.size) // GROUP\n", "    g = np.arange(q8.size) // (GROUP // 2)\n")],
 "N17_packed_bytes_floor": [("return n // 2 + nb + 4 * ((nb + GROUP - 1) // GROUP)", "return n // 2 + nb + 4 * (nb // GROUP)")],
 "N18_bits_255": [("return 8.0 / BLOCK + 32.0 / (BLOCK * GROUP)", "return 8.0 / BLOCK + 32.0 / (BLOCK * 255)")],
 "N19_dq_global_max": [("        seg = c1[g * GROUP:(g + 1) * GROUP]\n        c2 = np.float32(np.max(seg))\n        scale = np.float32(c2 / np.float32(Q8_MAX))",
                        "        seg = c1[g * GROUP:(g + 1) * GROUP]\n        c2 = np.float32(np.max(c1))\n        scale = np.float32(c2 / np.float32(Q8_MAX))")],
 "N23_int4_range": [("for k in range(-8, 8)], dtype=np.float64)", "for k in range(-7, 9)], dtype=np.float64)")],
 "N24_drop_dx_no_mask": [("dX = dY @ Wt + M * (s * (U @ L1.T))", "dX = dY @ Wt + (s * (U @ L1.T))")],
 "N25_drop_dl2_plain_x": [("dL2 = s * ((Xd @ L1).T @ dY)\n    return dX, dL1, dL2\n", "dL2 = s * ((X @ L1).T @ dY)\n    return dX, dL1, dL2\n")],
 "N26_dq_zero_group_q8": [("        if scale == 0.0:\n            continue\n        ratio", "        if scale == 0.0:\n            q8[g * GROUP:(g + 1) * GROUP] = 1\n            continue\n        ratio")],
})


MUTS.update({
 "P1_quantile_swap": [("        if normal_cdf(mid) < p:", "        if normal_cdf(mid) > p:")],
 "P2_e4m3_sat": [("hi = np.clip(np.searchsorted(vals, x, side=\"left\"), 0, 0x7E)", "hi = np.clip(np.searchsorted(vals, x, side=\"left\"), 0, 0x7D)")],
 "P3_int_signed_lo": [("lo = -qmax if signed else 0", "lo = -qmax - 1 if signed else 0")],
 "P4_merge_bound_loose": [("return 2.0 * (r + 2) * 2.0 ** -24 * mag", "return 400.0 * (r + 2) * 2.0 ** -24 * mag")],
 "P5_rms_as_mean_abs": [("float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0", "float(np.mean(np.abs(ref))) if ref.size else 0.0")],
 "P6_bits_no_dq": [("        return 32.0 / BLOCK", "        return 16.0 / BLOCK")],
 "P7_storage_div4": [("return n_params * bits / 8.0", "return n_params * bits / 4.0")],
 "P8_drop_fwd_no_scale": [("Xd = X * np.asarray(keep, dtype=np.float64) * dropout_scale(p)", "Xd = X * np.asarray(keep, dtype=np.float64)")],
 "P9_bf16_nan_quiet": [("rounded = np.where(nan, ((u >> 16) | 0x40).astype(np.uint16), rounded)", "rounded = np.where(nan, (u >> 16).astype(np.uint16), rounded)")],
})


def _copy_tree(dst):
    skip = shutil.ignore_patterns("__pycache__")
    for sub in ("oracle", "tests", "include", "bit_quantized_lora_03_b200"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(dst, sub), ignore=skip)
    for f in ("pytest.ini", "bench.py"):
        shutil.copy2(os.path.join(ROOT, f), os.path.join(dst, f))


def run(name, tmp):
    d = os.path.join(tmp, name)
    _copy_tree(d)
    path = os.path.join(d, ORACLE)
    text = open(path).read()
    for old, new in MUTS.get(name, []):
        if text.count(old) != 1:
            return name, f"PATTERN NOT FOUND ({old[:40]!r})"
        text = text.replace(old, new)
    with open(path, "w") as f:
        f.write(text)
    env = dict(os.environ, OMP_NUM_THREADS="2", OPENBLAS_NUM_THREADS="2", MKL_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", *TESTS, "-q", "-x", "-m", "not gpu",
                        "-p", "no:cacheprovider"], cwd=d, env=env, capture_output=True,
                       text=True, timeout=900)
    failed = [line for line in r.stdout.splitlines() if line.startswith("FAILED")]
    outcome = "caught" if r.returncode != 0 else "SURVIVED"
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
