"""Mutation check of the oracle's pins (test infrastructure; run by hand:
``python tests/oracle_mutants.py [--scratch DIR] [index ...]``, about four
minutes on CPU; scratch copies go to DIR, else the system's temporary folder).

Each entry plants one plausible mistake (a wrong exponent bias, a dropped term,
a swapped gate/up, a transposed or reversed scale index, a wrong rounding rule,
an unstable grouping ...) in a scratch copy of ``oracle/`` and runs the CPU pin
tests against it.  A mistake that no pin catches is reported.  Entries marked
``equivalent`` compute the same function as the oracle on every input (the
reason is given), so no test can catch them; they stay in the list to show
that they were considered.  Nothing outside the scratch copy is modified.
"""
import os
import shutil
import subprocess
import sys
import tempfile

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
F, L = "oracle/formats.py", "oracle/layer.py"
PIN_TESTS = ["tests/test_oracle_formats.py", "tests/test_oracle_layer.py",
             "tests/test_oracle_bf16.py", "tests/test_oracle_route_property.py",
             "tests/test_oracle_requant_property.py", "tests/test_golden_params.py",
             "tests/test_workload_recipe.py"]
# What a scratch copy needs for the pin tests to import and run.
COPIED = ("oracle", "tests", "workloads", "moe_expert_ffn_permute_b200")

_TAIL = ("                out[t] += w[t, j] * y[t * k + j]\n    if keep:\n        inter.update("
         "counts=counts, offsets=offsets, perm=perm, inv=inv, y=y)\n        return out, inter\n"
         "    return out\n\n\ndef layer_bf16")

# (file, text, replacement, note); note starting with "equivalent:" gives the reason.
MUTANTS = [
    (F, "np.exp2(exp - 7.0)", "np.exp2(exp - 8.0)", "E4M3 exponent bias"),
    (F, "sub = (man / 8.0) * np.exp2(-6.0)", "sub = (man / 8.0) * np.exp2(-7.0)",
     "E4M3 subnormal scale"),
    (F, "(exp == 15) & (man == 7)", "(exp == 15) & (man == 6)", "E4M3 NaN code"),
    (F, "(codes[hi] % 2 == 0)", "(codes[hi] % 2 == 1)", "E4M3 ties to odd"),
    (F, "(d_hi < d_lo) |", "(d_hi <= d_lo) |", "E4M3 ties always up"),
    (F, "a_sat = np.minimum(a, E4M3_MAX)", "a_sat = np.minimum(a, 480.0)",
     "equivalent: the table search clamps to the last finite code (448) anyway"),
    (F, "_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])",
     "_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 4.0, 3.0, 6.0])", "E2M1 table order"),
    (F, "np.stack([lo, hi]", "np.stack([hi, lo]", "E2M1 nibble order"),
    (F, "np.exp2(b - 127.0)", "np.exp2(b - 128.0)", "UE8M0 bias"),
    (F, "np.where(b == 255, np.nan, val)", "val", "UE8M0 NaN code"),
    (F, "r = np.rint(a / q) * q", "r = np.floor(a / q + 0.5) * q", "BF16 ties away"),
    (F, "q = np.ldexp(1.0, (E - 7).astype(np.int64))", "q = np.ldexp(1.0, (E - 8).astype(np.int64))",
     "BF16 mantissa width"),
    (F, "E = np.maximum(ex.astype(np.int64) - 1, -126)", "E = ex.astype(np.int64) - 1",
     "BF16 subnormal spacing"),
    (F, "c = np.where(np.signbit(v), c | 0x80, c)", "c = np.where(v < 0, c | 0x80, c)",
     "E4M3 sign of -0"),
    (L, "    return v * np.repeat(s, BLOCK, axis=1)\n\n\ndef dequant_w_fp8",
     "    return v * np.tile(s, (1, BLOCK))\n\n\ndef dequant_w_fp8", "activation 1x128 block index"),
    (L, "s = np.repeat(np.repeat(s, BLOCK, axis=0), BLOCK, axis=1)",
     "s = np.repeat(np.repeat(s[::-1], BLOCK, axis=0), BLOCK, axis=1)", "weight scale row blocks"),
    (L, "s = np.repeat(np.repeat(s, BLOCK, axis=0), BLOCK, axis=1)",
     "s = np.repeat(np.repeat(s[:, ::-1], BLOCK, axis=0), BLOCK, axis=1)",
     "weight scale column blocks"),
    (L, "return v * np.repeat(s, FP4_BLOCK, axis=1)", "return v * np.tile(s, (1, FP4_BLOCK))",
     "FP4 1x32 block index"),
    (L, "        a = swiglu(h[:, :I], h[:, I:], alpha, up_bias, limit)   # [n_e, I]\n        q, sf",
     "        a = swiglu(h[:, I:], h[:, :I], alpha, up_bias, limit)   # [n_e, I]\n        q, sf",
     "gate / up swapped"),
    (L, "return gc * sigmoid(alpha * gc) * (uc + up_bias)",
     "return gc * sigmoid(gc) * (uc + up_bias)", "alpha dropped"),
    (L, "return gc * sigmoid(alpha * gc) * (uc + up_bias)",
     "return gc * sigmoid(alpha * gc) * (uc - up_bias)", "up_bias sign"),
    (L, "return gc * sigmoid(alpha * gc) * (uc + up_bias)",
     "return gc * sigmoid(alpha * gc) * uc + up_bias", "up_bias outside the product"),
    (L, "return gc * sigmoid(alpha * gc) * (uc + up_bias)",
     "return g * sigmoid(alpha * gc) * (uc + up_bias)", "unclamped gate factor"),
    (L, "uc = np.clip(u, -limit, limit)", "uc = np.minimum(u, limit)", "up clamped one-sided"),
    (L, "gc = np.minimum(g, limit)", "gc = np.clip(g, -limit, limit)", "gate clamped two-sided"),
    (L, "return 1.0 / (1.0 + np.exp(-z))", "return 1.0 / (1.0 + np.exp(z))", "sigmoid sign"),
    (L, "sf[r, b] = n + 127", "sf[r, b] = n + 128", "requant scale byte bias"),
    (L, "AMAX_FLOOR = 1e-4 ", "AMAX_FLOOR = 1e-3 ", "requant amax floor"),
    (L, "    while a > E4M3_MAX * 2.0 ** n:          # repair",
     "    while False:          # repair", "requant exponent: no upward repair"),
    (L, "    while a <= E4M3_MAX * 2.0 ** (n - 1):", "    while False:",
     "equivalent: a <= 448*2^m implies a/448 <= 2^m and log2 <= m, so the ceiling never "
     "overshoots and the downward repair never runs"),
    (L, "n = math.ceil(math.log2(a / E4M3_MAX))", "n = math.floor(math.log2(a / E4M3_MAX))",
     "equivalent: the upward repair loop moves any low first guess to the smallest n"),
    (L, "encode_e4m3_rne_satfinite(blk / 2.0 ** n)", "encode_e4m3_rne_satfinite(blk * 2.0 ** n)",
     "requant multiplies by 2^n instead of dividing"),
    (L, "n = ue8m0_exponent_for(np.max(np.abs(blk)))", "n = ue8m0_exponent_for(np.max(blk))",
     "requant max instead of amax"),
    (L, "slots = np.nonzero(flat == e)[0]           # ascending",
     "slots = np.nonzero(flat == e)[0][::-1]           # ascending", "unstable grouping"),
    (L, "offsets[1:] = np.cumsum(counts)", "offsets[1:] = np.cumsum(counts[::-1])[::-1]",
     "offsets scanned the wrong way"),
    (L, "        tokens = slots // k\n        W1", "        tokens = slots % T\n        W1",
     "slot -> token index"),
    (L, _TAIL, _TAIL.replace("out[t] += w[t, j]", "out[t] = w[t, j]"),
     "combine overwrites instead of summing"),
    (L, _TAIL, _TAIL.replace("y[t * k + j]", "y[j * T + t]"), "combine reads y in the wrong order"),
    (L, _TAIL, _TAIL.replace("w[t, j] *", "w[t, k - 1 - j] *"), "combine pairs the wrong weight"),
    (L, "        ah = dequant_act(q, sf)\n", "        ah = a\n", "requant skipped"),
    (L, "    xh = dequant_act(x, x_scales)\n", "    xh = _E4M3[np.asarray(x, dtype=np.uint8)]\n",
     "x scales dropped"),
    (L, "        y[slots] = decode_bf16(ab) @ decode_bf16(w2[e]).T",
     "        y[slots] = a @ decode_bf16(w2[e]).T", "BF16 activation rounding skipped"),
    (L, "        a = swiglu(h[:, :I], h[:, I:], alpha, up_bias, limit)   # [n_e, I]\n        ab",
     "        a = swiglu(h[:, I:], h[:, :I], alpha, up_bias, limit)   # [n_e, I]\n        ab",
     "BF16 gate / up swapped"),
    (L, "        h = xh[tokens] @ decode_bf16(w1[e]).T",
     "        h = xh[tokens] @ decode_bf16(w1[e][::-1]).T", "BF16 W1 rows reversed"),
    (L, "nib = byte & 0xF if c % 2 == 0 else byte >> 4",
     "nib = byte >> 4 if c % 2 == 0 else byte & 0xF", "brute-force tier nibble order"),
    (L, "    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)",
     "    return s * (1.0 + m / 8.0) * 2.0 ** (e - 8)", "brute-force tier E4M3 bias"),
    (L, "        if best is None or d < best or (d == best and code % 2 == 0):",
     "        if best is None or d < best:", "brute-force tier E4M3 ties"),
    (L, "r = round(abs(v) / 2.0 ** (e - 7)) * 2.0 ** (e - 7)",
     "r = math.floor(abs(v) / 2.0 ** (e - 7) + 0.5) * 2.0 ** (e - 7)",
     "brute-force tier BF16 ties"),
]


def _scratch_copy(scratch_root):
    scratch = tempfile.mkdtemp(prefix="oracle_mutant_", dir=scratch_root)
    for d in COPIED:
        shutil.copytree(os.path.join(ROOT, d), os.path.join(scratch, d),
                        ignore=shutil.ignore_patterns("*.so", "_build", "__pycache__"))
    return scratch


def _pins(scratch):
    return subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                           *PIN_TESTS], cwd=scratch, capture_output=True, text=True)


def run(selected=None, scratch_root=None):
    # The unmutated copy must pass, or every mutant would look caught.
    scratch = _scratch_copy(scratch_root)
    try:
        base = _pins(scratch)
    finally:
        shutil.rmtree(scratch, ignore_errors=True)
    if base.returncode != 0:
        print("the pins fail on an unmutated copy; nothing to check:\n" + base.stdout[-2000:])
        return False
    survivors, missing = [], []
    for i, (rel, text, repl, note) in enumerate(MUTANTS):
        if selected and i not in selected:
            continue
        scratch = _scratch_copy(scratch_root)
        try:
            path = os.path.join(scratch, rel)
            with open(path) as f:
                src = f.read()
            if text not in src:
                missing.append(i)
                print(f"[{i:2d}] text not found ({note})")
                continue
            with open(path, "w") as f:
                f.write(src.replace(text, repl, 1))
            r = _pins(scratch)
        finally:
            shutil.rmtree(scratch, ignore_errors=True)
        caught = r.returncode != 0
        equivalent = note.startswith("equivalent:")
        status = "caught" if caught else ("equivalent" if equivalent else "SURVIVED")
        print(f"[{i:2d}] {status:10s} {note}")
        if not caught and not equivalent:
            survivors.append(i)
    print(f"{len(survivors)} non-equivalent mutants survived: {survivors}; "
          f"{len(missing)} not applied: {missing}")
    return not survivors and not missing


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser()
    ap.add_argument("--scratch", default=None, help="folder for the scratch copies")
    ap.add_argument("index", nargs="*", type=int, help="run only these mutants")
    a = ap.parse_args()
    sys.exit(0 if run(a.index, a.scratch) else 1)
