"""The oracle's pins catch plausible mistakes.

Each mutant below plants one mistake in a copy of the oracle's C source: a
wrong rounding, a reciprocal in place of the division, a transposed
operand, a dropped term, a different order of the epilogue's roundings, a
wrong tile or swizzle offset, and so on.  The copy is compiled like the
oracle and the pins of that step run against it (in a subprocess that loads
it through W8A8_ORACLE_LIB).  Every mutant must make at least one pin fail,
and the unaltered source, built and run the same way, must pass them all.
Mutants that cannot change any result (the clamp of the dynamic codes,
which |x / s| <= 127 never reaches) are not listed.
"""
import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

from oracle import build as oracle_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "w8a8_oracle.c")

Q, G, E, P, L, N = ("tests/test_oracle_quant.py", "tests/test_oracle_gemm.py",
                    "tests/test_oracle_epilogue.py", "tests/test_oracle_pack.py",
                    "tests/test_oracle_gelu.py", "tests/test_oracle_next.py")

# (name, text in the oracle source (exactly one occurrence), replacement, pin files)
MUTANTS = [
    ("quant rounds ties away from zero",
     "      float r = nearbyintf(v);          /* default mode: nearest, ties even */",
     "      float r = roundf(v);", [Q]),
    ("quant multiplies by the reciprocal",
     "      float v = bf16_to_f32(xr[k]) / s; /* IEEE fp32 division */",
     "      float v = bf16_to_f32(xr[k]) * (1.0f / s);", [Q]),
    ("quant scale amax / 128",
     "    float s = amax / 127.0f;",
     "    float s = amax / 128.0f;", [Q]),
    ("quant row maximum without the absolute value",
     "      float a = fabsf(bf16_to_f32(xr[k]));",
     "      float a = bf16_to_f32(xr[k]);", [Q]),
    ("quant zero row gets scale 1",
     "      a_scale[m] = 0.0f;\n      for (int64_t k = 0; k < K; ++k) qr[k] = 0;",
     "      a_scale[m] = 1.0f;\n      for (int64_t k = 0; k < K; ++k) qr[k] = 0;", [Q]),
    ("quant row maximum skips the last element",
     "    for (int64_t k = 0; k < K; ++k) {\n      float a = fabsf(bf16_to_f32(xr[k]));",
     "    for (int64_t k = 0; k + 1 < K; ++k) {\n      float a = fabsf(bf16_to_f32(xr[k]));", [Q]),
    ("gemm reads the weight transposed",
     "      const int8_t *wr = w + n * K;\n      int64_t s = 0;\n"
     "      for (int64_t k = 0; k < K; ++k) s += (int64_t)qr[k] * (int64_t)wr[k];",
     "      int64_t s = 0;\n"
     "      for (int64_t k = 0; k < K; ++k) s += (int64_t)qr[k] * (int64_t)w[k * N + n];", [G]),
    ("gemm accumulates in int32",
     "      const int8_t *wr = w + n * K;\n      int64_t s = 0;",
     "      const int8_t *wr = w + n * K;\n      int32_t s = 0;", [G]),
    ("gemm drops the overflow check",
     "      if (s > INT32_MAX || s < INT32_MIN) overflow = 1;\n      acc[m * N + n] = (int32_t)s;",
     "      acc[m * N + n] = (int32_t)s;", [G]),
    ("gemm drops the last k term",
     "      for (int64_t k = 0; k < K; ++k) s += (int64_t)qr[k] * (int64_t)wr[k];\n"
     "      if (s > INT32_MAX || s < INT32_MIN) overflow = 1;\n      acc[m * N + n]",
     "      for (int64_t k = 0; k + 1 < K; ++k) s += (int64_t)qr[k] * (int64_t)wr[k];\n"
     "      if (s > INT32_MAX || s < INT32_MIN) overflow = 1;\n      acc[m * N + n]", [G]),
    ("epilogue multiplies the two scales first",
     "  t = t * as;\n  t = t * ws;",
     "  t = t * (as * ws);", [E]),
    ("epilogue adds the bias before the weight scale",
     "  t = t * as;\n  t = t * ws;\n  if (bias) t = t + bf16_to_f32(bias[n]);",
     "  t = t * as;\n  if (bias) t = t + bf16_to_f32(bias[n]);\n  t = t * ws;", [E]),
    ("epilogue drops the bias",
     "  if (bias) t = t + bf16_to_f32(bias[n]);",
     "  (void)bias;", [E]),
    ("bf16 rounding ties away from zero",
     "  u += 0x7fffu + lsb;",
     "  u += 0x8000u + 0u * lsb;", [E]),
    ("repack swizzles with r mod 4",
     "(((c / 16) ^ (r % 8)) * 16)",
     "(((c / 16) ^ (r % 4)) * 16)", [P]),
    ("repack orders tiles k-major",
     "      int64_t tile = (nb * kblocks + kb) * 16384;",
     "      int64_t tile = (kb * (Np / 128) + nb) * 16384;", [P]),
    ("gelu cubic coefficient 0.04715",
     "0.044715 * v * v * v",
     "0.04715 * v * v * v", [L]),
    ("gelu sigmoid without the negative branch",
     "    double sig = u >= 0.0 ? 1.0 / (1.0 + e) : e / (1.0 + e);",
     "    double sig = 1.0 / (1.0 + e);", [L]),
    ("double to bf16 rounds twice (no round-to-odd)",
     "    u |= 1u;",
     "    u |= 0u;", [L, E]),
    ("int32 storage unbiased by 127",
     "(int8_t)((int)byte - 128)",
     "(int8_t)((int)byte - 127)", [N]),
    ("int32 storage bytes in reverse order",
     "(word >> (8 * (k % 4)))",
     "(word >> (8 * (3 - k % 4)))", [N]),
    ("static scale accepts a negative scale",
     "  const int usable = scale > 0.0f; /* false for NaN too */",
     "  const int usable = scale != 0.0f;", [N]),
    ("epilogue in double precision, one rounding at the end",
     "  float t = (float)acc; /* int32 -> fp32, nearest even */\n  t = t * as;\n  t = t * ws;\n"
     "  if (bias) t = t + bf16_to_f32(bias[n]);\n  return f32_to_bf16_rne(t);",
     "  double t = (double)acc * as * ws;\n"
     "  if (bias) t = t + bf16_to_f32(bias[n]);\n  return f64_to_bf16_rne(t);", [E]),
    ("layer ignores the row stride",
     "    rc = w8a8o_quant_act(x, M, K, ldx, q, as);",
     "    rc = w8a8o_quant_act(x, M, K, K, q, as);", [E]),
    ("sampled reads the weight row of the output row",
     "    const int8_t *wr = w + cols[i] * K;",
     "    const int8_t *wr = w + rows[i] * K;", [G]),
    ("sampled adds the bias of the row index",
     "w_scale[cols[i]], bias, cols[i]);",
     "w_scale[cols[i]], bias, rows[i]);", [G]),
    ("repack leaves the padding unzeroed",
     "  memset(packed, 0, (size_t)(Np * Kp));",
     "  memset(packed, 0x11, (size_t)(Np * Kp));", [P]),
    ("packed size rounds N up to 128",
     "  return ((N + 255) / 256 * 256) * ((K + 127) / 128 * 128);",
     "  return ((N + 127) / 128 * 128) * ((K + 127) / 128 * 128);", [P]),
    ("gelu multiplies the sigmoid by |x|",
     "    y[i] = f64_to_bf16_rne(v * sig);",
     "    y[i] = f64_to_bf16_rne(fabs(v) * sig);", [L]),
    ("static codes clamp below at -128",
     "      if (r < -127.0f) r = -127.0f;\n      q[m * K + k] = (int8_t)r;",
     "      if (r < -128.0f) r = -128.0f;\n      q[m * K + k] = (int8_t)r;", [N]),
    ("static scale reported for an unusable scale",
     "    if (a_scale_out) a_scale_out[m] = usable ? scale : 0.0f;",
     "    if (a_scale_out) a_scale_out[m] = scale;", [N]),
    ("static scale reads rows at the dense stride",
     "      float v = bf16_to_f32(x[m * ldx + k]) / scale;",
     "      float v = bf16_to_f32(x[m * K + k]) / scale;", [N]),
    ("round-to-odd without the truncation toward zero",
     "    if (fabs((double)f) > fabs(g)) f = nextafterf(f, 0.0f);\n",
     "", [L, E]),
    ("static codes clamp at 126",
     "      float v = bf16_to_f32(x[m * ldx + k]) / scale;\n      float r = nearbyintf(v);\n"
     "      if (r > 127.0f) r = 127.0f;",
     "      float v = bf16_to_f32(x[m * ldx + k]) / scale;\n      float r = nearbyintf(v);\n"
     "      if (r > 126.0f) r = 126.0f;", [N]),
]


def _run_pins(lib_path, files):
    env = dict(os.environ, W8A8_ORACLE_LIB=lib_path, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        *files], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return r.returncode, (r.stdout + r.stderr)[-1500:]


def _build_and_run(tmpdir, tag, text, files):
    src = os.path.join(tmpdir, f"oracle_{tag}.c")
    with open(src, "w") as f:
        f.write(text)
    lib = oracle_build.compile_lib(src, os.path.join(tmpdir, f"liboracle_{tag}.so"))
    return _run_pins(lib, files)


def test_mutants_are_listed_once_each():
    text = open(SRC).read()
    for name, old, new, files in MUTANTS:
        assert text.count(old) == 1, name
        assert old != new and files, name


def test_every_planted_mistake_fails_a_pin(tmp_path):
    text = open(SRC).read()
    all_files = sorted({f for m in MUTANTS for f in m[3]})
    jobs = {"control": (text, all_files)}
    for i, (name, old, new, files) in enumerate(MUTANTS):
        jobs[name] = (text.replace(old, new), files)
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with cf.ThreadPoolExecutor(workers) as ex:
        futs = {name: ex.submit(_build_and_run, str(tmp_path), f"m{i}", t, files)
                for i, (name, (t, files)) in enumerate(jobs.items())}
        results = {name: f.result() for name, f in futs.items()}
    rc, out = results.pop("control")
    assert rc == 0, "the unaltered oracle must pass its pins:\n" + out
    # pytest exits with 1 when tests ran and some failed; anything else
    # (collection error, crash) does not count as the pins catching it
    survivors = {name: (rc, out) for name, (rc, out) in results.items() if rc != 1}
    assert not survivors, "mistakes no pin catches: " + ", ".join(
        f"{n} (exit {rc})" for n, (rc, _) in survivors.items())
