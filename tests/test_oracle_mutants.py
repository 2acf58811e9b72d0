"""The oracle's pins catch plausible mistakes.  Each case below plants one mistake (a
dropped term, a wrong sign, index or constant, a transposed operand, a wrong rounding)
into a copy of the C oracle, builds it with the same compiler flags, and runs the
oracle's pin tests against that build (W8_ORACLE_LIB): at least one pin must fail.  The
unmodified copy, built the same way, must pass them all.  Mistakes in the Python front
end (the grouped GEMM) are planted in a copy of the package imported ahead of it.  The mistakes keep every
access in bounds, so a mutant fails by assertion, never by a crash."""
import concurrent.futures
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "w8_oracle.c")
PINS = {
    "formats": ["tests/test_oracle_formats.py"],
    "quant": ["tests/test_oracle_quant.py"],
    "gemm": ["tests/test_oracle_gemm.py", "tests/test_oracle_grouped.py"],
    "qknr": ["tests/test_oracle_qknr.py"],
    "sumsq": ["tests/test_oracle_sumsq.py"],
}

# (name, text of the oracle, planted replacement, pin files that must catch it)
MUTANTS = [
    ("bf16 output rounded twice (through fp32)",
     "r = nearbyint(a / step) * step;            /* default mode: ties to even */",
     "r = nearbyint((double)(float)a / step) * step;", "formats"),
    ("e4m3 ties away from zero",
     "double r = nearbyint(a / step) * step;         /* ties to even mantissa */",
     "double r = round(a / step) * step;", "formats"),
    ("e4m3 saturates to the NaN code",
     "if (a >= 448.0) return (uint8_t)(sign | 0x7E);",
     "if (a >= 448.0) return (uint8_t)(sign | 0x7F);", "formats"),
    ("e4m3 saturation only past the next binade",
     "if (a >= 448.0) return (uint8_t)(sign | 0x7E);",
     "if (a >= 512.0) return (uint8_t)(sign | 0x7E);", "formats"),
    ("e4m3 subnormal spacing wrong",
     "double step = (a < ldexp(1.0, -6)) ? ldexp(1.0, -9) : ldexp(1.0, ilogb(a) - 3);",
     "double step = (a < ldexp(1.0, -7)) ? ldexp(1.0, -10) : ldexp(1.0, ilogb(a) - 3);", "formats"),
    ("int8 truncates",
     "double r = nearbyint((double)v);",
     "double r = trunc((double)v);", "formats"),
    ("int8 clamps to -128",
     "if (r < -127.0) r = -127.0;",
     "if (r < -128.0) r = -128.0;", "formats"),
    ("fp8 scale constant 447",
     "float qmax = (qfmt == ORC_Q_FP8) ? 448.0f : 127.0f;",
     "float qmax = (qfmt == ORC_Q_FP8) ? 447.0f : 127.0f;", "quant"),
    ("codes by multiplying with 1/s",
     "float t = v[k] / s;                        /* true division, not v * (1/s) */",
     "float t = v[k] * (1.0f / s);", "quant"),
    ("UE8M0 rounds the exponent down",
     "int p = (f == 0.5f) ? e - 1 : e;               /* smallest 2^p >= r */",
     "int p = e - 1;", "formats"),
    ("all-zero group gets scale 0",
     "if (!(amax > 0.0f)) return 1.0f;",
     "if (!(amax > 0.0f)) return 0.0f;", "quant"),
    ("weight block scales transposed",
     "scale[(size_t)bn * nbk + bk] = s;",
     "scale[(size_t)bk * nbn + bn] = s;", "quant"),
    ("rms_norm without eps",
     "        float r = 1.0f / sqrtf(mean + eps);\n        for (int k = 0; k < H; ++k)",
     "        float r = 1.0f / sqrtf(mean);\n        for (int k = 0; k < H; ++k)", "quant"),
    ("rms_norm mean over H - 1",
     "float mean = ss / (float)H;",
     "float mean = ss / (float)(H - 1);", "quant"),
    ("sum of squares drops the sticky bits",
     "for (int i = lsb - 2; i >= 0 && !sticky; --i) sticky = ORC_SQ_BIT(i);",
     "for (int i = lsb - 2; i >= lsb - 2 && !sticky; --i) sticky = ORC_SQ_BIT(i);", "sumsq"),
    ("sum of squares rounds ties up",
     "if (half && (sticky || (mant & 1u))) ++mant;",
     "if (half) ++mant;", "sumsq"),
    ("sum of squares with the exponent of normal values off by one",
     "const int e = (E == 0) ? -133 : (int)E - 134;",
     "const int e = (E == 0) ? -133 : (int)E - 133;", "sumsq"),
    ("sum of squares keeps fp32 subnormals one bit too fine",
     "if (lsb < 117) lsb = 117;",
     "if (lsb < 116) lsb = 116;", "sumsq"),
    ("sum of squares loses the carry between words",
     "add = (add >> 32) + (t >> 32);",
     "add = (add >> 32);", "sumsq"),
    ("rms_norm without gamma",
     "y[(size_t)m * H + k] = (orc_bf16_to_float(xr[k]) * r) * orc_bf16_to_float(gamma[k]);",
     "y[(size_t)m * H + k] = orc_bf16_to_float(xr[k]) * r;", "quant"),
    ("silu sign flipped",
     "float den = 1.0f + orc_exp_f32(-g);",
     "float den = 1.0f + orc_exp_f32(g);", "quant"),
    ("gate and up swapped",
     "float g = orc_bf16_to_float(row[k]);\n            float u = orc_bf16_to_float(row[I + k]);",
     "float g = orc_bf16_to_float(row[I + k]);\n            float u = orc_bf16_to_float(row[k]);", "quant"),
    ("exp polynomial loses its 1/24 term",
     "p = fmaf(p, r, 0x1.555556p-5f);        /* 1/24 */",
     "p = fmaf(p, r, 0.0f);", "quant"),
    ("fp8 GEMM drops the weight scale",
     "                ref = acc * (double)sA[m] * (double)sW[n];\n            }\n            if (ref_f64)",
     "                ref = acc * (double)sA[m];\n            }\n            if (ref_f64)", "gemm"),
    ("int8 GEMM pairs k with K-1-k",
     "for (int k = 0; k < K; ++k) acc += (int64_t)(int8_t)a[k] * (int64_t)(int8_t)b[k];",
     "for (int k = 0; k < K; ++k) acc += (int64_t)(int8_t)a[k] * (int64_t)(int8_t)b[K - 1 - k];", "gemm"),
    ("block GEMM takes the next block's weight scale",
     "                    ref += (double)sA[(size_t)m * nbk + kb] * (double)sW[(size_t)(n / 128) * nbk + kb] * part;",
     "                    ref += (double)sA[(size_t)m * nbk + kb] * (double)sW[(size_t)(n / 128) * nbk + (kb + 1) % nbk]"
     " * part;", "gemm"),
    ("block GEMM uses the first token's activation scales",
     "                    ref += (double)sA[(size_t)m * nbk + kb] * (double)sW[(size_t)(n / 128) * nbk + kb] * part;",
     "                    ref += (double)sA[(size_t)(m % 1) * nbk + kb] * (double)sW[(size_t)(n / 128) * nbk + kb]"
     " * part;", "gemm"),
    ("split-K forgets its last chunk",
     "for (int s = 0; s < S; ++s) v += part[s];",
     "for (int s = 0; s < S - 1; ++s) v += part[s];", "gemm"),
    ("Swap-AB writes the transpose untransposed",
     "for (int n = 0; n < N; ++n) ref_f64[(size_t)m * N + n] = outT[(size_t)n * M + m];",
     "for (int n = 0; n < N; ++n) ref_f64[(size_t)m * N + n] = outT[(size_t)m * N + n];", "gemm"),
    ("rotary sine sign flipped",
     "const float lo = y[i] * c - y[half + i] * sn;",
     "const float lo = y[i] * c + y[half + i] * sn;", "qknr"),
    ("rotary sine read from the cosine half",
     "const float c = cs[i], sn = cs[half + i];",
     "const float c = cs[i], sn = cs[i];", "qknr"),
    ("query heads normalised with the key weight",
     "const uint16_t* w = (h < Hq) ? q_weight : k_weight;",
     "const uint16_t* w = k_weight;", "qknr"),
    ("value heads normalised too",
     "if (h >= Hq + Hkv) {",
     "if (h >= Hq + 2 * Hkv) {", "qknr"),
    ("rotary table row by token index",
     "const float* cs = cos_sin + (size_t)p * D;",
     "const float* cs = cos_sin + (size_t)t * D;", "qknr"),
]


# the same for the oracle's Python front end (a mutated copy of the package, imported
# ahead of the original)
PY_MUTANTS = [
    ("grouped GEMM takes the next expert's weights",
     "np.asarray(Wq)[e], np.asarray(sW)[e])",
     "np.asarray(Wq)[(e + 1) % E], np.asarray(sW)[e])"),
    ("grouped GEMM uses the first expert's scales",
     "np.asarray(Wq)[e], np.asarray(sW)[e])",
     "np.asarray(Wq)[e], np.asarray(sW)[0])"),
    ("matmul reference applies the weight scale per token",
     "return (acc * sA.astype(np.float64)[:, None]) * sW.astype(np.float64)[None, :]",
     "return (acc * sA.astype(np.float64)[:, None]) * sW.astype(np.float64)[:acc.shape[0], None]"),
    ("matmul reference takes the next block's weight scale",
     "sc = sA2[:, kb][:, None] * sW2[np.arange(N) // 128, kb][None, :]",
     "sc = sA2[:, kb][:, None] * sW2[np.arange(N) // 128, (kb + 1) % nbk][None, :]"),
    ("grouped GEMM does not slice the token scales",
     "np.asarray(sA)[lo:hi]",
     "np.asarray(sA)[:hi - lo]"),
]


def _build(src_text, path):
    c = path + ".c"
    with open(c, "w") as fh:
        fh.write(src_text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                    "-frounding-math", "-o", path, c, "-lm"], check=True, capture_output=True)
    return path


def _pins(lib, files, pkg_dir=None):
    env = dict(os.environ, W8_ORACLE_LIB=lib)
    cwd = ROOT
    if pkg_dir is not None:
        # the copy first on the path (and not the working directory, which would put the
        # original first)
        env["PYTHONPATH"] = os.pathsep.join([pkg_dir, ROOT])
        cwd = pkg_dir
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                        "--rootdir", ROOT] + [os.path.join(ROOT, f) for f in files],
                       cwd=cwd, env=env, capture_output=True, text=True, timeout=600)
    return p.returncode, p.stdout[-1500:]


def _py_copy(text, path):
    """A copy of the oracle package whose oracle.py is `text`."""
    pkg = os.path.join(path, "oracle")
    os.makedirs(pkg)
    for f in ("__init__.py", "build_oracle.py", "w8_oracle.c"):
        shutil.copy2(os.path.join(ROOT, "oracle", f), pkg)
    with open(os.path.join(pkg, "oracle.py"), "w") as fh:
        fh.write(text)
    return path


def test_planted_mistakes_fail_a_pin(tmp_path):
    src = open(SRC).read()
    jobs = [("unmodified", src, sum(PINS.values(), []), True)]
    for name, old, new, group in MUTANTS:
        assert src.count(old) == 1, "planting site not found (oracle edited?): %s" % name
        jobs.append((name, src.replace(old, new), PINS[group], False))

    py_src = open(os.path.join(ROOT, "oracle", "oracle.py")).read()
    py_jobs = [("unmodified Python front end", py_src, True)]
    for name, old, new in PY_MUTANTS:
        assert py_src.count(old) == 1, "planting site not found (oracle edited?): %s" % name
        py_jobs.append((name, py_src.replace(old, new), False))
    clean_lib = _build(src, str(tmp_path / "clean.so"))

    def run(job):
        name, text, files, clean = job
        if files is None:      # Python front-end mutant, on the unmodified C library
            d = _py_copy(text, str(tmp_path / ("p%d" % abs(hash(name)))))
            rc, out = _pins(clean_lib, PINS["gemm"], d)
        else:
            lib = _build(text, str(tmp_path / ("m%d.so" % abs(hash(name)))))
            rc, out = _pins(lib, files)
        return name, clean, rc, out

    jobs += [(name, text, None, clean) for name, text, clean in py_jobs]

    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(run, jobs))
    survivors, broken = [], []
    for name, clean, rc, out in results:
        if clean:
            if rc != 0:
                broken.append((name, rc, out))
        else:
            # caught = a pin failed on an assertion: exit status 1 and a summary line with
            # "failed" and no "error" (0: all passed; other statuses: a crash or a
            # collection error, which would not show that a pin catches the mistake)
            summary = out.strip().splitlines()[-1] if out.strip() else ""
            if rc != 1 or "failed" not in summary or "error" in summary:
                survivors.append((name, rc, out))
    assert not broken, broken
    assert not survivors, survivors
