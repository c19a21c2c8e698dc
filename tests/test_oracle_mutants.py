"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/pa_oracle.c (on the CPU, in
a temporary directory), builds it, and runs the oracle's pin tests against
that copy: at least one pin must fail. The unmodified copy must pass them
all. The mistakes are the kind a restatement of the method could make: a
dropped or misplaced factor, a wrong index or grouping, a wrong rounding rule
or exponent bias, a softmax that is right only without overflow.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle")
PINS = ["tests/test_oracle_decode.py", "tests/test_oracle_codecs.py",
        "tests/test_oracle_append_copy.py", "tests/test_kv_formula.py"]

MUTANTS = [
    ("scale_dropped", "s[k] = (double)scale * dot;", "s[k] = dot;"),
    ("gqa_group_by_modulo", "const int h = i / group;", "const int h = i % num_kv_heads;"),
    ("row_reversed_in_block", "int64_t r = j % block_size;",
     "int64_t r = block_size - 1 - j % block_size;"),
    ("first_table_row_for_all",
     "int64_t blk = block_tables[(int64_t)b * max_blocks_per_seq + j / block_size];",
     "int64_t blk = block_tables[j / block_size];"),
    ("plus_max_in_exponent", "s[k] = exp(s[k] - m);", "s[k] = exp(s[k] + m);"),
    ("max_skips_last_score", "for (int32_t k = 1; k < n; ++k)\n        if (s[k] > m)",
     "for (int32_t k = 1; k < n - 1; ++k)\n        if (s[k] > m)"),
    ("mean_not_softmax_normaliser", "for (int c = 0; c < D; ++c) o[c] /= denom;",
     "for (int c = 0; c < D; ++c) o[c] /= (double)n;"),
    ("window_one_short", "(window > 0 && L > window) ? L - window : 0",
     "(window > 0 && L > window) ? L - window + 1 : 0"),
    ("k_scale_without_head", "kv *= (double)k_scale[h * D + c];", "kv *= (double)k_scale[c];"),
    ("v_scale_missing", "vv *= (double)v_scale[h * D + c];", "vv *= 1.0;"),
    ("f16_bias_14", "v = ldexp(1.0 + (double)m / 1024.0, e - 15);",
     "v = ldexp(1.0 + (double)m / 1024.0, e - 14);"),
    ("bf16_bias_126", "v = ldexp(1.0 + (double)m / 128.0, e - 127);",
     "v = ldexp(1.0 + (double)m / 128.0, e - 126);"),
    ("e4m3_subnormal_step", "v = ldexp((double)m, -9); /* subnormal: m * 2^(1-7-3) */",
     "v = ldexp((double)m, -10); /* subnormal */"),
    ("e4m3_round_half_away", "double r = rint(a / ldexp(1.0, e - 3));",
     "double r = round(a / ldexp(1.0, e - 3));"),
    ("e4m3_sign_dropped", "uint8_t s = signbit(x) ? 0x80 : 0x00;", "uint8_t s = 0x00;"),
    ("e4m3_no_saturation", "if (a >= 448.0) return (uint8_t)(s | 0x7e);",
     "if (a >= 480.0) return (uint8_t)(s | 0x7f);"),
    ("append_channels_reversed",
     "int64_t dst = ((blk * block_size + r) * num_kv_heads + h) * head_dim + c;",
     "int64_t dst = ((blk * block_size + r) * num_kv_heads + h) * head_dim + (head_dim - 1 - c);"),
    ("append_quantises_without_scale", "float yk = xk * k_inv_scale[h * head_dim + c];",
     "float yk = xk;"),
    ("copy_skips_v", "(const char*)v_cache + s * block_bytes",
     "(const char*)v_cache + d * block_bytes"),
    ("kv_formula_one_factor_short", "return 2 * layers * kv_heads", "return layers * kv_heads"),
]


def run_pins(workdir, source: str) -> subprocess.CompletedProcess:
    pkg = workdir / "oracle_copy"
    pkg.mkdir(parents=True)
    shutil.copy(os.path.join(ORACLE, "__init__.py"), pkg / "__init__.py")
    (pkg / "pa_oracle.c").write_text(source)
    env = dict(os.environ, PA_ORACLE_UNDER_TEST=str(pkg))
    return subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q",
                           "-p", "no:cacheprovider"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


def test_every_planted_mistake_fails_a_pin(tmp_path):
    src = open(os.path.join(ORACLE, "pa_oracle.c")).read()
    for name, old, _ in MUTANTS:
        assert src.count(old) == 1, name
    jobs = [("unmodified", src)] + [(name, src.replace(old, new)) for name, old, new in MUTANTS]

    def one(job):
        name, text = job
        r = run_pins(tmp_path / name, text)
        return name, r.returncode, r.stdout[-2000:]

    # one pytest process per copy, several at a time
    with ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
        results = list(ex.map(one, jobs))
    name, rc, out = results[0]
    assert rc == 0, out                                  # the real oracle passes every pin
    # exit status 1: tests ran and at least one failed (not a build or usage error)
    survivors = [(name, rc, out) for name, rc, out in results[1:] if rc != 1]
    assert not survivors, survivors
