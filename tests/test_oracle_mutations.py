"""The pins catch plausible mistakes in the oracle's arithmetic.

Each case plants one mistake in a copy of the oracle (on the CPU, in a
temporary directory) and runs the pins against it: at least one pin must
fail.  Mistakes in the C core are built into a separate library and run
against the numeric pins; mistakes in the Python accounting
(``oracle/plan.py``) go into a copy of the oracle package that the pins
import in place of the real one, and run against the accounting pins.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "zero_oracle.c")

MUTATIONS = {
    "omb1_uses_beta2": ("sc[4] = (float)(1.0 - beta1);", "sc[4] = (float)(1.0 - beta2);"),
    "eps_inside_sqrt": ("float root = sqrtf(v_new);", "float root = sqrtf(v_new + eps);"),
    "no_bias_correction_1": ("sc[6] = (float)(lr / bc1);", "sc[6] = (float)lr;"),
    "no_bias_correction_2": ("sc[7] = (float)(1.0 / sqrt(bc2));", "sc[7] = 1.0f;"),
    "second_moment_missing_g": ("float v_new_part = v_g * g;", "float v_new_part = v_g;"),
    "update_sign": ("float w_new = w_decayed - delta;", "float w_new = w_decayed + delta;"),
    "grad_scale_dropped": ("float g_scaled = g_sum * grad_scale;", "float g_scaled = g_sum;"),
    "sum_starts_at_zero": ("float s = bf16_bits_to_float(grads[e]);\n    for (uint32_t r = 1;",
                           "float s = 0.0f;\n    for (uint32_t r = 0;"),
    "sum_reverse_order": ("float x = bf16_bits_to_float(grads[(uint64_t)r * rank_stride + e]);",
                          "float x = bf16_bits_to_float(grads[(uint64_t)(nd - r) * rank_stride + e]);"),
    "bf16_truncates": ("uint32_t rounded = u + 0x7fffu + lsb;", "uint32_t rounded = u + 0u * lsb;"),
    "bf16_ties_away": ("uint32_t rounded = u + 0x7fffu + lsb;", "uint32_t rounded = u + 0x8000u + 0u * lsb;"),
    "beta1_for_v": ("float v_old = beta2 * (*v);", "float v_old = beta1 * (*v);"),
    "decay_after_update": ("float w_decayed = (*w) * decay;", "float w_decayed = ((*w) - delta) * decay + delta;"),
    "decay_ignores_lr": ("sc[8] = (float)(1.0 - lr * weight_decay);", "sc[8] = (float)(1.0 - weight_decay);"),
    "clip_ignored": ("float g = g_scaled * clip_coef;", "float g = g_scaled;"),
}

# oracle/plan.py: (old, new) -- the byte and element accounting of the step
PLAN_MUTATIONS = {
    "gather_counts_padding": ("return gathers_per_unit * sum(4 * n for n in pl.unit_len)",
                              "return gathers_per_unit * sum(4 * n for n in pl.unit_pad)"),
    "gather_once_per_step": ("def hbm_gather_bytes(pl: Plan, gathers_per_unit: int = 2)",
                             "def hbm_gather_bytes(pl: Plan, gathers_per_unit: int = 1)"),
    "comm_bytes_fp32": ("return 2 * comm_elems_per_rank(pl)", "return 4 * comm_elems_per_rank(pl)"),
    "comm_ring_factor_nd": ("one = (pl.nd - 1) * pl.S", "one = pl.nd * pl.S"),
    "comm_counts_padding_once": ("one = (pl.nd - 1) * pl.S", "one = (pl.nd - 1) * pl.psi // pl.nd"),
    "comm_stage3_one_gather": ("return 3 * one if pl.stage == 3 else 2 * one", "return 2 * one"),
    "hbm_replicas_written_once": ("        per += 2 * pl.nd\n    if with_reduced:",
                                  "        per += 2\n    if with_reduced:"),
}

ACCOUNTING_PINS = "comm or gather or hbm or memory"

NUMERIC_PINS = ("reduce or bf16 or adam or closed_form or constant or zero_gradient "
                "or norm or partitioned or owner_view or clip or guarded or weight_decay")


PIN_FILES = [os.path.join(ROOT, "tests", f) for f in ("test_oracle_pins.py",
                                                     "test_oracle_guard_pins.py")]


def _run_mutant(name, tmp):
    old, new = MUTATIONS[name]
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == 1, name
    mutated = os.path.join(tmp, name + ".c")
    with open(mutated, "w", encoding="utf-8") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(tmp, "lib" + name + ".so")
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
                    mutated, "-o", lib, "-lm"], check=True)
    env = dict(os.environ, ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *PIN_FILES, "-k", NUMERIC_PINS],
                       env=env, cwd=os.path.join(ROOT, "tests"), capture_output=True, text=True,
                       timeout=600)
    return r.returncode, r.stdout[-1500:]


def _run_plan_mutant(name, tmp):
    """Copy of the oracle package with one mistake in plan.py; the pins
    import it through ORACLE_PKG_ROOT and use the real C core."""
    old, new = PLAN_MUTATIONS[name]
    root = os.path.join(tmp, "pkg_" + name)
    pkg = os.path.join(root, "oracle")
    shutil.copytree(os.path.join(ROOT, "oracle"), pkg,
                    ignore=shutil.ignore_patterns("__pycache__", "*.so", "*.tmp.*"))
    src = open(os.path.join(pkg, "plan.py"), encoding="utf-8").read()
    assert src.count(old) == 1, name
    with open(os.path.join(pkg, "plan.py"), "w", encoding="utf-8") as f:
        f.write(src.replace(old, new))
    from oracle import build
    env = dict(os.environ, ORACLE_PKG_ROOT=root, ORACLE_LIB=build.build())
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-k", ACCOUNTING_PINS],
                       env=env, cwd=os.path.join(ROOT, "tests"), capture_output=True, text=True,
                       timeout=600)
    return r.returncode, r.stdout[-1500:]


def test_planted_accounting_mistakes_are_caught(tmp_path):
    names = sorted(PLAN_MUTATIONS)
    workers = max(1, min(len(names), (os.cpu_count() or 2) - 1))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        results = dict(zip(names, ex.map(lambda n: _run_plan_mutant(n, str(tmp_path)), names)))
    survived = {n: out for n, (rc, out) in results.items() if rc != 1}
    assert not survived, survived


def test_planted_mistakes_are_caught(tmp_path):
    names = sorted(MUTATIONS)
    workers = max(1, min(len(names), (os.cpu_count() or 2) - 1))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        results = dict(zip(names, ex.map(lambda n: _run_mutant(n, str(tmp_path)), names)))
    survived = {n: out for n, (rc, out) in results.items() if rc != 1}
    assert not survived, survived
