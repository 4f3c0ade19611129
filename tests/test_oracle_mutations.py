"""The oracle's pins catch plausible mistakes: each case plants one slip in a scratch copy of the
oracle's C source (a dropped term, a wrong constant, operand or index, a reversed order, floor
instead of ceiling, a different rounding rule), rebuilds that copy and runs the pins against it
(tests/test_oracle_pins.py, test_oracle_scaler_clip.py and test_oracle_accounting.py, on the
CPU).  Every planted slip must fail at least one pin.  The
repository's oracle is never modified; the copies live in a temporary directory.

Left out on purpose: letting the Adam loop also update a shard's zero padding (returning the
padded shard length) is an equivalent change -- padding has zero gradient and zero state, which
the update maps to zero -- so no pin can or should catch it."""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (what the slip is, exact text in oracle/zero_oracle.c, planted text)
MUTATIONS = [
    ("eps inside the bias-corrected denominator",
     "float den = sqrtf(vi) / c->sbc2 + c->eps;", "float den = (sqrtf(vi) + c->eps) / c->sbc2;"),
    ("decoupled weight decay dropped",
     "if (c->apply_decay) pi = pi * c->decay;", "(void)0;"),
    ("beta2 used in the first-moment update",
     "float mi = c->beta1 * m[i] + c->omb1 * g[i];", "float mi = c->beta2 * m[i] + c->omb1 * g[i];"),
    ("replicas summed in reverse rank order",
     "for (int q = 0; q < Nd; q++) s = s + grad_value(grads[q], i, dtype);",
     "for (int q = Nd - 1; q >= 0; q--) s = s + grad_value(grads[q], i, dtype);"),
    ("shard length rounded down",
     "if (S * Nd < N) S = S + 1;", "(void)0;"),
    ("bf16 rounding ties away from zero",
     "if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept = kept + 1u;",
     "if (dropped >= 0x8000u) kept = kept + 1u;"),
    ("first-moment bias correction missing",
     "c->step_size = (float)(lr / bc1);", "c->step_size = (float)lr;"),
    ("square root of the second-moment correction missing",
     "c->sbc2 = (float)sqrt(bc2);", "c->sbc2 = (float)bc2;"),
    ("gradient summed, not averaged over ranks",
     "double denom = average ? (double)Nd * ls : ls;", "double denom = ls;"),
    ("overflow check removed",
     "if (!isfinite(g)) *overflow = 1;", "(void)0;"),
    ("fp16 exponent bias off by one",
     "mag = ldexp((double)(1024 + frac), e - 25);", "mag = ldexp((double)(1024 + frac), e - 24);"),
    ("layer gather reads the wrong shard element",
     "if (j < L) full[j] = shards[r][k];", "if (j < L) full[j] = shards[r][k ? k - 1 : 0];"),
    ("second-moment update loses a factor of g",
     "float vi = c->beta2 * v[i] + (c->omb2 * g[i]) * g[i];",
     "float vi = c->beta2 * v[i] + c->omb2 * g[i];"),
    # dynamic loss scale, clipping, the bf16-kept reduced gradient
    ("loss scale grows instead of backing off after an overflow",
     "*scale = *scale * backoff;", "*scale = *scale * growth;"),
    ("loss scale grows one clean step late",
     "if (*good >= interval) {", "if (*good > interval) {"),
    ("loss scale may leave the finite fp32 range",
     "if (grown <= fp32_max) *scale = grown;", "*scale = grown;"),
    ("clipping by the sum of squares instead of the norm",
     "double coef = max_norm / (sqrt(sumsq) + 1e-6);", "double coef = max_norm / (sumsq + 1e-6);"),
    ("clipping factor allowed above 1",
     "if (coef > 1.0) coef = 1.0;", "(void)0;"),
    ("bf16-kept gradient not rounded",
     "float g = oracle_bf16_to_f32(oracle_f32_to_bf16(s * inv));", "float g = s * inv;"),
    # the all-gather and the per-element driver used for full-size sampled checks
    ("all-gather skips the last replica",
     "    for (int dst = 0; dst < Nd; dst++)\n        for (int r = 0; r < Nd; r++)",
     "    for (int dst = 0; dst < Nd - 1; dst++)\n        for (int r = 0; r < Nd; r++)"),
    ("sampled elements read the gradient matrix transposed",
     "for (int q = 0; q < Nd; q++) s = s + grad_value(grads, e * Nd + q, dtype);\n        float g = s * c.inv;\n        if (gout)",
     "for (int q = 0; q < Nd; q++) s = s + grad_value(grads, q * n + e, dtype);\n        float g = s * c.inv;\n        if (gout)"),
    ("sampled elements updated on a skipped step",
     "if (!skip) oracle_adam(p + e, m + e, v + e, &g, 1, &c);", "oracle_adam(p + e, m + e, v + e, &g, 1, &c);"),
    ("sampled elements of the clipping driver updated on a skipped step",
     "float g = (s * c.inv) * coef;\n        if (!skip) oracle_adam(p + e, m + e, v + e, &g, 1, &c);",
     "float g = (s * c.inv) * coef;\n        oracle_adam(p + e, m + e, v + e, &g, 1, &c);"),
    # step bookkeeping, scalars, buckets, norms
    ("bucket windows drop their last element",
     "int64_t hi = lo + w < Np ? lo + w : Np;", "int64_t hi = lo + w - 1 < Np ? lo + w - 1 : Np;"),
    ("weight decay factor without the learning rate",
     "c->decay = (float)(1.0 - lr * wd);", "c->decay = (float)(1.0 - wd);"),
    ("second-moment coefficient from beta1",
     "c->omb2 = (float)(1.0 - b2);", "c->omb2 = (float)(1.0 - b1);"),
    ("sum of squares accumulates g instead of g^2",
     "*sumsq += (double)g * (double)g;", "*sumsq += (double)g;"),
    ("unsharded reference forgets the unscale",
     "g[i] = s * c.inv;\n        if (!isfinite(g[i])) *overflow = 1;", "g[i] = s;\n        if (!isfinite(g[i])) *overflow = 1;"),
    ("clip factor computed but not applied",
     "for (int64_t i = 0; i < N; i++) g[i] = g[i] * coef;", "(void)coef;"),
    # the ZeRO-3 layer layout
    ("ZeRO-3 layers packed without their padding",
     "        off += part[1];\n", "        off += layer_len[l];\n"),
    ("ZeRO-3 bf16 shards not refreshed after the update",
     "for (int64_t k = 0; k < n; k++) shard16[o + k] = oracle_f32_to_bf16(master[o + k]);",
     "(void)n;"),
    # memory and communication accounting
    ("ZeRO-1 counted as partitioning the gradients",
     "double g[4] = {G, G, G / d, G / d};", "double g[4] = {G, G / d, G / d, G / d};"),
    ("ZeRO-3 communication counted like ZeRO-1/2",
     "if (stage == 3) return 3.0 * one;", "if (stage == 3) return 2.0 * one;"),
    ("ring collective volume without the (Nd-1)/Nd factor",
     "double one = (double)(Nd - 1) / (double)Nd * N;", "double one = N;"),
]

PIN_FILES = ["test_oracle_pins.py", "test_oracle_scaler_clip.py", "test_oracle_accounting.py"]


def _run_mutant(k, old, new, base):
    d = os.path.join(base, "m%s" % k)
    os.makedirs(d)
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "*.tmp.*", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "synth"), os.path.join(d, "synth"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    for f in PIN_FILES:
        shutil.copy(os.path.join(ROOT, "tests", f), d)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(d, "golden"))
    src = os.path.join(d, "oracle", "zero_oracle.c")
    text = open(src).read()
    if old is not None:  # None: the unmodified control copy
        assert text.count(old) >= 1, "mutation %d does not apply: %r" % (k, old)
        open(src, "w").write(text.replace(old, new))  # every occurrence (e.g. each reduce loop)
    env = dict(os.environ)
    env.pop("PYTHONPATH", None)
    p = subprocess.run([sys.executable, "-m", "pytest", "--noconftest", "-p", "no:cacheprovider",
                        "-x", "-q", *PIN_FILES], cwd=d, env=env, capture_output=True,
                       text=True, timeout=900)
    return p.returncode, p.stdout[-2000:]


def test_every_planted_slip_fails_a_pin(tmp_path):
    with ThreadPoolExecutor(max_workers=min(len(MUTATIONS) + 1, os.cpu_count() or 4)) as ex:
        control = ex.submit(_run_mutant, "control", None, None, str(tmp_path))
        futs = [ex.submit(_run_mutant, k, old, new, str(tmp_path))
                for k, (_, old, new) in enumerate(MUTATIONS)]
        results = [f.result() for f in futs]
        rc, out = control.result()
    # the unmodified copy passes the same pins the same way, so a failure below is the slip's
    assert rc == 0, "unmodified oracle copy fails its pins (exit %d)\n%s" % (rc, out)
    survivors = []
    for (what, _, _), (rc, out) in zip(MUTATIONS, results):
        # pytest exit code 1: some pin failed (the planted slip was caught); anything else --
        # 0 (all passed) or 2-5 (the run itself broke) -- is not a catch
        if rc != 1:
            survivors.append("%s (pytest exit %d)\n%s" % (what, rc, out))
    assert not survivors, "\n\n".join(survivors)
