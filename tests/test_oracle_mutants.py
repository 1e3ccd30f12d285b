"""Mistakes planted in a copy of the CPU oracle must fail its pins.

Each mutant below is one plausible slip in ``oracle/oracle.c`` -- a dropped
term, a wrong sign, index or group, a transposed operand, a swapped input --
applied to a copy of the oracle in a temporary directory.  The pin suite
(``tests/test_oracle_pins.py``) runs against that copy in a child process,
which must fail.  The unchanged copy, run the same way, must pass: so a
failing mutant fails because of its mistake, not because of the set-up.
The oracle in the tree is never touched.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")
PINS = os.path.join("tests", "test_oracle_pins.py")

# (name, text in oracle.c, replacement); each text occurs exactly once.
MUTANTS = [
    # group-affine dequantised product ("FMA-optimised dequantisation kernels")
    ("qgemv: scale and bias swapped",
     "oracle_bf16(s[(size_t)r * ng + j / G]) +\n                 oracle_bf16(b[(size_t)r * ng + j / G]);",
     "oracle_bf16(b[(size_t)r * ng + j / G]) +\n                 oracle_bf16(s[(size_t)r * ng + j / G]);"),
    ("qgemv: scales read column-major",
     "oracle_bf16(s[(size_t)r * ng + j / G]) +\n                 oracle_bf16(b[(size_t)r * ng + j / G]);",
     "oracle_bf16(s[(size_t)(j / G) * rows + r]) +\n                 oracle_bf16(b[(size_t)(j / G) * rows + r]);"),
    ("qgemv: group index one group late",
     "oracle_bf16(s[(size_t)r * ng + j / G]) +\n                 oracle_bf16(b[(size_t)r * ng + j / G]);",
     "oracle_bf16(s[(size_t)r * ng + (j / G + 1) % ng]) +\n"
     "                 oracle_bf16(b[(size_t)r * ng + (j / G + 1) % ng]);"),
    ("qgemv: bias added once per input instead of multiplied by it",
     "      acc += w * x[j];\n      mag += fabs(w * x[j]);",
     "      { double bb = oracle_bf16(b[(size_t)r * ng + j / G]); acc += (w - bb) * x[j] + bb; }\n"
     "      mag += fabs(w * x[j]);"),
    ("qgemv: error scale without absolute values",
     "      mag += fabs(w * x[j]);", "      mag += w * x[j];"),
    # dense product of the router and the shared gate
    ("gemv_f32: matrix read transposed",
     "double t = (double)W[(size_t)r * cols + j] * x[j];",
     "double t = (double)W[(size_t)j * rows + r] * x[j];"),
    # routing ("Understanding Mixture-of-Experts")
    ("topk: ties to the higher index", "else better = le > lb;", "else better = le >= lb;"),
    ("topk: NaN ordered above every number",
     "if (isnan(le)) better = 0;\n      else if (isnan(lb)) better = 1;",
     "if (isnan(le)) better = 1;\n      else if (isnan(lb)) better = 0;"),
    ("topk: NaN logit not reported", "if (isnan(logits[e])) nan_seen = 1;", "if (isnan(logits[e])) nan_seen = 0;"),
    ("topk: softmax of the negated logits", "p[t] = isnan(l) ? 0.0 : exp(l - m);",
     "p[t] = isnan(l) ? 0.0 : exp(m - l);"),
    ("topk: weights not renormalised", "for (int t = 0; t < k; ++t) p[t] /= z;",
     "for (int t = 0; t < k; ++t) p[t] /= z + 1.0;"),
    # activations
    ("sigmoid: sign of the exponent", "return 1.0 / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(z));"),
    ("swiglu: gate and up operands exchanged", "return g * oracle_sigmoid(g) * u;",
     "return u * oracle_sigmoid(u) * g;"),
    ("expert: gate and up matrices exchanged",
     "oracle_qgemv(ex->q, ex->scale, ex->bias, I, H, G, x, g, S_g);\n"
     "  oracle_qgemv(ex->q + n, ex->scale + ng, ex->bias + ng, I, H, G, x, u, S_u);",
     "oracle_qgemv(ex->q, ex->scale, ex->bias, I, H, G, x, u, S_u);\n"
     "  oracle_qgemv(ex->q + n, ex->scale + ng, ex->bias + ng, I, H, G, x, g, S_g);"),
    ("expert: down product on the up outputs",
     "oracle_qgemv(qd, sd, bd, H, I, G, a, y, S_y);", "oracle_qgemv(qd, sd, bd, H, I, G, u, y, S_y);"),
    ("S_a: silu derivative without its g sigmoid' term", "fabs(u[i] * (sg + g[i] * sg * (1.0 - sg)))",
     "fabs(u[i] * sg)"),
    ("S_a: gate and up scales exchanged", "* S_g[i] + fabs(g[i] * sg) * S_u[i];",
     "* S_u[i] + fabs(g[i] * sg) * S_g[i];"),
    ("S_y: down rows without absolute values", "prop += fabs(w) * S_a[j];", "prop += w * S_a[j];"),
    ("S_y: |Wd| read transposed",
     "double w = (double)qd[(size_t)r * I + j] * oracle_bf16(sd[(size_t)r * ngd + j / G]) +\n"
     "                 oracle_bf16(bd[(size_t)r * ngd + j / G]);",
     "double w = (double)qd[(size_t)j * H + r] * oracle_bf16(sd[(size_t)j * (H / G) + r / G]) +\n"
     "                 oracle_bf16(bd[(size_t)j * (H / G) + r / G]);"),
    # combine, residual, shared gate, RMSNorm ("Hand-tuned Metal compute shaders")
    ("combine: residual dropped", "double v = h[i], mag = fabs(h[i]);", "double v = 0.0, mag = fabs(h[i]);"),
    ("combine: shared expert not gated", "    v += gamma * ys;", "    v += ys;"),
    ("combine: gate weights in reverse order", "v += p[t] * yt;", "v += p[k - 1 - t] * yt;"),
    ("rmsnorm: mean over H - 1", "double ms = ss / H;", "double ms = ss / (H - 1);"),
    ("rmsnorm: no square root", "double r = 1.0 / sqrt(ms + eps);", "double r = 1.0 / (ms + eps);"),
    ("rmsnorm: eps outside the root", "double r = 1.0 / sqrt(ms + eps);",
     "double r = 1.0 / (sqrt(ms) + eps);"),
    ("rmsnorm: sum of squares of the residual input instead of h'", "    ss += v * v;",
     "    ss += h[i] * h[i];"),
    ("rmsnorm: norm weight not applied", "xn_out[i] = h_out[i] * r * (double)w[i];",
     "xn_out[i] = h_out[i] * r;"),
    ("S_h: shared gate's error dropped", "mag += fabs(gamma * ys) + fabs(ys) * S_gamma;",
     "mag += fabs(gamma * ys);"),
    ("S_h: expert errors not weighted", "if (S_y) mag += p[t] * S_y[(size_t)t * H + i];",
     "if (S_y) mag += S_y[(size_t)t * H + i];"),
    ("S_xn: error of r without the |h'| weights", "rho += fabs(h_out[i]) * S_h[i];", "rho += S_h[i];"),
    ("S_xn: error of r without 1/H", "rho /= (double)H * (ms + eps);", "rho /= (ms + eps);"),
    ("S_xn: h' error without the factor r", "S_xn[i] = fabs((double)w[i]) * r * S_h[i]",
     "S_xn[i] = fabs((double)w[i]) * S_h[i]"),
    # one layer
    ("layer: router on the residual stream instead of xn",
     "oracle_gemv_f32(L->w_router, E, H, xn, logits, S_l);",
     "oracle_gemv_f32(L->w_router, E, H, h, logits, S_l);"),
    ("layer: shared gate on the residual stream instead of xn",
     "oracle_gemv_f32(L->w_shared_gate, 1, H, xn, &z, &S_z);",
     "oracle_gemv_f32(L->w_shared_gate, 1, H, h, &z, &S_z);"),
    ("layer: experts on the residual stream instead of xn",
     "oracle_expert_ffn(ex, H, I, L->G, xn, g, u, a,", "oracle_expert_ffn(ex, H, I, L->G, h, g, u, a,"),
    ("layer: shared expert taken from slot 0", "int slot = (t < k) ? ids[t] : E;",
     "int slot = (t < k) ? ids[t] : 0;"),
    ("layer: shared gate's error without the sigmoid derivative",
     "double S_gamma = gamma * (1.0 - gamma) * S_z;", "double S_gamma = gamma * S_z;"),
    ("topk: an expert selected twice", "if (ids[u] == e) taken = 1;", "if (ids[u] == e) taken = 0;"),
    ("topk: NaN logit given a weight", "p[t] = isnan(l) ? 0.0 : exp(l - m);", "p[t] = exp(l - m);"),
    ("gemv_f32: error scale without absolute values", "      mag += fabs(t);", "      mag += t;"),
    ("S_y: own terms dropped", "    S_y[r] += prop;", "    S_y[r] = prop;"),
    ("S_h: weighted terms without absolute values", "mag += fabs(p[t] * yt);", "mag += p[t] * yt;"),
    ("S_h: the inputs' slack dropped", "S_h[i] = mag + 1e-2;", "S_h[i] = mag;"),
    ("rmsnorm: normalises the residual input instead of h'", "xn_out[i] = h_out[i] * r * (double)w[i];",
     "xn_out[i] = h[i] * r * (double)w[i];"),
    # quantisers (the offline conversion)
    ("quantize: scale over 2^bits steps", "double sc = (hi - lo) / qmax;", "double sc = (hi - lo) / (qmax + 1);"),
    ("quantize_f32: scale and bias stored in each other's place",
     "    s[g] = oracle_f32_to_bf16(sc);\n    b[g] = oracle_f32_to_bf16(lo);",
     "    s[g] = oracle_f32_to_bf16(lo);\n    b[g] = oracle_f32_to_bf16(sc);"),
    ("quantize: codes truncated instead of rounded", "double c = sc > 0.0 ? nearbyint((w[g0 + j] - lo) / sc) : 0.0;",
     "double c = sc > 0.0 ? floor((w[g0 + j] - lo) / sc) : 0.0;"),
    ("quantize_f32: bf16 ties rounded away from zero", "u += 0x7FFFu + ((u >> 16) & 1u);", "u += 0x8000u;"),
    ("quantize_f32: codes from the unrounded scale and bias",
     "const float t = (x[j] - B) / S;", "const float t = (x[j] - lo) / sc;"),
    ("quantize_f32: code range one too wide", "const int qmax = (1 << bits) - 1;", "const int qmax = (1 << bits);"),
    ("quantize_f32: -0 minimum kept", "lo = lo + 0.0f;", "lo = lo;"),
    ("dequantize: scale and bias swapped",
     "oracle_bf16(s[(size_t)r * ng + j / G]) +\n                                oracle_bf16(b[(size_t)r * ng + j / G]);",
     "oracle_bf16(b[(size_t)r * ng + j / G]) +\n                                oracle_bf16(s[(size_t)r * ng + j / G]);"),
]


def _copy_oracle(dst, src_text):
    """The oracle package with oracle.c replaced by src_text, built."""
    pkg = os.path.join(dst, "oracle")
    os.makedirs(pkg)
    shutil.copy(os.path.join(ORACLE_DIR, "__init__.py"), pkg)
    with open(os.path.join(pkg, "oracle.c"), "w") as f:
        f.write(src_text)
    out = os.path.join(pkg, "liboracle.so")
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
                    os.path.join(pkg, "oracle.c"), "-lm", "-o", out], check=True, capture_output=True)
    return dst


def _run_pins(path):
    """The pin suite with `path` first on the import path: returns
    (exit code, output tail, file of the oracle module it imported)."""
    env = dict(os.environ, PYTHONPATH=os.pathsep.join([path, ROOT]), ORACLE_MUTANT_CHECK="1")
    code = ("import sys, pytest, oracle; print('ORACLE_FILE=' + oracle.__file__); "
            f"sys.exit(pytest.main(['-x', '-q', '-p', 'no:cacheprovider', {PINS!r}]))")
    p = subprocess.run([sys.executable, "-P", "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    where = next((l.split("=", 1)[1] for l in p.stdout.splitlines() if l.startswith("ORACLE_FILE=")), "")
    return p.returncode, p.stdout[-1500:] + p.stderr[-500:], where


def _source():
    with open(os.path.join(ORACLE_DIR, "oracle.c")) as f:
        return f.read()


def test_every_mutant_text_occurs_once():
    src = _source()
    names = [m[0] for m in MUTANTS]
    assert len(set(names)) == len(names)
    for name, old, new in MUTANTS:
        assert src.count(old) == 1, f"{name}: the text to replace occurs {src.count(old)} times"
        assert old != new


@pytest.fixture(scope="module", autouse=True)
def _generator_built():
    """The children share the input generator's library: built once here,
    not by several children at the same time."""
    import synth
    synth.lib()


def test_unchanged_copy_passes_the_pins(tmp_path):
    path = _copy_oracle(str(tmp_path), _source())
    rc, out, where = _run_pins(path)
    assert where.startswith(path), f"the child imported {where}, not the copy"
    assert rc == 0, out


def test_every_planted_mistake_fails_a_pin(tmp_path):
    src = _source()

    def one(i):
        name, old, new = MUTANTS[i]
        path = _copy_oracle(str(tmp_path / f"m{i}"), src.replace(old, new))
        rc, out, where = _run_pins(path)
        return name, rc, out, where, path

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(one, range(len(MUTANTS))))
    survivors = []
    for name, rc, out, where, path in results:
        assert where.startswith(path), f"{name}: the child imported {where}, not the mutant"
        # 1: tests failed; anything else (2 interrupted, 3 internal, 4 usage) is a set-up fault
        assert rc in (0, 1), f"{name}: pytest exit {rc}\n{out}"
        if rc == 0:
            survivors.append(name)
    assert not survivors, f"mistakes no pin catches: {survivors}"
