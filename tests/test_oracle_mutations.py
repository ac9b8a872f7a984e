"""The oracle's pins catch plausible mistakes.  Each case copies moe_oracle.c, plants one mistake
(a dropped term, a wrong sign, bound, index or order, a swapped operand), builds the copy and runs
tests/test_oracle_pins.py against it (oracle/__init__.py loads MOE_ORACLE_LIB instead of its own
build): every mutant must fail a pin, and the unmodified copy must pass.  CPU only; the mistakes
live in temporary copies of the oracle, never in the GPU path."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

# name -> (text in moe_oracle.c, replacement)
MUTATIONS = {
    # MXFP4 decode (OCP MX v1.0 table and packing)
    "high nibble first": ("int code = (k & 1) ? (byte >> 4) : (byte & 15);",
                          "int code = (k & 1) ? (byte & 15) : (byte >> 4);"),
    "scale per 16 elements": ("s[row * (K / 32) + k / 32]", "s[row * (K / 32) + (k / 16) % (K / 32)]"),
    "E8M0 bias 126": ("return ldexp(1.0, byte - 127);", "return ldexp(1.0, byte - 126);"),
    "E2M1 subnormal doubled": ("double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);",
                               "double mag = (e == 0) ? 1.0 * m : ldexp(1.0 + 0.5 * m, e - 1);"),
    "bf16 rounding truncates": ("r = ldexp(nearbyint(m * 256.0), e - 8);", "r = ldexp(floor(m * 256.0), e - 8);"),
    # router
    "ties to the higher id": ("(best < 0 || logits[e] > logits[best])", "(best < 0 || logits[e] >= logits[best])"),
    "no renormalisation": ("w[j] = p[ids[j]] / sel;", "w[j] = p[ids[j]];"),
    "bias ignored": ("if (bias) acc += (double)bias[e];", "if (bias) acc += 0.0;"),
    # route remap
    "unstable scatter": ("    for (int f = 0; f < n; ++f) {\n        int e = topk_ids[f];",
                         "    for (int f = n - 1; f >= 0; --f) {\n        int e = topk_ids[f];"),
    # expert MLP
    "gate and up swapped": ("            g += mx_weight(w13q, w13s, H, n, kk) * xv;\n"
                            "            u += mx_weight(w13q, w13s, H, (long)I + n, kk) * xv;",
                            "            u += mx_weight(w13q, w13s, H, n, kk) * xv;\n"
                            "            g += mx_weight(w13q, w13s, H, (long)I + n, kk) * xv;"),
    "gate clamped below too": ("double a = g < 7.0 ? g : 7.0;", "double a = g < 7.0 ? (g > -7.0 ? g : -7.0) : 7.0;"),
    "up not clamped below": ("double c = u < -7.0 ? -7.0 : (u > 7.0 ? 7.0 : u);", "double c = u > 7.0 ? 7.0 : u;"),
    "silu sign": ("double silu = a / (1.0 + exp(-a));", "double silu = a / (1.0 + exp(a));"),
    # combine
    "slot weights reversed": ("out64[(long)t * H + c] += topk_w[(long)t * k + j] * y[c];",
                              "out64[(long)t * H + c] += topk_w[(long)t * k + (k - 1 - j)] * y[c];"),
}


def _run_pins(lib_path):
    env = dict(os.environ, MOE_ORACLE_LIB=lib_path, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, (r.stdout.strip().splitlines() or [""])[-1]


def _case(tmp, idx, name):
    text = open(SRC).read()
    if name is not None:
        old, new = MUTATIONS[name]
        assert text.count(old) == 1, "mutation site not found: %s" % name
        text = text.replace(old, new)
    src = os.path.join(tmp, "mutant%d.c" % idx)
    open(src, "w").write(text)
    lib = oracle.compile_lib(src, os.path.join(tmp, "mutant%d.so" % idx))
    return name, _run_pins(lib)


def test_every_planted_mistake_fails_a_pin(tmp_path):
    names = [None] + sorted(MUTATIONS)
    with ThreadPoolExecutor(max_workers=max(1, min(8, (os.cpu_count() or 2) // 2))) as pool:
        results = list(pool.map(lambda a: _case(str(tmp_path), *a), enumerate(names)))
    control = results[0][1]
    assert control[0] == 0, "the unmodified copy must pass the pins: %s" % control[1]
    missed = [(n, last) for n, (rc, last) in results[1:] if rc == 0]
    assert not missed, "mistakes no pin catches: %s" % missed
