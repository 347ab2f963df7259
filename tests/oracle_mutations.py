"""Strength check of the oracle's pins: plant one plausible mistake at a time in a temporary copy
of the oracle, run the CPU pin tests against that copy, and report every mistake that no pin
catches.  The working tree is never modified.

    python tests/oracle_mutations.py            # every mutation
    python tests/oracle_mutations.py 3 17       # only these

Each mutation is (file under oracle/, original text, planted text, what the mistake is).  A
mutation that leaves every result unchanged (an equivalent rewrite) does not belong here."""
import os
import shutil
import subprocess
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
C = "sp24_oracle.c"
PY = "__init__.py"
PIN_TESTS = ["tests/test_oracle_pins.py", "tests/test_oracle_nvfp4_library.py"]

MUTATIONS = [
    (C, "if (e == 0) v = ldexp((double)f, -24);", "if (e == 0) v = ldexp((double)f, -25);", "f16 subnormal scale"),
    (C, "else v = ldexp(1.0 + f / 1024.0, e - 15);", "else v = ldexp(1.0 + f / 1024.0, e - 14);", "f16 exponent bias"),
    (C, "else if (e == 31) v = f ? NAN : INFINITY;", "else if (e == 31) v = INFINITY;", "f16 NaN read as inf"),
    (C, "(raw & 0x7fffffffu) : (raw & 0x7fffu)", "(raw & 0x7fffffffu) : (raw & 0xffffu)", "-0 not counted as zero"),
    (C, "int ok = zeros >= 2;", "int ok = zeros > 2;", "check needs three zeros"),
    (C, "(mag[j] == mag[i] && j < i)) rank++;", "(mag[j] == mag[i] && j > i)) rank++;", "prune ties to the higher index"),
    (C, "if (mag[j] > mag[i] ||", "if (mag[j] < mag[i] ||", "prune keeps the smallest"),
    (C, "return ((k * C + (4 * j + i)) * R + r) * S + s;", "return ((k * C + (j + (C / 4) * i)) * R + r) * S + s;",
     "conv groups strided along C"),
    (C, "return ((k * (C / 2) + (2 * j + t)) * R + r) * S + s;",
     "return ((k * (C / 2) + (j + (C / 4) * t)) * R + r) * S + s;", "conv values layout"),
    (C, "meta[g / 2] |= (uint8_t)((g % 2) ? (nib << 4) : nib);", "meta[g / 2] |= (uint8_t)((g % 2) ? nib : (nib << 4));",
     "nibble order within a byte"),
    (C, "int i0 = nib & 3, i1 = nib >> 2;\n    if (i0 >= i1)", "int i0 = nib & 3, i1 = nib >> 2;\n    if (i0 > i1)",
     "decompress accepts i0 == i1"),
    (C, "if (!na && sa != sb) return sa > sb;", "if (!na && sa != sb) return sa < sb;", "4:8 keeps the smallest pairs"),
    (C, "if (na != nb) return na;", "if (na != nb) return nb;", "4:8 NaN score lowest"),
    (C, "int ok = nonzero_pairs <= 2;", "int ok = nonzero_pairs < 2;", "4:8 check too strict"),
    (C, "if (a || b) nonzero_pairs++;", "if (a && b) nonzero_pairs++;", "4:8 pair nonzero when both are"),
    (C, "volatile float sum = a + b;", "volatile float sum = a > b ? a : b;", "4:8 score is the max"),
    (C, "put_raw_bits(values, dtype, 4 * c + 1, raw_bits(w, dtype, 8 * c + 2 * i0 + 1));",
     "put_raw_bits(values, dtype, 4 * c + 1, raw_bits(w, dtype, 8 * c + 2 * i0));", "4:8 second entry of a pair"),
    (C, "if (j == i1) v = raw_bits(values, dtype, 4 * c + 2 + h);", "if (j == i1) v = raw_bits(values, dtype, 4 * c + 2);",
     "4:8 decompress of the second pair"),
    (C, "ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e - 2)", "E2M1 exponent bias"),
    (C, "ldexp(m / 8.0, -6)", "ldexp(m / 8.0, -7)", "E4M3 subnormal scale"),
    (C, "if (mag == 0x7f) return NAN;", "if (mag == 0x7f) return 448.0;", "E4M3 NaN code finite"),
    (C, "if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {", "if (d <= bestd) {",
     "rounding ties away from even"),
    (C, "volatile float s = amax / 2688.0f;", "volatile float s = amax / 2680.0f;", "tensor scale constant"),
    (C, "volatile float d = s_t * 6.0f;", "volatile float d = s_t * 4.0f;", "E2M1 maximum"),
    (C, "if (d != 0.0f) {\n        volatile float q = bmax / d;", "if (d != 0.0f) {\n        volatile float q = bmax / d * 1.0001f;",
     "block-scale quotient slightly off"),
    (C, "volatile float q = fabsf(v) / sc;", "volatile float q = fabsf(v) * (1.0f / sc);", "code quotient by reciprocal"),
    (C, "volatile float sc = (float)sp24o_e4m3_value(sb) * s_t;", "volatile float sc = (float)sp24o_e4m3_value(sb) * s_t * 2.0f;",
     "element divisor"),
    (C, "int code = (signbit(v) ? 8 : 0) | mag;", "int code = (v < 0 ? 8 : 0) | mag;", "sign of -0 dropped"),
    (C, "if (e % 2 == 0) *byte = (uint8_t)((*byte & 0xf0) | code);", "if (e % 2 == 1) *byte = (uint8_t)((*byte & 0xf0) | code);",
     "code nibble order"),
    (C, "    float a = fabsf(elem_f32(t, dtype, i));\n    if (a > amax) amax = a;",
     "    float a = elem_f32(t, dtype, i);\n    if (a > amax) amax = a;", "amax of signed values"),
    (C, "double sb = sp24o_e4m3_value(scales[r * (cols / block) + c / block]);",
     "double sb = sp24o_e4m3_value(scales[r * (cols / block) + c / 16]);", "decode block size"),
    (C, "out[e] = sp24o_e2m1_value(code) * sb * (double)s_t;", "out[e] = sp24o_e2m1_value(code & 7) * sb * (double)s_t;",
     "decode drops the sign"),
    (C, "if (dtype == O_BF16) return bf16_value(((const uint16_t*)p)[i]);",
     "if (dtype == O_BF16) return (double)((const uint16_t*)p)[i];", "bf16 read as an integer"),
    (C, "    if (shape[ndim - 1] % 4) { *err = O_ESHAPE; return 0; }", "    if (shape[0] % 4) { *err = O_ESHAPE; return 0; }",
     "matmul groups along the wrong axis"),
    (C, "return shape[0] * (shape[1] / 4) * shape[2] * shape[3];", "return shape[0] * (shape[1] / 4) * shape[2] * shape[2];",
     "conv group count"),
    (C, "int64_t s = g % S, t = g / S;\n  int64_t r = t % R;", "int64_t s = g % R, t = g / R;\n  int64_t r = t % S;",
     "conv R / S swapped"),
    (C, "aacc += fabs(X[m * K + k]) * fabs(W[n * K + k]);", "aacc += X[m * K + k] * W[n * K + k];", "GEMM tolerance scale signed"),
    (C, "double x0 = X[m * K + 4 * j + i0], x1 = X[m * K + 4 * j + i1];",
     "double x0 = X[m * K + 4 * j + i0], x1 = X[m * K + 4 * j + i0];", "sparse GEMM second index"),
    (C, "acc += x1 * v1;", "acc += x1 * v0;", "sparse GEMM second value"),
    (C, "aacc += fabs(x1) * fabs(v1);", "aacc += fabs(x1) * fabs(v0);", "sparse tolerance scale"),
    (C, "const double* We = W + (int64_t)routing[t * topk + s] * N * K;",
     "const double* We = W + (int64_t)routing[t * topk] * N * K;", "MoE routes every slot to slot 0"),
    (C, "Y[(t * topk + s) * N + n] = acc;", "Y[(t * topk + s) * N + n] = acc * 1.0000001;", "MoE output scaled"),
    (C, "if (routing[i] < 0 || routing[i] >= E) return O_EARG;", "if (routing[i] < 0 || routing[i] > E) return O_EARG;",
     "MoE accepts expert id E"),
    (PY, "h = round_to_16(g / (1.0 + np.exp(-g)) * u, hdtype)", "h = round_to_16(g / (1.0 + np.exp(g)) * u, hdtype)",
     "SiLU sign"),
    (PY, "h = round_to_16(g / (1.0 + np.exp(-g)) * u, hdtype)", "h = g / (1.0 + np.exp(-g)) * u", "h not held in 16 bits"),
    (PY, "S[t] += abs(r) * (np.abs(Wd[e]) @ np.abs(h))", "S[t] += abs(r) * (np.abs(Wd[e]) @ h)", "block tolerance scale signed"),
    (PY, "Y[t] += r * (Wd[e] @ h)", "Y[t] += (Wd[e] @ h)", "router weight dropped"),
    (PY, "r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16", "r = ((u + 0x8000) >> 16) << 16", "bf16 hold ties up"),
    (PY, "    return x.astype(np.float16).astype(np.float64)", "    return x.astype(np.float32).astype(np.float64)",
     "f16 hold skipped"),
    (PY, "return nvfp4_tensor_scale(np.concatenate([f for f in flat if f.size]), dtype)",
     "return nvfp4_tensor_scale(flat[0], dtype)", "group scale from the first tensor only"),
]


def _copy_tree(dst):
    for name in ("oracle", "tests", "synth"):
        shutil.copytree(os.path.join(ROOT, name), os.path.join(dst, name),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    for name in ("conftest.py", "pytest.ini", "pyproject.toml", "setup.cfg"):
        if os.path.exists(os.path.join(ROOT, name)):
            shutil.copy(os.path.join(ROOT, name), dst)


def main(argv):
    only = [int(a) for a in argv]
    survivors = []
    with tempfile.TemporaryDirectory() as tmp:
        _copy_tree(tmp)
        paths = {C: os.path.join(tmp, "oracle", C), PY: os.path.join(tmp, "oracle", PY)}
        orig = {k: open(p).read() for k, p in paths.items()}
        for i, (f, old, new, what) in enumerate(MUTATIONS):
            if only and i not in only:
                continue
            if old not in orig[f]:
                print(f"[{i:2d}] pattern not found ({what})", flush=True)
                survivors.append(i)
                continue
            for k, p in paths.items():
                with open(p, "w") as fh:
                    fh.write(orig[k].replace(old, new, 1) if k == f else orig[k])
            r = subprocess.run([sys.executable, "-m", "pytest", *PIN_TESTS, "-x", "-q", "-p", "no:cacheprovider"],
                               cwd=tmp, capture_output=True, text=True, env={**os.environ, "PYTHONDONTWRITEBYTECODE": "1"})
            caught = r.returncode != 0
            tail = r.stdout.strip().splitlines()[-1] if r.stdout.strip() else ""
            print(f"[{i:2d}] {'caught  ' if caught else 'SURVIVED'} {what} :: {tail}", flush=True)
            if not caught:
                survivors.append(i)
    print(f"{len(survivors)} of {len(only) or len(MUTATIONS)} planted mistakes survived: {survivors}")
    return 1 if survivors else 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
