"""The oracle's pins catch plausible mistakes: each mutant below is a copy of the oracle with one
planted error (a dropped term, a wrong sign, index or bound, a flipped tie rule, a lost sign of
zero), compiled on the CPU into a temporary library. Every pin of ``test_oracle_pins.py`` is then
run against the mutant, cheapest first, and at least one of them must fail.

The mistakes are planted in a temporary copy only; the oracle itself is never changed. Each
planted text must occur exactly once in the current oracle source, so the list stays tied to it.
No mutant writes outside its own buffers (an out-of-range index would crash the test process
rather than fail a pin), so the mutants change values, comparisons and loop bounds only.
"""
import functools
import importlib.util
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
C_SRC = os.path.join(ROOT, "oracle", "osc_oracle.c")
PY_SRC = os.path.join(ROOT, "oracle", "oracle.py")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (name, file, planted text, replacement): "c" mutants change the C oracle, "py" the Python face
MUTANTS = [
    # Algorithm 1 (§3.1) and the density (§2.2)
    ("event_strict_threshold", "c",
     "return (double)G * best >= (double)alpha * (double)s;",
     "return (double)G * best > (double)alpha * (double)s;"),
    ("event_alpha_and_G_swapped", "c",
     "return (double)G * best >= (double)alpha * (double)s;",
     "return (double)alpha * best >= (double)G * (double)s;"),
    ("event_tie_to_highest_channel", "c",
     "if (a > best) { best = a; jb = j; }",
     "if (a >= best) { best = a; jb = j; }"),
    ("event_on_all_zero_group", "c",
     "if (!(best > 0.0)) return 0;",
     "if (best < 0.0) return 0;"),
    ("hits_tie_to_highest_channel", "c",
     "if (hits[j] > hits[js]) js = j;",
     "if (hits[j] >= hits[js]) js = j;"),
    ("channel_zero_dropped", "c",
     "L[k] = (hits[js] >= (int64_t)min_hits && hits[js] > 0) ? (int8_t)js : (int8_t)-1;",
     "L[k] = (js > 0 && hits[js] >= (int64_t)min_hits) ? (int8_t)js : (int8_t)-1;"),
    ("min_hits_off_by_one", "c",
     "L[k] = (hits[js] >= (int64_t)min_hits && hits[js] > 0) ? (int8_t)js : (int8_t)-1;",
     "L[k] = (hits[js] > (int64_t)min_hits) ? (int8_t)js : (int8_t)-1;"),
    ("hits_not_reset_per_group", "c",
     "memset(hits, 0, (size_t)G * sizeof(int64_t));",
     "(void)0;"),
    ("density_counts_every_token", "c",
     "if (group_event(X + (int64_t)t * K + (int64_t)k * G, G, alpha, &j)) {\n"
     "                n_total[k] += 1;",
     "group_event(X + (int64_t)t * K + (int64_t)k * G, G, alpha, &j);\n"
     "            {\n                n_total[k] += 1;"),
    ("density_hit_ignores_table", "c",
     "if (L[k] >= 0 && j == L[k]) n_hit[k] += 1;",
     "if (L[k] >= 0) n_hit[k] += 1;"),
    # extraction and W_L (§3.2, §3.3)
    ("slot_not_zeroed", "c",
     "Xz[(int64_t)t * K + c] = 0x0000u;",
     "(void)0;"),
    ("slot_zeroed_as_negative_zero", "c",
     "Xz[(int64_t)t * K + c] = 0x0000u;",
     "Xz[(int64_t)t * K + c] = 0x8000u;"),
    ("wl_ignores_table_channel", "c",
     "for (int n = 0; n < N; ++n) WL[(int64_t)n * K_L + pos] = W[(int64_t)n * K + c];",
     "for (int n = 0; n < N; ++n) WL[(int64_t)n * K_L + pos] = W[(int64_t)n * K + k * G];"),
    # microscaling (§3.2; OCP MX E2M1 / E4M3 / E8M0)
    ("exponent_off_by_one", "c",
     "int e = (ex - 1) - emax_elem;",
     "int e = ex - emax_elem;"),
    ("exponent_clamp_low_bound", "c",
     "if (e < -127) e = -127;",
     "if (e < -126) e = -126;"),
    ("zero_block_exponent", "c",
     "if (!(amax > 0.0)) return -127;",
     "if (!(amax > 0.0)) return 0;"),
    ("amax_of_signed_values", "c",
     "double a = fabs(orc_bf16_to_double(x[i]));\n        if (a > amax) amax = a;",
     "double a = orc_bf16_to_double(x[i]);\n        if (a > amax) amax = a;"),
    ("e2m1_wrong_emax", "c",
     "fmt == ORC_FMT_E2M1 ? 2 : 8",
     "fmt == ORC_FMT_E2M1 ? 3 : 8"),
    ("e2m1_subnormal_range", "c",
     "double quantum = (a < 2.0) ? 0.5 : (a < 4.0 ? 1.0 : 2.0);",
     "double quantum = (a < 1.0) ? 0.5 : (a < 4.0 ? 1.0 : 2.0);"),
    ("e2m1_ties_away_from_zero", "c",
     "double q = nearbyint(a / quantum) * quantum;\n    if (q > 6.0) q = 6.0;",
     "double q = round(a / quantum) * quantum;\n    if (q > 6.0) q = 6.0;"),
    ("e2m1_no_saturation", "c",
     "if (q > 6.0) q = 6.0;",
     "(void)0;"),
    ("e2m1_sign_of_zero_lost", "c",
     "uint8_t sign = signbit(v) ? 0x8 : 0x0;",
     "uint8_t sign = (v < 0.0) ? 0x8 : 0x0;"),
    ("e4m3_subnormal_quantum", "c",
     "quantum = ldexp(1.0, -9);",
     "quantum = ldexp(1.0, -10);"),
    ("e4m3_saturates_to_nan", "c",
     "if (q > 448.0) q = 448.0;",
     "if (q > 480.0) q = 480.0;"),
    ("e4m3_ties_away_from_zero", "c",
     "double q = nearbyint(a / quantum) * quantum;\n    if (q > 448.0) q = 448.0;",
     "double q = round(a / quantum) * quantum;\n    if (q > 448.0) q = 448.0;"),
    ("e2m1_decode_subnormal", "c",
     "double mag = (E == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, E - 1);",
     "double mag = (E == 0) ? 1.0 * m : ldexp(1.0 + 0.5 * m, E - 1);"),
    ("e4m3_decode_bias", "c",
     "double mag = (E == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, E - 7);",
     "double mag = (E == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, E - 8);"),
    ("g64_as_two_32_blocks", "c",
     "int blk = (fmt == ORC_FMT_E4M3) ? 32 : G;",
     "int blk = (fmt == ORC_FMT_E4M3) ? 32 : (G > 32 ? 32 : G);"),
    ("dequantize_slot_width", "c",
     "out[(int64_t)t * K + k] = ldexp(d, exps[(int64_t)t * nslot + k / V]);",
     "out[(int64_t)t * K + k] = ldexp(d, exps[(int64_t)t * nslot + k / 32]);"),
    ("bf16_rounding_truncates", "c",
     "double q = nearbyint(a / quantum) * quantum;   /* default mode: ties to even */",
     "double q = floor(a / quantum) * quantum;"),
    # the dual-path product (§3.2, the equation for Y)
    ("compensation_dropped", "c",
     "acc += orc_bf16_to_double(B[(int64_t)t * K_L + i]) *",
     "acc += 0.0 * orc_bf16_to_double(B[(int64_t)t * K_L + i]) *"),
    ("compensation_columns_reversed", "c",
     "acc += orc_bf16_to_double(B[(int64_t)t * K_L + i]) *",
     "acc += orc_bf16_to_double(B[(int64_t)t * K_L + (K_L - 1 - i)]) *"),
    ("scale_exponents_subtracted", "c",
     "acc += ldexp(part, ex[(int64_t)t * nslot + b] + ew[(int64_t)n * nslot + b]);",
     "acc += ldexp(part, ex[(int64_t)t * nslot + b] - ew[(int64_t)n * nslot + b]);"),
    ("weight_scale_of_first_slot", "c",
     "acc += ldexp(part, ex[(int64_t)t * nslot + b] + ew[(int64_t)n * nslot + b]);",
     "acc += ldexp(part, ex[(int64_t)t * nslot + b] + ew[(int64_t)n * nslot]);"),
    ("half_of_each_slot", "c",
     "for (int i = b * V; i < (b + 1) * V; ++i) part += xr[i] * qw[i];",
     "for (int i = b * V; i < b * V + V / 2; ++i) part += xr[i] * qw[i];"),
    ("weights_decoded_as_e2m1", "c",
     "qw[k] = (fmt == ORC_FMT_E2M1) ? orc_decode_e2m1(c) : orc_decode_e4m3(c);",
     "qw[k] = orc_decode_e2m1(c);"),
    # several protected channels per group
    ("multi_round_sees_earlier_channels", "c",
     "for (int t = 0; t < S; ++t) work[(int64_t)t * K + k * G + Lr[k]] = 0x0000u;",
     "(void)0;"),
    ("multi_extract_copies_original", "c",
     "B[(int64_t)t * K_L + pos] = Xz[(int64_t)t * K + c];",
     "B[(int64_t)t * K_L + pos] = X[(int64_t)t * K + c];"),
    ("multi_wl_first_slot_only", "c",
     "int jw = L[(int64_t)k * R + m];",
     "int jw = L[(int64_t)k * R];"),
    ("multi_extract_slot_ignored", "c",
     "int j = L[k * R + m];",
     "int j = L[k * R];"),
    # the RMSNorm step before the quantize (its order of operations is a stated reading)
    ("rms_sum_left_to_right_over_blocks", "c",
     "for (int h = P / 2; h >= 1; h /= 2)\n        for (int b = 0; b < h; ++b) s[b] = s[b] + s[b + h];",
     "for (int b = 1; b < P; ++b) s[0] = s[0] + s[b];"),
    ("rms_block_summed_descending", "c",
     "float v = f32_of_bf16(x[b * 32 + j]);",
     "float v = f32_of_bf16(x[b * 32 + 31 - j]);"),
    ("rms_mean_over_blocks", "c",
     "float mean = total / (float)K;",
     "float mean = total / (float)(K / 32);"),
    ("rms_eps_outside_sqrt", "c",
     "float root = sqrtf(mean + eps);",
     "float root = sqrtf(mean) + eps;"),
    ("rms_gamma_dropped", "c",
     "float b = a * f32_of_bf16(gamma[j]);",
     "float b = a;"),
    ("rms_gamma_reversed", "c",
     "float b = a * f32_of_bf16(gamma[j]);",
     "float b = a * f32_of_bf16(gamma[K - 1 - j]);"),
    ("rms_quantizes_raw_rows", "py",
     "out = osc_forward(Yn, G, L, K_L, cw, ew, WL, rows)",
     "out = osc_forward(X, G, L, K_L, cw, ew, WL, rows)"),
    # the step order of the layer (oracle.py)
    ("quantize_before_extraction", "py",
     "cx, ex = mx_quantize(Xz, G, FMT_E2M1)",
     "cx, ex = mx_quantize(X, G, FMT_E2M1)"),
    ("weights_quantized_with_table_zeroed", "py",
     "cw, ew = mx_quantize(W, G, FMT_E2M1)\n    WL = gather_wl(W, G, L, K_L)",
     "WL = gather_wl(W, G, L, K_L)\n    cw, ew = mx_quantize(extract(W, G, L, K_L)[0], G, FMT_E2M1)"),
    ("fallback_weights_in_e2m1", "py",
     "cw, ew = mx_quantize(W, 32, FMT_E4M3)",
     "cw, ew = mx_quantize(W, 32, FMT_E2M1)"),
]

# pins that take seconds run last, so a mutant is usually caught within milliseconds
_SLOW = ("test_group_size_sweep_roundtrip", "test_density_tiers_follow_table1",
         "test_reconstruction_bound", "test_table_recovers_planted_qkv")


def _load(path, name):
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@functools.lru_cache(maxsize=1)
def _pin_cases():
    pins = _load(PINS, "_pins_for_mutants")
    cases = []
    for name in sorted(n for n in dir(pins) if n.startswith("test_")):
        fn = getattr(pins, name)
        params = [{}]
        for mark in getattr(fn, "pytestmark", []):
            if mark.name == "parametrize":
                argname, values = mark.args[0], mark.args[1]
                params = [dict(p, **{argname: v}) for p in params for v in values]
        cases += [(name, fn, p) for p in params]
    cases.sort(key=lambda c: (c[0] in _SLOW, _SLOW.index(c[0]) if c[0] in _SLOW else 0))
    return tuple(cases)


def _first_failing_pin(face, cases):
    for name, fn, kw in cases:
        try:
            fn(face, **kw)
        except (KeyboardInterrupt, SystemExit):
            raise
        except BaseException as exc:          # AssertionError, ValueError, pytest.raises' Failed
            return f"{name}{kw or ''}: {type(exc).__name__}"
    return None


@pytest.fixture(scope="module")
def mutant_faces(tmp_path_factory):
    """Compile every C mutant at once (gcc, same flags as the oracle) and load a separate copy
    of the oracle's Python face bound to each one."""
    d = tmp_path_factory.mktemp("oracle_mutants")
    c_text, py_text = open(C_SRC).read(), open(PY_SRC).read()
    from oracle import oracle as O
    plain_lib = O.build()
    jobs, faces = [], {}
    for name, kind, old, new in MUTANTS:
        text = c_text if kind == "c" else py_text
        assert text.count(old) == 1, f"{name}: planted text must occur exactly once"
        if kind == "c":
            src, lib = str(d / f"{name}.c"), str(d / f"lib{name}.so")
            open(src, "w").write(c_text.replace(old, new))
            jobs.append((name, src, lib, subprocess.Popen(
                ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                 "-fno-fast-math", "-w", "-o", lib, src, "-lm"])))
        else:
            path = str(d / f"face_{name}.py")
            open(path, "w").write(py_text.replace(old, new))
            face = _load(path, f"_oracle_face_{name}")
            face._SRC, face._LIB = C_SRC, plain_lib
            faces[name] = face
    for name, src, lib, proc in jobs:
        assert proc.wait() == 0, f"{name}: mutant did not compile"
        face = _load(PY_SRC, f"_oracle_face_{name}")
        face._SRC, face._LIB = src, lib
        faces[name] = face
    return faces


def test_unmutated_oracle_passes_every_pin(oracle):
    assert _first_failing_pin(oracle, _pin_cases()) is None


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(mutant_faces, name):
    caught = _first_failing_pin(mutant_faces[name], _pin_cases())
    assert caught is not None, f"no pin fails with the planted mistake '{name}'"
