"""Mutation check of the CPU oracle's pins (a test-quality tool, not a test).

Each entry below plants one plausible mistake in a scratch copy of
``oracle/bitlinear_oracle.c`` (a dropped eps, a wrong rounding order or mode, a
transposed index, a swapped gamma, a missing residual, ...), rebuilds that copy
and runs the CPU pins (``tests/test_oracle.py``, ``tests/test_tp_ffn.py``)
against it. A pin set is adequate when every mistake makes some pin fail. The
repository's own oracle and tests are never modified.

Two entries are equivalent mutants and are expected to survive: the lower clip of
an int8 code at -128 never binds: with s = 127 / max |x|, every product satisfies
|x * s| <= 127 * (1 + 2^-24)^2 < 127.5, so rint gives codes in
[-127, 127] (``test_quant_act_invariants`` checks that range).

    python tests/oracle_mutations.py --workdir <scratch dir> [name ...]

prints one line per mutation and exits 1 if a mutation that is not expected to
survive passes every pin. It takes a few minutes (each mutation rebuilds the
oracle with gcc and runs the CPU pins).
"""
import argparse
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = ["tests/test_oracle.py", "tests/test_tp_ffn.py"]
EXPECTED_SURVIVORS = {"qa clip -127", "tpdn no lower clip"}

# (name, text in bitlinear_oracle.c, replacement); each text occurs exactly once
MUTATIONS = [
    ('bf16 tie up',
     '(rest == 0x8000u && (keep & 1u))',
     '(rest == 0x8000u)'),
    ('bf16 truncate',
     'if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1u;',
     ''),
    ('absmean n-1',
     'return (float)(s / (double)n);',
     'return (float)(s / (double)(n - 1));'),
    ('absmean no fabs',
     'for (int64_t i = 0; i < n; ++i) s += fabs((double)W[i]);\n    return (float)',
     'for (int64_t i = 0; i < n; ++i) s += ((double)W[i]);\n    return (float)'),
    ('absmean float acc',
     'double s = 0.0;\n    for (int64_t i = 0; i < n; ++i) s += fabs((double)W[i]);\n    return (float)',
     'float s = 0.0f;\n    for (int64_t i = 0; i < n; ++i) s += fabsf(W[i]);\n    return (float)'),
    ('tern no eps',
     'float d = gamma + ORC_W_EPS;',
     'float d = gamma;'),
    ('tern roundf',
     'float r = rintf(W[i] / d);',
     'float r = roundf(W[i] / d);'),
    ('tern no upper clip',
     '        if (r > 1.0f) r = 1.0f;\n        if (r < -1.0f) r = -1.0f;\n        q[i]',
     '        if (r < -1.0f) r = -1.0f;\n        q[i]'),
    ('tern mul',
     'float r = rintf(W[i] / d);',
     'float r = rintf(W[i] * d);'),
    ('pack bit order',
     'b |= code << (2 * i);',
     'b |= code << (2 * (3 - i));'),
    ('pack offset',
     'unsigned code = (unsigned)(q[n * K + 4 * j + i] + 1);',
     'unsigned code = (unsigned)(q[n * K + 4 * j + i] & 3);'),
    ('unpack sign',
     'q[n * K + k] = (int8_t)((int)code - 1);',
     'q[n * K + k] = (int8_t)(1 - (int)code);'),
    ('unpack bad no count',
     '                ++bad;\n',
     ''),
    ('qa no floor',
     'float sm = ORC_QB / fmaxf(amax, ORC_X_EPS);',
     'float sm = ORC_QB / amax;'),
    ('qa roundf',
     'float r = rintf(xr[k] * sm);',
     'float r = roundf(xr[k] * sm);'),
    ('qa clip -127',
     'if (r < -128.0f) r = -128.0f;\n            xq[m * K + k]',
     'if (r < -127.0f) r = -127.0f;\n            xq[m * K + k]'),
    ('qa no fabs',
     'float a = fabsf(xr[k]);',
     'float a = xr[k];'),
    ('qa xsum abs',
     'sum += (int32_t)r;',
     'sum += (int32_t)fabsf(r);'),
    ('qa scale 128',
     'float sm = ORC_QB / fmaxf(amax, ORC_X_EPS);',
     'float sm = 128.0f / fmaxf(amax, ORC_X_EPS);'),
    ('gemm transposed q',
     'for (int64_t k = 0; k < K; ++k) a += (int64_t)q[n * K + k] * (int64_t)xq[m * K + k];',
     'for (int64_t k = 0; k < K; ++k) a += (int64_t)q[k * N + n] * (int64_t)xq[m * K + k];'),
    ('gemmp field',
     'int code = (int)(((unsigned)Wp[n * KB + k / 4] >> (2 * (k % 4))) & 3u);',
     'int code = (int)(((unsigned)Wp[n * KB + k / 4] >> (2 * (3 - k % 4))) & 3u);'),
    ('gemmp offset',
     'a += (int64_t)(code - 1) * (int64_t)xq[m * K + k];',
     'a += (int64_t)(code) * (int64_t)xq[m * K + k];'),
    ('deq inverted',
     'float deq = gamma / s[m];',
     'float deq = s[m] / gamma;'),
    ('deq mul order',
     'float deq = gamma / s[m];\n        for (int64_t n = 0; n < N; ++n) {\n            float v = (float)acc[m * N + n] * deq;',
     'float deq = 1.0f / s[m];\n        for (int64_t n = 0; n < N; ++n) {\n            float v = ((float)acc[m * N + n] * deq) * gamma;'),
    ('deq no residual',
     '            if (residual) v = orc_bf16_to_f32(residual[m * N + n]) + v;\n            if (y32)',
     '            if (y32)'),
    ('rms no eps',
     'float r = 1.0f / sqrtf(ms + ORC_RMS_EPS);\n    for',
     'float r = 1.0f / sqrtf(ms);\n    for'),
    ('rms no mean',
     'float ms = (float)(ss / (double)f);',
     'float ms = (float)(ss);'),
    ('rms float sum',
     'double ss = 0.0;\n    for (int64_t j = 0; j < f; ++j) ss += (double)h[j] * (double)h[j];',
     'float ss = 0.0f;\n    for (int64_t j = 0; j < f; ++j) ss += h[j] * h[j];'),
    ('relu2 no square',
     'return (t * t) * u;',
     'return t * u;'),
    ('relu2 no relu',
     'float t = g > 0.0f ? g : 0.0f;',
     'float t = g;'),
    ('relu2 order',
     'return (t * t) * u;',
     'return t * (t * u);'),
    ('ffn gate gamma swap',
     '        float deqg = gg / s[m];\n        float dequ = gu / s[m];\n        for (int64_t j = 0; j < f; ++j) {',
     '        float deqg = gu / s[m];\n        float dequ = gg / s[m];\n        for (int64_t j = 0; j < f; ++j) {'),
    ('ffn g u swap',
     '            h[m * f + j] = orc_relu2_gate(g, u);',
     '            h[m * f + j] = orc_relu2_gate(u, g);'),
    ('ffn no subln',
     '    orc_quant_act(hn, M, f, q2, s2, NULL);',
     '    orc_quant_act(h, M, f, q2, s2, NULL);'),
    ('ffn no residual',
     '    orc_dequant(accd, gd, s2, M, d, residual, y, NULL);',
     '    orc_dequant(accd, gd, s2, M, d, NULL, y, NULL);'),
    ('ffn gamma down',
     '    orc_dequant(accd, gd, s2, M, d, residual, y, NULL);',
     '    orc_dequant(accd, gg, s2, M, d, residual, y, NULL);'),
    ('ex gamma first',
     '            float deq = gammas[i] / s[m];',
     '            float deq = gammas[0] / s[m];'),
    ('ex gamma last',
     '            float deq = gammas[i] / s[m];',
     '            float deq = gammas[nseg - 1] / s[m];'),
    ('ex no rms',
     '        if (rmsnorm)\n            orc_subln_rms',
     '        if (0)\n            orc_subln_rms'),
    ('ex no residual',
     '                if (residual) v = orc_bf16_to_f32(residual[m * N + n]) + v;\n                y[m * N + n]',
     '                y[m * N + n]'),
    ('rw gamma m',
     '            float deq = gammas[n] / s[m];',
     '            float deq = gammas[m] / s[m];'),
    ('rw gamma 0',
     '            float deq = gammas[n] / s[m];',
     '            float deq = gammas[0] / s[m];'),
    ('rw gamma stride',
     '        gammas[n] = orc_absmean(W + n * K, K);',
     '        gammas[n] = orc_absmean(W + n, K);'),
    ('rw tern wrong gamma',
     '        orc_ternarize(W + n * K, K, gammas[n], q + n * K);',
     '        orc_ternarize(W + n * K, K, gammas[0], q + n * K);'),
    ('rw no residual',
     '            if (residual) v = orc_bf16_to_f32(residual[m * N + n]) + v;\n            y[m * N + n] = orc_f32_to_bf16(v);\n        }\n    }\n    if (acc_out) memcpy(acc_out, acc, sizeof(int32_t) * (size_t)(M * N));\ndone:\n    free(xf); free(xq); free(s); free(acc);',
     '            y[m * N + n] = orc_f32_to_bf16(v);\n        }\n    }\n    if (acc_out) memcpy(acc_out, acc, sizeof(int32_t) * (size_t)(M * N));\ndone:\n    free(xf); free(xq); free(s); free(acc);'),
    ('asum no fabs',
     '    for (int64_t i = 0; i < n; ++i) s += fabs((double)W[i]);\n    return s;',
     '    for (int64_t i = 0; i < n; ++i) s += ((double)W[i]);\n    return s;'),
    ('glob count',
     'float gamma = (float)(total_sum / (double)total_count);',
     'float gamma = (float)(total_sum / (double)(N * K));'),
    ('glob no eps path',
     'float gamma = (float)(total_sum / (double)total_count);\n    orc_ternarize(W, N * K, gamma, q);',
     'float gamma = (float)(total_sum / (double)total_count);\n    orc_ternarize(W, N * K, gamma - ORC_W_EPS, q);'),
    ('tpup hmax no abs',
     '            if (fabsf(hv) > mx) mx = fabsf(hv);',
     '            if (hv > mx) mx = hv;'),
    ('tpup ss float',
     '            acc_ss += (double)hv * (double)hv;',
     '            acc_ss += (double)(hv * hv);'),
    ('tpup gamma swap',
     '        float deqg = gg / s[m];\n        float dequ = gu / s[m];\n        double acc_ss',
     '        float deqg = gu / s[m];\n        float dequ = gg / s[m];\n        double acc_ss'),
    ('tpdn no r in scale',
     'float sm = ORC_QB / fmaxf(hmax_all[m] * r, ORC_X_EPS);',
     'float sm = ORC_QB / fmaxf(hmax_all[m], ORC_X_EPS);'),
    ('tpdn f local',
     'float ms = (float)(ss_all[m] / (double)f_total);',
     'float ms = (float)(ss_all[m] / (double)fl);'),
    ('tpdn order',
     'float v = rintf((h[m * fl + j] * r) * sm);',
     'float v = rintf(h[m * fl + j] * (r * sm));'),
    ('tpdn no eps',
     '        float r = 1.0f / sqrtf(ms + ORC_RMS_EPS);\n        float sm',
     '        float r = 1.0f / sqrtf(ms);\n        float sm'),
    ('bf16 nan dropped',
     '    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);\n',
     ''),
    ('absmean f32 div',
     'return (float)(s / (double)n);',
     'return (float)s / (float)n;'),
    ('pack transposed',
     'Wp[n * KB + j] = (uint8_t)b;',
     'Wp[j * N + n] = (uint8_t)b;'),
    ('unpack field',
     'unsigned code = ((unsigned)Wp[n * KB + k / 4] >> (2 * (k % 4))) & 3u;',
     'unsigned code = ((unsigned)Wp[n * KB + k / 4] >> (2 * (3 - k % 4))) & 3u;'),
    ('qa amax first only',
     '            if (a > amax) amax = a;',
     '            if (k == 0) amax = a;'),
    ('qa x*s via div',
     'float r = rintf(xr[k] * sm);',
     'float r = rintf(xr[k] / (fmaxf(amax, ORC_X_EPS) / ORC_QB));'),
    ('rms rsqrt order',
     'float r = 1.0f / sqrtf(ms + ORC_RMS_EPS);\n    for',
     'float r = sqrtf(1.0f / (ms + ORC_RMS_EPS));\n    for'),
    ('rms hn div',
     'for (int64_t j = 0; j < f; ++j) hn[j] = h[j] * r;',
     'for (int64_t j = 0; j < f; ++j) hn[j] = h[j] / (1.0f / r);'),
    ('rms eps outside',
     'float r = 1.0f / sqrtf(ms + ORC_RMS_EPS);\n    for',
     'float r = 1.0f / (sqrtf(ms) + ORC_RMS_EPS);\n    for'),
    ('rms ms double',
     'float ms = (float)(ss / (double)f);\n    float r = 1.0f / sqrtf(ms + ORC_RMS_EPS);',
     'double ms = ss / (double)f;\n    float r = (float)(1.0 / sqrt(ms + (double)ORC_RMS_EPS));'),
    ('deq residual bf16 first',
     '            if (residual) v = orc_bf16_to_f32(residual[m * N + n]) + v;\n            if (y32)',
     '            if (residual) v = orc_bf16_to_f32(residual[m * N + n]) + orc_bf16_to_f32(orc_f32_to_bf16(v));\n            if (y32)'),
    ('ffn g bf16 rounded',
     '            float g = (float)accg[m * f + j] * deqg;\n            float u = (float)accu[m * f + j] * dequ;\n            h[m * f + j]',
     '            float g = orc_bf16_to_f32(orc_f32_to_bf16((float)accg[m * f + j] * deqg));\n            float u = (float)accu[m * f + j] * dequ;\n            h[m * f + j]'),
    ('ffn h bf16 rounded',
     '            h[m * f + j] = orc_relu2_gate(g, u);',
     '            h[m * f + j] = orc_bf16_to_f32(orc_f32_to_bf16(orc_relu2_gate(g, u)));'),
    ('ffn deq via mul',
     '        float deqg = gg / s[m];\n        float dequ = gu / s[m];\n        for (int64_t j = 0; j < f; ++j) {',
     '        float deqg = gg * (1.0f / s[m]);\n        float dequ = gu * (1.0f / s[m]);\n        for (int64_t j = 0; j < f; ++j) {'),
    ('ex rms eps K',
     '            orc_subln_rms(xf + m * K, K, xn + m * K);',
     '            orc_subln_rms(xf + m * K, K - 1, xn + m * K);'),
    ('ex xn bf16',
     '        if (rmsnorm)\n            orc_subln_rms(xf + m * K, K, xn + m * K);',
     '        if (rmsnorm) {\n            orc_subln_rms(xf + m * K, K, xn + m * K);\n            for (int64_t k = 0; k < K; ++k) xn[m * K + k] = orc_bf16_to_f32(orc_f32_to_bf16(xn[m * K + k]));\n        }'),
    ('tpdn eps clamp r',
     'float sm = ORC_QB / fmaxf(hmax_all[m] * r, ORC_X_EPS);',
     'float sm = ORC_QB / (fmaxf(hmax_all[m], ORC_X_EPS) * r);'),
    ('tpdn no lower clip',
     '            if (v < -128.0f) v = -128.0f;\n            q2[m * fl + j]',
     '            q2[m * fl + j]'),
    ('tpup x not quant whole',
     '    orc_quant_act(xf, M, d, xq, s, NULL);\n    orc_int_gemm_packed(Wg, xq, M, fl, d, accg);',
     '    orc_quant_act(xf, M, d - 4, xq, s, NULL);\n    orc_int_gemm_packed(Wg, xq, M, fl, d, accg);'),
    ('rowwise absmean over N',
     '        gammas[n] = orc_absmean(W + n * K, K);',
     '        gammas[n] = orc_absmean(W, N * K);'),
    ('forward xsum unset',
     '    if (xsum_out) memcpy(xsum_out, xsum, sizeof(int32_t) * (size_t)M);',
     ''),
]


def run_one(workdir: str, src: str, name: str, old: str, new: str) -> bool:
    """Build a scratch tree with one mutation; True when some pin fails."""
    if src.count(old) != 1:
        raise SystemExit(f"{name}: the text to replace occurs {src.count(old)} times")
    d = os.path.join(workdir, name.replace(" ", "_").replace("*", "x").replace("/", "_"))
    if os.path.exists(d):
        shutil.rmtree(d)
    os.makedirs(os.path.join(d, "oracle"))
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), os.path.join(d, "oracle"))
    with open(os.path.join(d, "oracle", "bitlinear_oracle.c"), "w") as f:
        f.write(src.replace(old, new))
    shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(d, "tests"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.symlink(os.path.join(ROOT, "bitlinear_w1_a8_02_b200"), os.path.join(d, "bitlinear_w1_a8_02_b200"))
    r = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-m", "not gpu",
                        "-p", "no:cacheprovider"], cwd=d, capture_output=True, text=True)
    shutil.rmtree(d)
    return r.returncode != 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workdir", required=True, help="scratch directory for the mutated copies")
    ap.add_argument("names", nargs="*", help="run only these mutations")
    args = ap.parse_args()
    os.makedirs(args.workdir, exist_ok=True)
    with open(os.path.join(ROOT, "oracle", "bitlinear_oracle.c")) as f:
        src = f.read()
    bad = []
    for name, old, new in MUTATIONS:
        if args.names and name not in args.names:
            continue
        caught = run_one(args.workdir, src, name, old, new)
        expected = name not in EXPECTED_SURVIVORS
        print(f"{name:28s} {'caught' if caught else 'survived'}"
              f"{'' if caught == expected else '  <-- unexpected'}", flush=True)
        if not caught and expected:
            bad.append(name)
    if bad:
        print("not caught by any pin:", ", ".join(bad))
        sys.exit(1)


if __name__ == "__main__":
    main()
