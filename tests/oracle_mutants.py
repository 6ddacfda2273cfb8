"""Planted mistakes in the CPU oracle, for the mutation test (tests/test_oracle_mutants.py).

Each mutant is one plausible slip in ``oracle/csa2_oracle.c`` (a dropped term, a wrong sign,
bias or index, a transposed operand, an off-by-one in a range, a reversed order), applied to
a copy of the source and compiled with the oracle's own flags.  The oracle pins
(tests/test_oracle_*.py) must fail against every one of them: a mutant that passes them
marks a part of the oracle the pins do not hold down.

Run as a script, it builds every mutant, runs the pin files against each build in this
process (``pytest.main`` with CSA2_ORACLE_LIB pointing at the build) and writes
{name: pytest exit code} as JSON to the path given, with an unmutated copy built and
loaded the same way as the control.  Nothing here touches a GPU.
"""
import concurrent.futures
import json
import os
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
PIN_FILES = [os.path.join(HERE, f) for f in ("test_oracle_formats.py", "test_oracle_pack.py",
                                             "test_oracle_index.py", "test_oracle_attn.py")]

# (name, exact text in csa2_oracle.c, replacement); the first occurrence is replaced
MUTANTS = [
    # element formats
    ("e2m1 exponent bias", "ldexp(1.0 + 0.5 * f, (int)e - 1)", "ldexp(1.0 + 0.5 * f, (int)e - 2)"),
    ("e2m1 sign dropped", "return (code & 8u) ? -mag : mag;", "return mag;"),
    ("e2m1 ties to the odd code", "(d == best_d && (m & 1u) == 0)", "(d == best_d && (m & 1u) == 1)"),
    ("e2m1 saturation at 4", "if (a >= 6.0) return 7u | sign;", "if (a >= 4.0) return 6u | sign;"),
    ("e4m3 exponent bias", "ldexp(1.0 + m / 8.0, (int)e - 7)", "ldexp(1.0 + m / 8.0, (int)e - 8)"),
    ("e4m3 subnormal step", "ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    ("e4m3 saturates to 240", "if (a >= 448.0) return 0x7Eu | sign;", "if (a >= 240.0) return 0x77u | sign;"),
    # packing
    ("kv scale amax/4", "float sf = amax / 6.0f;", "float sf = amax / 4.0f;"),
    ("kv scale from the unrounded quotient", "float qv = x[c] / sd;", "float qv = x[c] / sf;"),
    ("kv nibble order swapped", "out[c / 2] |= (uint8_t)(code << ((c & 1) ? 4 : 0));",
     "out[c / 2] |= (uint8_t)(code << ((c & 1) ? 0 : 4));"),
    ("kv scale byte index", "out[256 + b] = (uint8_t)s;", "out[256 + (b ^ 1)] = (uint8_t)s;"),
    ("kv amax over 15 channels", "for (int i = 0; i < 16; ++i) {\n      float a = fabsf(x[16 * b + i]);",
     "for (int i = 0; i < 15; ++i) {\n      float a = fabsf(x[16 * b + i]);"),
    ("ik scale amax/7", "float s = amax / 6.0f;", "float s = amax / 7.0f;"),
    ("ratio-2 mean drops the second token", "x[c] = (a + b) * 0.5f;", "x[c] = a;"),
    ("ratio-2 sum without the half", "y[d] = (a + b) * 0.5f;", "y[d] = (a + b);"),
    ("kv dequant scale index", "orc_e4m3_value(e[256 + c / 16])", "orc_e4m3_value(e[256 + c / 32])"),
    ("ik dequant nibble order", "unsigned code = (e[d / 2] >> ((d & 1) ? 4 : 0)) & 15u;\n    out[d] = (double)s",
     "unsigned code = (e[d / 2] >> ((d & 1) ? 0 : 4)) & 15u;\n    out[d] = (double)s"),
    # indexer
    ("score without ReLU", "s += (double)w[h] * (dot > 0.0 ? dot : 0.0);", "s += (double)w[h] * dot;"),
    ("score without head weights", "s += (double)w[h] * (dot > 0.0 ? dot : 0.0);",
     "s += (dot > 0.0 ? dot : 0.0);"),
    ("score with the query transposed", "dot += (double)q[h * ORC_DI + d] * k[d];",
     "dot += (double)q[d * HI + h] * k[d];"),
    ("score misses the last dim", "for (int d = 0; d < ORC_DI; ++d) dot += (double)q[h * ORC_DI + d] * k[d];",
     "for (int d = 0; d < ORC_DI - 1; ++d) dot += (double)q[h * ORC_DI + d] * k[d];"),
    ("top-k ties prefer the higher index", "return (x->i < y->i) ? -1 : (x->i > y->i) ? 1 : 0;",
     "return (x->i > y->i) ? -1 : (x->i < y->i) ? 1 : 0;"),
    ("top-k ascending", "if (x->s > y->s) return -1;\n  if (x->s < y->s) return 1;",
     "if (x->s < y->s) return -1;\n  if (x->s > y->s) return 1;"),
    ("full scan sees one entry less", "int64_t n = n_vis[bq];\n    double* sc = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));\n    orc_index_scores",
     "int64_t n = n_vis[bq] - 1;\n    double* sc = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));\n    orc_index_scores"),
    ("full scan ignores the sequence base", "ik_pool + seq_base[b] * ORC_IK_BYTES, n,\n                     sc);\n    topk_labeled(sc, NULL, n, K",
     "ik_pool, n,\n                     sc);\n    topk_labeled(sc, NULL, n, K"),
    ("block score is the first entry", "if (sc[j] > m) m = sc[j];", "if (m == -HUGE_VAL) m = sc[j];"),
    ("block count drops the ragged block", "int64_t nb = (n + block - 1) / block;", "int64_t nb = n / block;"),
    ("reindex ignores visibility", "for (int64_t j = c * block; j < (c + 1) * block && j < n; ++j) {\n        lab[m]",
     "for (int64_t j = c * block; j < (c + 1) * block; ++j) {\n        lab[m]"),
    # attention
    ("window one token too long", "int64_t lo = t - window + 1;", "int64_t lo = t - window;"),
    ("window ignores its buffer start", "int64_t r = u - swa_start[b];", "int64_t r = u;"),
    ("logits without the softmax scale", "logit[i] = sm_scale * dot;", "logit[i] = dot;"),
    ("lse without the max", "lse[bq * H + h] = mx + log(l);", "lse[bq * H + h] = log(l);"),
    ("output not normalised", "for (int c = 0; c < ORC_D; ++c) oh[c] /= l;", ""),
    ("value is the query", "oh[c] += p * keys[(size_t)i * ORC_D + c];", "oh[c] += p * (double)qh[c];"),
    ("empty slots not skipped", "if (j < 0) continue;\n      orc_dequant_kv", "if (j < -1) continue;\n      orc_dequant_kv"),
    # second batch
    ("e4m3 0x7F is a number", "if (e == 15 && m == 7) return NAN;", ""),
    ("e4m3 ties to the odd code", "(d == best_d && (c & 1u) == 0)", "(d == best_d && (c & 1u) == 1)"),
    ("bf16 bits shifted by 15", "uint32_t u = (uint32_t)bits << 16;", "uint32_t u = (uint32_t)bits << 15;"),
    ("ik amax over half the dims", "for (int d = 0; d < ORC_DI; ++d) {\n    float a = fabsf(x[d]);",
     "for (int d = 0; d < ORC_DI / 2; ++d) {\n    float a = fabsf(x[d]);"),
    ("ik nibble order swapped", "out[d / 2] |= (uint8_t)(code << ((d & 1) ? 4 : 0));",
     "out[d / 2] |= (uint8_t)(code << ((d & 1) ? 0 : 4));"),
    ("kv dequant nibble order", "unsigned code = (e[c / 2] >> ((c & 1) ? 4 : 0)) & 15u;",
     "unsigned code = (e[c / 2] >> ((c & 1) ? 0 : 4)) & 15u;"),
    ("ratio-2 mean of the second token twice", "float a = orc_bf16_value(kv[(2 * j) * ORC_D + c]);",
     "float a = orc_bf16_value(kv[(2 * j + 1) * ORC_D + c]);"),
    ("top-k drops its last slot", "    if (k < n) {\n      idx_out[k]", "    if (k < n - 1) {\n      idx_out[k]"),
    ("block score reaches into the next block", "for (int64_t j = c * block; j < (c + 1) * block && j < n; ++j)\n        if (sc[j] > m)",
     "for (int64_t j = c * block; j <= (c + 1) * block && j < n; ++j)\n        if (sc[j] > m)"),
    ("reindex skips block 0", "if (c < 0) continue;\n      for (int64_t j", "if (c <= 0) continue;\n      for (int64_t j"),
    ("window token decoded as e2m1", "keys[(size_t)nk * ORC_D + c] = orc_e4m3_value(row[c]);",
     "keys[(size_t)nk * ORC_D + c] = orc_e2m1_value(row[c] & 15u);"),
    ("window misses the current token", "for (int64_t u = lo; u <= t; ++u) {", "for (int64_t u = lo; u < t; ++u) {"),
    ("softmax without the max shift", "double p = exp(logit[i] - mx);", "double p = exp(logit[i]);"),
    ("window rows ignore the sequence", "const uint8_t* row = swa + ((size_t)b * S_w + (size_t)r) * ORC_D;",
     "const uint8_t* row = swa + ((size_t)r) * ORC_D;"),
    ("entries ignore the sequence base", "orc_dequant_kv(kv_pool + (seq_base[b] + j) * ORC_KV_BYTES",
     "orc_dequant_kv(kv_pool + (j) * ORC_KV_BYTES"),
    # producer: RMSNorm + rotation
    ("norm sums half of each block", "for (int h = 8; h >= 1; h /= 2)", "for (int h = 4; h >= 1; h /= 2)"),
    ("norm mean over 256 channels", "float m = blk[0] / 512.0f;", "float m = blk[0] / 256.0f;"),
    ("norm without eps", "float r = 1.0f / sqrtf(m + eps);", "float r = 1.0f / sqrtf(m);"),
    ("gain ignored", "if (gamma) n[c] = n[c] * gamma[c];", ""),
    ("rotation sign", "y[2 * i] = ac - bs;", "y[2 * i] = ac + bs;"),
    ("rotation pair crossed", "y[2 * i + 1] = as + bc;", "y[2 * i + 1] = bs + ac;"),
    ("rotation table of the next position", "rope_cos + p * (ORC_D / 2), rope_sin + p * (ORC_D / 2)",
     "rope_cos + (p + 1) * (ORC_D / 2), rope_sin + (p + 1) * (ORC_D / 2)"),
    ("bf16 rounding truncates", "return (uint16_t)((u + 0x7FFFu + lsb) >> 16);", "return (uint16_t)(u >> 16);"),
    ("bad position keeps its entry", "    if (zero) {\n      memset(kv_out", "    if (0) {\n      memset(kv_out"),
    # context-parallel decomposition
    ("labeled top-k drops the labels", "p[i].i = labels ? labels[i] : i;", "p[i].i = i;"),
    ("combine without the max shift", "double wc = exp(lse_parts[(int64_t)c * N + r] - mx);",
     "double wc = exp(lse_parts[(int64_t)c * N + r]);"),
    ("combine unnormalised", "for (int d = 0; d < ORC_D; ++d) o[d] /= l;\n    lse[r] = mx + log(l);",
     "lse[r] = mx + log(l);"),
    ("combine lse without the max", "lse[r] = mx + log(l);", "lse[r] = log(l);"),
    ("combine skips the last part", "for (int c = 0; c < C; ++c) {\n      double wc",
     "for (int c = 0; c + 1 < C; ++c) {\n      double wc"),
]


CONTROL = "control (no mutation)"


def mutated_source(src: str, old: str, new: str) -> str:
    if old not in src:
        raise ValueError(f"mutation site not found in the oracle source: {old[:60]!r}")
    return src.replace(old, new, 1)


def build_all(workdir: str) -> dict:
    sys.path.insert(0, ROOT)
    from oracle import build as obuild
    src = open(obuild.SRC).read()
    jobs = {}
    for k, (name, old, new) in enumerate(MUTANTS):
        c = os.path.join(workdir, f"m{k}.c")
        with open(c, "w") as f:
            f.write(mutated_source(src, old, new))
        jobs[name] = (c, os.path.join(workdir, f"libm{k}.so"))
    # control: an unmutated copy, built and loaded the same way, must pass the pins
    c = os.path.join(workdir, "control.c")
    with open(c, "w") as f:
        f.write(src)
    jobs[CONTROL] = (c, os.path.join(workdir, "libcontrol.so"))
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        futs = {ex.submit(obuild.compile_to, c, so): name for name, (c, so) in jobs.items()}
        for f in concurrent.futures.as_completed(futs):
            f.result()
    return {name: so for name, (_, so) in jobs.items()}


def main(out_json: str) -> None:
    import pytest
    sys.path.insert(0, ROOT)
    import oracle
    with tempfile.TemporaryDirectory() as d:
        libs = build_all(d)
        codes = {}
        for name, so in libs.items():
            os.environ["CSA2_ORACLE_LIB"] = so
            oracle._lib = None
            codes[name] = int(pytest.main(["-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                                           "--no-header", "--tb=no", *PIN_FILES]))
        os.environ.pop("CSA2_ORACLE_LIB", None)
        oracle._lib = None
    with open(out_json, "w") as f:
        json.dump(codes, f, indent=1)


if __name__ == "__main__":
    main(sys.argv[1])
